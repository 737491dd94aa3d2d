// Newton-Schulz GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent, warp-specialised kernel runs one of the three products of
// a Newton-Schulz iteration (SignMuon summary, section 2 "Core mechanism"
// item 1: the momentum is orthogonalised toward its polar factor) over every
// (matrix, worker) unit of a launch:
//   stage Gram:   A = X X^T            (X^T X for tall X), symmetric output,
//                                       stored as Q = A + b/(2c) I (c != 0)
//   stage Square: B' = c Q Q + a2 I        (Q = A + b/(2c) I, symmetric, stored
//                                            by the Gram stage in fp16 for the
//                                            diagonal's sake; a2 = a - b^2/(4c):
//                                            the same a I + b A + c A^2)
//   stage Apply:  X' = B' X            (X B' for tall X), i.e. a X + (b A + c A^2) X
// with, in the last iteration, the entrywise sign fused into the epilogue and
// written as packed bits or int8 (steps 2-3 of the summary's flow), or the
// update W <- W - eta U (the optional local polar step, step 5).
// Of the symmetric A and B' only the 256x256 blocks on and above the
// diagonal are computed and stored; the stages that consume them read a
// k-block below the diagonal as the transpose of the stored block.
//
// Two tile modes (chosen per launch by the host from the padding cost):
//   single: one CTA per SM computes a 128x256 tile with
//           tcgen05.mma.cta_group::1 (A 128 rows + B 256 rows per k-block,
//           48 KB stages, 4 stages);
//   pair:   a cluster of two CTAs on two SMs computes a 256x256 tile with
//           tcgen05.mma.cta_group::2 issued by the even CTA; each CTA holds
//           128 rows of A and 128 rows of B (32 KB stages, 6 stages), so each
//           SM streams a third less operand data per FLOP and keeps more
//           k-blocks in flight.  Each CTA loads its own halves (no TMA
//           multicast); the odd CTA's copies complete on the even CTA's
//           barrier, and one multicast commit frees a stage in both CTAs.
//           Launches whose every reduction is at least kLongK long use a
//           seventh stage instead of the epilogue's staging memory and store
//           their 16-bit outputs from registers (the long-reduction layout),
//           on 256x512 tiles (two N = 256 MMAs per K step into the two
//           halves of TMEM, 48 KB stages, 4 stages): a quarter less operand
//           data per FLOP.
// Roles (320 threads per CTA):
//   warp 0     TMA producer: 64x64 bf16 boxes, 128-byte swizzle
//   warp 1     MMA issuer (even CTA of a pair): kind::f16, N=256, K=16,
//              fp32 accumulators in TMEM, double-buffered (2 x 256 cols;
//              on 256x512 tiles the two halves of one accumulator)
//   warps 2-9  epilogue: tcgen05.ld 32x32b, fp32 math, stores (two warps per
//              TMEM lane quadrant, one per half of the accumulator columns)
// Every mbarrier wait is bounded; on timeout the kernel records an error
// code, lets the other roles drain, waits (bounded) for its own copies and
// MMAs, frees TMEM and returns.
#include "common.cuh"

namespace signmuon {

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `bar` with the given parity to complete.  Returns
// false if it did not within limit_ns, or if another role has already given
// up (abort flag set).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t n = 0;
  while (true) {
    if (mbar_test(bar, parity)) return true;
    if ((++n & 63) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t smem_dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// Pair mode: the copy completes on the barrier at `bar`, which may be the
// even CTA's (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t smem_dst, const CUtensorMap* map, uint32_t bar,
                                                 int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrivals that order execution only, with no memory release: an epilogue
// thread signals that it has finished reading an accumulator (its
// tcgen05.ld waited on, then tcgen05.fence::before_thread_sync).  The MMA
// thread reads nothing the epilogue wrote, so a release -- which would
// first wait for the epilogue's outstanding global stores to become
// visible across the cluster -- is not needed.
__device__ __forceinline__ void mbar_arrive_relaxed(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_relaxed_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Bulk tensor store of a 32x32 block from shared memory (async proxy).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until all but the most recent of this thread's bulk store groups
// have read their shared-memory sources.
__device__ __forceinline__ void bulk_wait_read_all_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Wait until this thread's bulk stores have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Make this thread's shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_smem_to_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16-bit conversions of the epilogue outputs (round to nearest even).
__device__ __forceinline__ uint16_t to16(float x, bool half) {
  return half ? __half_as_ushort(__float2half_rn(x)) : __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool half) {
  return (uint32_t)to16(lo, half) | ((uint32_t)to16(hi, half) << 16);
}

// W - eta * u rounded once, to nearest (ties to even), to bf16: the rare
// case of update_bf16 below.  The fp32 value s = fmaf(-eta, u, w) is a bf16
// midpoint; the exact difference lies on one side of it or on it.  In fp64
// p = eta * u is exact, the two-sum rule splits w - p exactly into hi + lo,
// and hi - s is exact (hi and s both lie within an fp32 ulp of the exact
// value), so the side is the sign of hi - s, or of lo when hi == s.
__device__ __noinline__ uint32_t update_bf16_midpoint(float w, float eta, float u, float s) {
  const double wd = (double)w;
  const double p = (double)eta * (double)u;
  const double hi = wd - p;
  const double z = hi - wd;
  const double lo = (wd - (hi - z)) + (-p - z);
  const double diff = hi - (double)s;
  const int side = diff > 0.0 ? 1 : diff < 0.0 ? -1 : (lo > 0.0 ? 1 : (lo < 0.0 ? -1 : 0));
  const uint32_t bits = __float_as_uint(s);
  const uint32_t t = bits >> 16;  // s truncated toward zero: the bf16 neighbour nearer 0
  const bool neg = (bits >> 31) != 0;
  const bool away = side == 0 ? (t & 1u) != 0 : (neg ? side < 0 : side > 0);
  return t + (away ? 1u : 0u);
}

// bf16 W - eta * u with a single rounding of the exact difference.  fmaf
// rounds the exact value to fp32; a bf16 rounding boundary is an fp32 value,
// so that fp32 value rounds to the same bf16 as the exact one unless it is
// itself a bf16 midpoint (low 16 bits 0x8000).
__device__ __forceinline__ __nv_bfloat16 update_bf16(float w, float eta, float u) {
  const float s = fmaf(-eta, u, w);
  if ((__float_as_uint(s) & 0xFFFFu) != 0x8000u || !isfinite(s)) return __float2bfloat16_rn(s);
  return __ushort_as_bfloat16((unsigned short)update_bf16_midpoint(w, eta, u, s));
}

// Byte offset of element (r, c) in a 32x32 16-bit staging block laid out as the
// 64-byte TMA swizzle expects: 64-byte rows, 16-byte chunk index XOR-ed with
// bits 1-2 of the row (the block base is 1 KB aligned).
__device__ __forceinline__ uint32_t stage_off(int r, int c) {
  return (uint32_t)(r * 64 + ((((c >> 3) ^ (r >> 1)) & 3) << 4) + (c & 7) * 2);
}

__device__ __forceinline__ void tensormap_acquire(const CUtensorMap* map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(
                   reinterpret_cast<uint64_t>(map))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Pair mode: one commit arrives on the barrier at the same shared-memory
// offset in both CTAs of the cluster (CTA mask 0b11).
__device__ __forceinline__ void tc_commit_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

template <bool kPair>
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  if constexpr (kPair)
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
  else
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

template <bool kPair>
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  if constexpr (kPair)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <bool kPair>
__device__ __forceinline__ void tmem_alloc(uint32_t slot_addr) {
  if constexpr (kPair) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_addr),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  } else {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_addr),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
}

template <bool kPair>
__device__ __forceinline__ void tmem_dealloc(uint32_t base) {
  if constexpr (kPair)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(kTmemCols) : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(kTmemCols) : "memory");
}

// Issues a 32-lane x 32-column fp32 TMEM load; the registers are valid only
// after tmem_wait_ld on the same array.
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Waits for this thread's outstanding TMEM loads.  The registers are tied to
// the wait so the compiler cannot read them before it.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                 "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                 "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled bf16 operand.
//   K-major:  rows of 64 K-elements (128 B), 8-row atoms of 1 KB stacked
//             along M/N (stride-byte-offset 1 KB); the leading offset is
//             unused for swizzled K-major layouts.
//   MN-major: rows of 64 M/N-elements (128 B) along K, 8-row atoms of 1 KB
//             stacked along K (stride-byte-offset 1 KB), 64-element M/N
//             blocks 8 KB apart (leading-byte-offset 8 KB, one TMA box).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, int mn_major) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(mn_major ? (kBoxBytes >> 4) : 1) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor: D fp32, A and B both bf16 (or both fp16), M = tile_m
// (128, or 256 for a CTA pair), N = 256.
__device__ __forceinline__ uint32_t instr_desc(int a_mn, int b_mn, int tile_m, bool fp16) {
  const uint32_t fmt = fp16 ? 0u : 1u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(tile_m >> 4) << 24);
}

// Per-mode tile and pipeline shape.  kLong (CTA pairs only): launches whose
// every tile has a long reduction (K >= kLongK) store their 16-bit outputs
// straight from registers and give the epilogue's staging memory to a
// seventh pipeline stage.  The mainloop of such tiles is long enough to hide
// the slower stores, and the extra stage covers more of the refill latency
// (the MMA issuer's wait for a stage that has to come back from L2).
//
// kWide (long layout only): a pair tile is 256 x 512, two N = 256 MMAs per
// K step into the two 256-column halves of TMEM, so the accumulator is no
// longer double-buffered: the halves take the place of the two buffers.  Each
// SM then streams 48 KB per 1024 MMA cycles instead of 32 KB per 512 (a
// quarter less operand traffic per FLOP), in four 48 KB stages.
template <bool kPair, bool kLong = false, bool kWide = false>
struct GemmCfg {
  static_assert(kPair || !kLong, "the long-reduction layout is a CTA-pair layout");
  static_assert(kLong || !kWide, "the 256x512 tile is a long-reduction layout");
  static constexpr int kTileM = kPair ? 256 : 128;  // output rows per tile
  static constexpr int kHalves = kWide ? 2 : 1;     // N = 256 accumulators per tile
  static constexpr int kTileN = kHalves * kBN;      // output columns per tile
  static constexpr int kRowsA = 128;                // A-operand rows held by one CTA
  static constexpr int kRowsBH = kPair ? 128 : 256; // B-operand rows per half held by one CTA
  static constexpr int kRowsB = kHalves * kRowsBH;
  static constexpr int kStageA = kRowsA * kBK * 2;
  static constexpr int kStageBH = kRowsBH * kBK * 2;
  static constexpr int kStageB = kRowsB * kBK * 2;
  static constexpr int kStageBytes = kStageA + kStageB;  // 32 KB or 48 KB
  static constexpr int kStages = kPair ? (kWide ? 4 : kLong ? 7 : 6) : 4;
  static constexpr int kStaging = kLong ? 0 : kStagingBytes;
  static constexpr int kSmem = kStages * kStageBytes + kStaging + kBarrierBytes + 1024 /*align*/;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert((2 * kStages + 5) * 8 + 8 <= kBarrierBytes, "barrier area");
};

// ---------------------------------------------------------------------------
// Tile scheduling.  The host lists a launch's tiles as records (unit, tile
// within the unit, shape) -- in unit order, or longest reduction first when
// each CTA gets few tiles; CTA (pair) b takes records b, b + grid,
// b + 2 grid, ...  Every role walks the same sequence.
// ---------------------------------------------------------------------------
// Tile records of one CTA's tiles t0, t0 + stride, ...: the record of the
// tile after the current one is loaded while the current one is processed.
struct RecStream {
  NsTileRec next;
  __device__ __forceinline__ void start(const NsLaunch& L, int t0) {
    if (t0 < L.total_tiles) next = load(L, t0);
  }
  // The record of tile t; issues the load of tile t + stride's.
  __device__ __forceinline__ NsTileRec advance(const NsLaunch& L, int t, int stride) {
    const NsTileRec cur = next;
    if (t + stride < L.total_tiles) next = load(L, t + stride);
    return cur;
  }
  static __device__ __forceinline__ NsTileRec load(const NsLaunch& L, int t) {
    const int4 v = __ldg(reinterpret_cast<const int4*>(L.recs + t));
    return NsTileRec{v.x, v.y, v.z, v.w};
  }
};

struct Tile {
  int M, N, K;
  int m0, n0;
  int a_mn, b_mn, sym;
  int a_up, b_up;  // operand is a symmetric matrix of which only the upper 256-blocks are stored
};

// Symmetric products (A, B') are stored as their 256x256 blocks (I, J)
// with J >= I only.  An operand that is one of them reads k-block
// [k0, k0 + 64) of its rows [r0, r0 + 128) -- all in 256-block r0 / 256 --
// directly when k0 / 256 >= r0 / 256, and otherwise as the transpose of the
// stored block (k0 / 256, r0 / 256): an MN-major box at (x = r0, y = k0).
// Both CTAs of a pair share the decision (their rows lie in one 256-block).
__device__ __forceinline__ int a_major(const Tile& T, int k0) {
  return T.a_mn | (T.a_up & (int)((k0 >> 8) < (T.m0 >> 8)));
}
__device__ __forceinline__ int b_major(const Tile& T, int k0, int n0) {
  return T.b_mn | (T.b_up & (int)((k0 >> 8) < (n0 >> 8)));
}

// Problem dimensions, operand majors and tile origin of local tile li of a
// unit with the given shape.
__device__ __forceinline__ Tile tile_of(int stage, int rows, int cols, int li, int tile_m, int tile_n) {
  const bool tall = rows > cols;
  const int s = tall ? cols : rows, l = tall ? rows : cols;
  Tile T;
  T.a_up = 0; T.b_up = 0;
  if (stage == kStageGram) {
    T.M = s; T.N = s; T.K = l; T.sym = 1; T.a_mn = tall; T.b_mn = tall;
  } else if (stage == kStageSquare) {  // A A: both operands the symmetric A
    T.M = s; T.N = s; T.K = s; T.sym = 1; T.a_mn = 0; T.b_mn = 0; T.a_up = 1; T.b_up = 1;
  } else if (!tall) {  // X' = B' X: A-op = B' (symmetric, K-major), B-op = X (MN-major)
    T.M = rows; T.N = cols; T.K = s; T.sym = 0; T.a_mn = 0; T.b_mn = 1; T.a_up = 1;
  } else {             // X' = X B': A-op = X (K-major), B-op = B' (symmetric, K-major)
    T.M = rows; T.N = cols; T.K = s; T.sym = 0; T.a_mn = 0; T.b_mn = 0; T.b_up = 1;
  }
  const int tiles_n = (T.N + tile_n - 1) / tile_n;
  int tm = 0, tn = 0;
  if (T.sym) {
    // Only the upper 256-blocks of a symmetric output are computed (and
    // stored): row tile tm starts at the column tile holding column
    // tm * tile_m.
    while (true) {
      const int first = tm * tile_m / tile_n;
      const int cnt = tiles_n - first;
      if (li < cnt) { tn = first + li; break; }
      li -= cnt;
      ++tm;
    }
  } else {
    tm = li / tiles_n;
    tn = li - tm * tiles_n;
  }
  T.m0 = tm * tile_m;
  T.n0 = tn * tile_n;
  return T;
}

// Whether the N = 256 half h of a tile (columns n0 + 256 h ..) is computed:
// it starts inside the matrix and, for a symmetric output, on or above the
// diagonal block (the tile's rows lie in one 256-block).  Half 0 of every
// 256-column tile is.
__device__ __forceinline__ bool half_ok(const Tile& T, int h) {
  const int n0 = T.n0 + h * kBN;
  return n0 < T.N && (!T.sym || n0 >= (T.m0 & ~255));
}

// Pair mode, Gram and square stages (the same matrix on both sides),
// diagonal block: each CTA's B rows of the half starting at column n0
// (n0 + 128 rank ..) are its A rows (m0 + 128 rank ..), so that half of B is
// read from the A buffer and not loaded.
template <bool kPair>
__device__ __forceinline__ bool diag_b_from_a(const NsLaunch& L, const Tile& T, int n0) {
  return kPair && L.stage != kStageApply && T.m0 == n0;
}

// Tensor maps of the two operands of a unit's tile.
__device__ __forceinline__ void operand_maps(const NsLaunch& L, const NsUnit* u, bool tall, const CUtensorMap*& ma,
                                             const CUtensorMap*& mb) {
  const CUtensorMap* xin = L.parity ? &u->map_xalt : &u->map_x;
  if (L.stage == kStageGram) {
    ma = xin; mb = xin;
  } else if (L.stage == kStageSquare) {
    ma = &u->map_a; mb = &u->map_a;  // A A (symmetric, K-major rows)
  } else if (!tall) {
    ma = &u->map_b; mb = xin;
  } else {
    ma = xin; mb = &u->map_b;
  }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <bool kPair, bool kLong, bool kWide>
__global__ void __launch_bounds__(kGemmThreads, 1) ns_gemm_kernel(const __grid_constant__ NsLaunch L) {
  using C = GemmCfg<kPair, kLong, kWide>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Stage buffers must be 1 KB aligned for the 128-byte swizzle atoms.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Layout: stage ring | epilogue staging (1 KB aligned) | barriers.
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes + C::kStaging);
  uint64_t* full_bar = bars;                          // [kStages]
  uint64_t* empty_bar = bars + C::kStages;            // [kStages]
  uint64_t* tfull_bar = bars + 2 * C::kStages;        // [2]
  uint64_t* tempty_bar = bars + 2 * C::kStages + 2;   // [2]
  uint64_t* drain_bar = bars + 2 * C::kStages + 4;    // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // Per-epilogue-warp output staging: two 2 KB blocks (1 KB aligned).
  uint8_t* staging = smem + C::kStages * C::kStageBytes;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Pair mode: rank 0 (even CTA) issues the MMAs; both CTAs load and drain.
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const int first_tile = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tile_stride = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_addr(&full_bar[s]), 1);
      mbar_init(smem_addr(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_addr(&tfull_bar[a]), 1);
      mbar_init(smem_addr(&tempty_bar[a]), (kPair ? 2 : 1) * kEpilogueThreads);
    }
    mbar_init(smem_addr(drain_bar), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc<kPair>(smem_addr(tmem_slot));
  tc_fence_before();
  if constexpr (kPair) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  uint32_t issued_kb = 0;  // producer: k-blocks issued (for the exit drain)

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      RecStream rs;
      rs.start(L, first_tile);
      int cur_unit = -1;
      const CUtensorMap* ma = nullptr;
      const CUtensorMap* mb = nullptr;
      for (int t = first_tile; t < L.total_tiles && ok; t += tile_stride) {
        const NsTileRec rec = rs.advance(L, t, tile_stride);
        if (rec.unit != cur_unit) {
          cur_unit = rec.unit;
          operand_maps(L, &L.units[rec.unit], rec.rows > rec.cols, ma, mb);
          tensormap_acquire(ma);
          tensormap_acquire(mb);
        }
        const Tile T = tile_of(L.stage, rec.rows, rec.cols, rec.li, C::kTileM, C::kTileN);
        const int nkb = (T.K + kBK - 1) / kBK;
        const int a_row0 = T.m0 + (int)rank * C::kRowsA;
        // B halves to load: computed, and not read from the A buffer.
        bool load_b[C::kHalves];
        int stage_bytes = C::kStageA;
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) {
          load_b[h] = half_ok(T, h) && !diag_b_from_a<kPair>(L, T, T.n0 + h * kBN);
          if (load_b[h]) stage_bytes += C::kStageBH;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(smem_addr(&empty_bar[stage]), phase ^ 1, abort_flag, L.wait_limit_ns)) {
            atomicCAS(L.err, 0u, (uint32_t)kErrWaitTimeoutProducer);
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (L.withhold_loads) {
            // Fault injection: nothing is armed or copied, so this stage's
            // full barrier never completes and the MMA issuer's wait runs
            // out (no copy is in flight at exit).
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            continue;
          }
          const uint32_t own_full = smem_addr(&full_bar[stage]);
          // Pair mode: both CTAs' copies complete on the even CTA's barrier,
          // which the even CTA arms for both.  On a diagonal block of a
          // symmetric product each CTA's B half is its A half (the same rows
          // of the same matrix), so that B half is not loaded; nor is a half
          // that is not computed.
          if (rank == 0) mbar_arrive_expect_tx(own_full, (kPair ? 2 : 1) * stage_bytes);
          const uint32_t fb = kPair ? map_to_rank(own_full, 0) : own_full;
          const uint32_t sa = smem_addr(smem + stage * C::kStageBytes);
          const int k0 = kb * kBK;
          const int amn = a_major(T, k0);
#pragma unroll
          for (int j = 0; j < C::kRowsA / kBoxRows; ++j) {
            const int mn = a_row0 + j * kBoxRows;
            if constexpr (kPair)
              tma_load_2d_pair(sa + j * kBoxBytes, ma, fb, amn ? mn : k0, amn ? k0 : mn);
            else
              tma_load_2d(sa + j * kBoxBytes, ma, fb, amn ? mn : k0, amn ? k0 : mn);
          }
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {
            if (!load_b[h]) continue;
            const int n0 = T.n0 + h * kBN;
            const int b_row0 = n0 + (int)rank * C::kRowsBH;
            const int bmn = b_major(T, k0, n0);
            const uint32_t sb = sa + C::kStageA + h * C::kStageBH;
#pragma unroll
            for (int j = 0; j < C::kRowsBH / kBoxRows; ++j) {
              const int mn = b_row0 + j * kBoxRows;
              if constexpr (kPair)
                tma_load_2d_pair(sb + j * kBoxBytes, mb, fb, bmn ? mn : k0, bmn ? k0 : mn);
              else
                tma_load_2d(sb + j * kBoxBytes, mb, fb, bmn ? mn : k0, bmn ? k0 : mn);
            }
          }
          ++issued_kb;
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      RecStream rs;
      rs.start(L, first_tile);
      for (int t = first_tile; t < L.total_tiles && ok; t += tile_stride) {
        const NsTileRec rec = rs.advance(L, t, tile_stride);
        const Tile T = tile_of(L.stage, rec.rows, rec.cols, rec.li, C::kTileM, C::kTileN);
        // The square stage multiplies the fp16 A by itself; all others are bf16.
        const bool fp16_ops = L.stage == kStageSquare;
        const int nkb = (T.K + kBK - 1) / kBK;
        if constexpr (kWide) {
          // 256x512 tile: accumulator half h (TMEM columns 256 h ..) takes
          // the barriers of buffer h.  So that draining one half overlaps
          // MMAs into the other, the first (and last) kStages k-blocks issue
          // their half-0 MMAs ahead of their half-1 MMAs: the tile starts as
          // soon as half 0 of the previous tile has been read out, and half 0
          // of this tile is handed to the epilogue while the half-1 MMAs of
          // its last k-blocks still run.  A stage is released once both of
          // its halves' MMAs are issued.
          bool hok[2], bfa[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            hok[h] = half_ok(T, h);
            bfa[h] = diag_b_from_a<kPair>(L, T, T.n0 + h * kBN);
          }
          const int s0 = stage;
          const uint32_t ph0 = phase;
          auto slot = [&](int i) { return (s0 + i) % C::kStages; };
          auto wait_full = [&](int i) {
            const int pos = s0 + i;
            if (!mbar_wait(smem_addr(&full_bar[pos % C::kStages]), ph0 ^ (uint32_t)((pos / C::kStages) & 1),
                           abort_flag, L.wait_limit_ns)) {
              atomicCAS(L.err, 0u, (uint32_t)kErrWaitTimeoutMma);
              *abort_flag = 1;
              return false;
            }
            tc_fence_after();
            return true;
          };
          auto wait_acc = [&](int h) {
            if (!mbar_wait(smem_addr(&tempty_bar[h]), acc_phase ^ 1, abort_flag, L.wait_limit_ns)) {
              atomicCAS(L.err, 0u, (uint32_t)kErrWaitTimeoutMma);
              *abort_flag = 1;
              return false;
            }
            tc_fence_after();
            return true;
          };
          auto issue = [&](int i, int h) {
            if (!hok[h]) return;
            const uint32_t sa = smem_addr(smem + slot(i) * C::kStageBytes);
            const uint32_t sb = bfa[h] ? sa : sa + C::kStageA + h * C::kStageBH;
            const int amn = a_major(T, i * kBK), bmn = b_major(T, i * kBK, T.n0 + h * kBN);
            const uint32_t idesc = instr_desc(amn, bmn, C::kTileM, fp16_ops);
            const uint32_t tmem_d = tmem_base + (uint32_t)(h * kAccCols);
#pragma unroll
            for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
              const uint32_t aoff = amn ? kk * (kUmmaK * 128) : kk * (kUmmaK * 2);
              const uint32_t boff = bmn ? kk * (kUmmaK * 128) : kk * (kUmmaK * 2);
              tc_mma<kPair>(tmem_d, smem_desc(sa + aoff, amn), smem_desc(sb + boff, bmn), idesc, (i | kk) != 0);
            }
          };
          auto release = [&](int i) { tc_commit_both(smem_addr(&empty_bar[slot(i)])); };
          const int P = min(C::kStages, nkb);
          const int E = min(C::kStages, nkb - P);
          ok = wait_acc(0);
          for (int i = 0; ok && i < P; ++i)
            if ((ok = wait_full(i))) issue(i, 0);
          if (ok) ok = wait_acc(1);
          for (int i = 0; ok && i < P; ++i) {
            issue(i, 1);
            release(i);
          }
          for (int i = P; ok && i < nkb - E; ++i) {
            if (!(ok = wait_full(i))) break;
            issue(i, 0);
            issue(i, 1);
            release(i);
          }
          for (int i = nkb - E; ok && i < nkb; ++i)
            if ((ok = wait_full(i))) issue(i, 0);
          if (!ok) break;
          tc_commit_both(smem_addr(&tfull_bar[0]));
          for (int i = nkb - E; i < nkb; ++i) {
            issue(i, 1);
            release(i);
          }
          tc_commit_both(smem_addr(&tfull_bar[1]));
          const int pos = s0 + nkb;
          stage = pos % C::kStages;
          phase = ph0 ^ (uint32_t)((pos / C::kStages) & 1);
          acc_phase ^= 1;
          continue;
        }
        const bool b_from_a = diag_b_from_a<kPair>(L, T, T.n0);
        if (!mbar_wait(smem_addr(&tempty_bar[acc]), acc_phase ^ 1, abort_flag, L.wait_limit_ns)) {
          atomicCAS(L.err, 0u, (uint32_t)kErrWaitTimeoutMma);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + (uint32_t)(acc * kAccCols);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(smem_addr(&full_bar[stage]), phase, abort_flag, L.wait_limit_ns)) {
            atomicCAS(L.err, 0u, (uint32_t)kErrWaitTimeoutMma);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * C::kStageBytes);
          const uint32_t sb = b_from_a ? sa : sa + C::kStageA;
          const int amn = a_major(T, kb * kBK), bmn = b_major(T, kb * kBK, T.n0);
          const uint32_t idesc = instr_desc(amn, bmn, C::kTileM, fp16_ops);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint32_t aoff = amn ? kk * (kUmmaK * 128) : kk * (kUmmaK * 2);
            const uint32_t boff = bmn ? kk * (kUmmaK * 128) : kk * (kUmmaK * 2);
            tc_mma<kPair>(tmem_d, smem_desc(sa + aoff, amn), smem_desc(sb + boff, bmn), idesc,
                          (kb | kk) != 0);
          }
          // The stage is free (in both CTAs of a pair) once these MMAs finish.
          if constexpr (kPair) tc_commit_both(smem_addr(&empty_bar[stage]));
          else tc_commit<kPair>(smem_addr(&empty_bar[stage]));
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        // Accumulator ready for the epilogue (of both CTAs of a pair).
        if constexpr (kPair) tc_commit_both(smem_addr(&tfull_bar[acc]));
        else tc_commit<kPair>(smem_addr(&tfull_bar[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // Drain: wait until every MMA this thread issued has completed.
      tc_commit<kPair>(smem_addr(drain_bar));
      if (!mbar_wait(smem_addr(drain_bar), 0, abort_flag, L.wait_limit_ns)) {
        // Ignore the abort flag for the drain itself: wait out the full limit.
        const uint64_t t0 = global_timer_ns();
        while (!mbar_test(smem_addr(drain_bar), 0)) {
          if (global_timer_ns() - t0 > L.wait_limit_ns) {
            atomicCAS(L.err, 0u, (uint32_t)kErrWaitTimeoutDrain);
            break;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two warps per TMEM lane quadrant: warp w reads lanes 32*(w%4).. and the
    // column half (w-2)/4 of the accumulator.  bf16 outputs (A, B', the next
    // X) are staged per 32x32 block in shared memory and written by TMA
    // stores (whole lines; rows/columns outside the matrix are dropped by the
    // TMA) -- in the long-reduction layout they are stored from registers;
    // the other outputs are stored directly.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int kChunks = kBN / 32 / 2;  // 32-column chunks per warp
    uint8_t* stg0 = staging + (warp - 2) * 2 * kStageBlockBytes;
    uint8_t* stg1 = stg0 + kStageBlockBytes;
    const uint32_t stg0_s = smem_addr(stg0), stg1_s = smem_addr(stg1);
    bool stores_pending = false;  // lane 0 of this warp has bulk stores in flight
    int stage_flip = 0;           // staging block of the next iterate store
    int acc = 0;
    uint32_t acc_phase = 0;
    RecStream rs;
    rs.start(L, first_tile);
    int cur_unit = -1;
    // The unit's fields are copied to registers once per unit: read through
    // a global pointer they would be reloaded after every store (aliasing).
    // Their loads are issued before the wait for the accumulator.
    struct {
      const CUtensorMap* st_out;  // store map of this stage's bf16 output
      void* out;                  // the last apply's output; square stage: the stored fp16 A
      int cols;
      uint8_t* o16;               // long layout: this stage's 16-bit output
      int ld;                     //   and its row stride (elements; square stage: A's)
    } uf = {nullptr, nullptr, 0, nullptr, 0};
    float s = 1.f;
    for (int t = first_tile; t < L.total_tiles; t += tile_stride) {
      const NsTileRec rec = rs.advance(L, t, tile_stride);
      if (rec.unit != cur_unit) {
        cur_unit = rec.unit;
        const NsUnit* un = &L.units[rec.unit];
        uf.st_out = L.stage == kStageGram ? &un->st_a
                  : L.stage == kStageSquare ? &un->st_b
                  : (L.parity ? &un->st_x : &un->st_xalt);
        uf.out = L.stage == kStageSquare ? un->a : un->out;
        uf.ld = L.stage == kStageApply ? un->ld_x : un->ld_s;
        if constexpr (kLong) {
          uf.o16 = static_cast<uint8_t*>(L.stage == kStageGram     ? un->a
                                         : L.stage == kStageSquare ? static_cast<void*>(un->b)
                                         : static_cast<void*>(L.parity ? un->x : un->xalt));
        }
        uf.cols = rec.cols;
        s = L.first ? __ldg(L.scales + rec.unit) : 1.f;
      }
      const Tile T = tile_of(L.stage, rec.rows, rec.cols, rec.li, C::kTileM, C::kTileN);
      // A 256x512 tile is drained as its two 256-column halves, each with the
      // barriers of accumulator buffer h (as two consecutive 256-column tiles).
      bool ep_ok = true;
#pragma unroll 1
      for (int h = 0; h < C::kHalves; ++h) {
        const int n0 = T.n0 + h * kBN;
        if (!mbar_wait(smem_addr(&tfull_bar[acc]), acc_phase, abort_flag, L.wait_limit_ns)) {
          atomicCAS(L.err, 0u, (uint32_t)kErrWaitTimeoutEpilogue);
          *abort_flag = 1;
          ep_ok = false;
          break;
        }
        tc_fence_after();
        const int grow0 = T.m0 + (int)rank * 128 + q * 32;  // first row of this warp's 32-row block
        const int grow = grow0 + lane;
        const bool row_ok = grow < T.M;
        const bool bf16_out = T.sym || L.out_kind == kOutIterate;
        // Chunks of this warp's column half that hold valid columns (warp-uniform).
        const int n_ch = half_ok(T, h) ? max(0, min(kChunks, (T.N - n0 - half * kChunks * 32 + 31) / 32)) : 0;
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kAccCols);
        uint32_t nxt[32];
        if (n_ch > 0) tmem_ld32_async(tbase + (uint32_t)(half * kChunks * 32), nxt);
#pragma unroll 1
        for (int cc = 0; cc < n_ch; ++cc) {
          const int ch = half * kChunks + cc;
          const int gc0 = n0 + ch * 32;
          tmem_wait_ld(nxt);
          uint32_t raw[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) raw[j] = nxt[j];
          // The next chunk's TMEM load overlaps this chunk's math and stores.
          if (cc + 1 < n_ch) tmem_ld32_async(tbase + (uint32_t)((ch + 1) * 32), nxt);
          const int nvalid = min(32, T.N - gc0);
          float v[32];
          if (L.stage == kStageGram) {
            // A, or Q = A + beta I (see NsLaunch::shift).
            const float s2 = s * s;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = fmaf(__uint_as_float(raw[j]), s2, (gc0 + j == grow) ? L.beta : 0.f);
          } else if (L.stage == kStageSquare && L.shift) {
            // B' = c Q Q + a2 I = a I + b A + c A^2 (the accumulator holds Q Q).
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = fmaf(L.c, __uint_as_float(raw[j]), (gc0 + j == grow) ? L.a2 : 0.f);
          } else if (L.stage == kStageSquare) {
            // c == 0, B' = a I + b A (+ c A A): A_ij is read back from the
            // stored fp16 A (this tile's block (I, J), J >= I, is one of the
            // stored upper blocks).
            const __half* arow = static_cast<const __half*>(uf.out) + (int64_t)grow * uf.ld + gc0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint4 w = make_uint4(0u, 0u, 0u, 0u);
              if (row_ok && 8 * k < nvalid) w = *reinterpret_cast<const uint4*>(arow + 8 * k);
              const __half2* h2 = reinterpret_cast<const __half2*>(&w);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float2 f = __half22float2(h2[q]);
                const int j = 8 * k + 2 * q;
                v[j] = fmaf(L.c, __uint_as_float(raw[j]), fmaf(L.b, f.x, (gc0 + j == grow) ? L.a : 0.f));
                v[j + 1] = fmaf(L.c, __uint_as_float(raw[j + 1]), fmaf(L.b, f.y, (gc0 + j + 1 == grow) ? L.a : 0.f));
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = s * __uint_as_float(raw[j]);
          }
          if (bf16_out) {
            // Each 32x32 block is staged in shared memory and written by a TMA
            // store.  The tiles of a symmetric output cover its upper
            // 256-blocks only, which is all that is stored of it (its
            // consumers read the other blocks transposed).
            // The Gram stage's A is fp16, everything else bf16.
            const bool half_out = L.stage == kStageGram;
            {
              if constexpr (kLong) {
                // Straight from registers: each lane writes its row's 32
                // columns (64 bytes) as four 16-byte stores, those starting
                // inside the matrix (the row stride is a multiple of 8, so a
                // store never crosses into the next row).
                if (row_ok) {
                  uint4* dst = reinterpret_cast<uint4*>(uf.o16 + ((int64_t)grow * uf.ld + gc0) * 2);
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) w[j] = pack2(v[8 * k + 2 * j], v[8 * k + 2 * j + 1], half_out);
                    if (8 * k < nvalid) dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
                  }
                }
              } else {
              const CUtensorMap* map = uf.st_out;
              // Stores alternate between the two staging blocks, so only the
              // store before last must have finished reading.
              uint8_t* dst = stg0;
              uint32_t dst_s = stg0_s;
              if (stage_flip ^= 1) { dst = stg1; dst_s = stg1_s; }
              if (stores_pending) {
                if (lane == 0) bulk_wait_read_all_but_one();
                __syncwarp();
              }
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) w[j] = pack2(v[8 * k + 2 * j], v[8 * k + 2 * j + 1], half_out);
                *reinterpret_cast<uint4*>(dst + stage_off(lane, 8 * k)) = make_uint4(w[0], w[1], w[2], w[3]);
              }
              fence_smem_to_async();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(map, dst_s, gc0, grow0);
                bulk_commit();
              }
              stores_pending = true;
              }
            }
          } else if (row_ok) {
            if (L.out_kind == kOutPack1) {
              uint32_t word = 0;
#pragma unroll
              for (int j = 0; j < 32; ++j) word |= (j < nvalid && !(v[j] < 0.f)) ? (1u << j) : 0u;
              const int wpr = (uf.cols + 31) >> 5;
              static_cast<uint32_t*>(uf.out)[(int64_t)grow * wpr + (gc0 >> 5)] = word;
            } else if (L.out_kind == kOutInt8) {
              // A lane writes 32 bytes of its row, in the widest stores the
              // row's alignment allows (the row starts at grow * cols bytes;
              // gc0 is a multiple of 32).
              int8_t* o = static_cast<int8_t*>(uf.out) + (int64_t)grow * uf.cols + gc0;
              uint32_t pk[8];
#pragma unroll
              for (int w = 0; w < 8; ++w) {
                uint32_t x = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) x |= (uint32_t)((v[4 * w + j] < 0.f) ? 0xFFu : 0x01u) << (8 * j);
                pk[w] = x;
              }
              if (nvalid == 32 && (uf.cols & 15) == 0) {
                reinterpret_cast<uint4*>(o)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                reinterpret_cast<uint4*>(o)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
              } else if (nvalid == 32 && (uf.cols & 7) == 0) {
#pragma unroll
                for (int w = 0; w < 4; ++w) reinterpret_cast<uint2*>(o)[w] = make_uint2(pk[2 * w], pk[2 * w + 1]);
              } else if (nvalid == 32 && (uf.cols & 3) == 0) {
#pragma unroll
                for (int w = 0; w < 8; ++w) reinterpret_cast<uint32_t*>(o)[w] = pk[w];
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nvalid) o[j] = v[j] < 0.f ? int8_t(-1) : int8_t(1);
              }
            } else if (L.out_kind == kOutUF32) {
              float* o = static_cast<float*>(uf.out) + (int64_t)grow * uf.cols + gc0;
              if (nvalid == 32 && (uf.cols & 3) == 0) {
#pragma unroll
                for (int w = 0; w < 8; ++w)
                  reinterpret_cast<float4*>(o)[w] = make_float4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nvalid) o[j] = v[j];
              }
            } else {  // kOutUpdateW: W <- W - eta * U
              // 16-byte vectors when the row is aligned for them; the loads
              // are all issued before the stores.
              const int64_t off = (int64_t)grow * uf.cols + gc0;
              if (L.w_dtype == SIGNMUON_BF16) {
                __nv_bfloat16* w = static_cast<__nv_bfloat16*>(uf.out) + off;
                if (nvalid == 32 && (uf.cols & 7) == 0) {
                  uint4 raw[4];
#pragma unroll
                  for (int q4 = 0; q4 < 4; ++q4) raw[q4] = reinterpret_cast<const uint4*>(w)[q4];
#pragma unroll
                  for (int q4 = 0; q4 < 4; ++q4) {
                    __nv_bfloat16* e = reinterpret_cast<__nv_bfloat16*>(&raw[q4]);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                      e[j] = update_bf16(__bfloat162float(e[j]), L.eta, v[8 * q4 + j]);
                    reinterpret_cast<uint4*>(w)[q4] = raw[q4];
                  }
                } else {
#pragma unroll
                  for (int j = 0; j < 32; ++j)
                    if (j < nvalid) w[j] = update_bf16(__bfloat162float(w[j]), L.eta, v[j]);
                }
              } else {
                float* w = static_cast<float*>(uf.out) + off;
                if (nvalid == 32 && (uf.cols & 3) == 0) {
#pragma unroll
                  for (int h = 0; h < 2; ++h) {  // two halves of 16 weights (register pressure)
                    float4 x[4];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) x[q4] = reinterpret_cast<const float4*>(w)[4 * h + q4];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                      const int j = 16 * h + 4 * q4;
                      x[q4].x = fmaf(-L.eta, v[j + 0], x[q4].x);
                      x[q4].y = fmaf(-L.eta, v[j + 1], x[q4].y);
                      x[q4].z = fmaf(-L.eta, v[j + 2], x[q4].z);
                      x[q4].w = fmaf(-L.eta, v[j + 3], x[q4].w);
                      reinterpret_cast<float4*>(w)[4 * h + q4] = x[q4];
                    }
                  }
                } else {
#pragma unroll
                  for (int j = 0; j < 32; ++j)
                    if (j < nvalid) w[j] = fmaf(-L.eta, v[j], w[j]);
                }
              }
            }
          }
        }
        tc_fence_before();
        if constexpr (kPair)
          mbar_arrive_relaxed_cluster(map_to_rank(smem_addr(&tempty_bar[acc]), 0));  // the even CTA's barrier
        else
          mbar_arrive_relaxed(smem_addr(&tempty_bar[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (!ep_ok) break;
    }
    // All of this warp's bulk stores must complete before the CTA exits.
    if (lane == 0 && stores_pending) bulk_wait_all();
    __syncwarp();
  }

  // ------------------------------------------------------------------ exit
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && issued_kb > 0) {
    // Wait (bounded) for every TMA copy this CTA issued.  The even CTA checks
    // that the last phase armed on each stage's full barrier completed; the
    // odd CTA (whose copies complete on the even CTA's barriers) waits until
    // its last load of each stage has been consumed.
    for (int s = 0; s < C::kStages; ++s) {
      if (issued_kb <= (uint32_t)s) continue;
      const uint32_t last_round = (issued_kb - 1 - s) / C::kStages;
      const uint32_t bar = rank == 0 ? smem_addr(&full_bar[s]) : smem_addr(&empty_bar[s]);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_test(bar, last_round & 1)) {
        if (global_timer_ns() - t0 > L.wait_limit_ns) {
          atomicCAS(L.err, 0u, (uint32_t)kErrWaitTimeoutDrain);
          break;
        }
      }
    }
  }
  tc_fence_before();
  if constexpr (kPair) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc<kPair>(tmem_base);
  }
}

static int g_num_sms[64] = {0};

cudaError_t launch_ns_gemm(const NsLaunch& p, cudaStream_t stream) {
  if (p.total_tiles <= 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_num_sms[dev] == 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ns_gemm_kernel<false, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<false, false, false>::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ns_gemm_kernel<true, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<true, false, false>::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ns_gemm_kernel<true, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<true, true, false>::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ns_gemm_kernel<true, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<true, true, true>::kSmem);
    if (e != cudaSuccess) return e;
    g_num_sms[dev] = n;
  }
  const int sms = g_num_sms[dev];
  if (!p.pair) {
    const int grid = p.total_tiles < sms ? p.total_tiles : sms;
    ns_gemm_kernel<false, false, false><<<grid, kGemmThreads, GemmCfg<false, false, false>::kSmem, stream>>>(p);
    return cudaGetLastError();
  }
  // One cluster of two CTAs per pair tile worker.
  const int pairs = p.total_tiles < sms / 2 ? p.total_tiles : sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = p.wide     ? GemmCfg<true, true, true>::kSmem
                         : p.long_k ? GemmCfg<true, true, false>::kSmem
                                    : GemmCfg<true, false, false>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.wide) return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<true, true, true>, p);
  if (p.long_k) return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<true, true, false>, p);
  return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<true, false, false>, p);
}

}  // namespace signmuon
