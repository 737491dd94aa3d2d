// C ABI of libsignmuon.so: argument validation, workspace layout, descriptor
// planning (tensor maps, unit tables) and kernel launches.  The declarations
// and their contracts are in include/signmuon.h.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"

using namespace signmuon;

namespace {

constexpr int kAbiVersion = 1;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int64_t wpr_of(int32_t cols) { return (cols + 31) / 32; }
inline int64_t packed_words_of(signmuon_shape s) { return ((int64_t)s.rows * wpr_of(s.cols) + 3) / 4 * 4; }

signmuon_status validate_shapes(const signmuon_shape* shapes, int n_mats) {
  if (!shapes || n_mats <= 0) return SIGNMUON_ERR_INVALID_ARG;
  for (int i = 0; i < n_mats; ++i)
    if (shapes[i].rows <= 0 || shapes[i].cols <= 0) return SIGNMUON_ERR_INVALID_ARG;
  return SIGNMUON_OK;
}

signmuon_status validate_ptrs(const void* const* p, int n, bool allow_null = false) {
  if (!p) return SIGNMUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (!p[i]) {
      if (allow_null) continue;
      return SIGNMUON_ERR_INVALID_ARG;
    }
    if (!aligned16(p[i])) return SIGNMUON_ERR_ALIGNMENT;
  }
  return SIGNMUON_OK;
}

signmuon_status check_workspace(void* ws, size_t have, size_t need) {
  if (!ws) return SIGNMUON_ERR_WORKSPACE;
  if (!aligned16(ws) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SIGNMUON_ERR_ALIGNMENT;
  if (have < need) return SIGNMUON_ERR_WORKSPACE;
  return SIGNMUON_OK;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// ----------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D 16-bit tensor [outer, inner] (bf16, or fp16 for A and P) with row
// stride ld elements.  Operand maps:
// 64x64 boxes, 128-byte swizzle, zero fill outside the tensor.  Store maps:
// 32x32 boxes, 64-byte swizzle (writes outside the tensor are dropped).
bool encode_bf16_2d(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld,
                    bool store_box = false, bool fp16 = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {store_box ? 32u : 64u, store_box ? 32u : 64u};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, store_box ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ----------------------------------------------------------------- NS planning
// Per-unit workspace: Gram A (s x s fp16), B' = aI + bA + cA^2 (s x s bf16)
// and the second X iterate (bf16).
struct UnitBytes {
  size_t a, xalt, total;
};

UnitBytes ns_unit_bytes(signmuon_shape sh) {
  const int64_t s = std::min(sh.rows, sh.cols);
  const int64_t ld_s = x_ld_of((int32_t)s);
  UnitBytes u;
  u.a = align_up((size_t)(s * ld_s * 2), 1024);
  u.xalt = align_up((size_t)sh.rows * x_ld_of(sh.cols) * 2, 1024);
  u.total = 2 * u.a + u.xalt;
  return u;
}

// Tiles of one unit in one stage; pair = 1 for 256x256 CTA-pair tiles,
// wide = 1 (pairs only) for 256x512 ones.
int ns_tiles(int rows, int cols, int stage, int pair, int wide = 0) {
  const bool tall = rows > cols;
  const int s = tall ? cols : rows;
  const int bm = ns_tile_m(pair);
  const int bn = wide ? 2 * kBN : kBN;
  if (stage == kStageApply) {
    return ((rows + bm - 1) / bm) * ((cols + bn - 1) / bn);
  }
  // Symmetric outputs: row tile i starts at the column tile holding column i * bm.
  const int tm = (s + bm - 1) / bm, tn = (s + bn - 1) / bn;
  int n = 0;
  for (int i = 0; i < tm; ++i) n += tn - i * bm / bn;
  return n;
}

// SMs of the current device (148 on B200; 148 if the query fails).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0)
    return 148;
  return n;
}

size_t ns_desc_bytes(int n_units) { return align_up((size_t)n_units * sizeof(NsUnit), 1024); }

// Bytes of the tile records of every unit in every stage, for whichever tile
// mode a wave picks (the larger count of the two).
size_t ns_rec_bytes(const signmuon_shape* shapes, int n_mats, int n_workers) {
  size_t n = 0;
  for (int i = 0; i < n_mats; ++i)
    for (int stg = 0; stg < 3; ++stg)
      n += (size_t)n_workers * std::max(ns_tiles(shapes[i].rows, shapes[i].cols, stg, 0),
                                         ns_tiles(shapes[i].rows, shapes[i].cols, stg, 1));
  return align_up(n * sizeof(NsTileRec), 1024);
}

}  // namespace

signmuon_status signmuon::cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SIGNMUON_OK;
  g_last_cuda_error = e;
  return SIGNMUON_ERR_CUDA;
}

extern "C" {

const char* signmuon_status_string(int status) {
  switch (status) {
    case SIGNMUON_OK: return "SIGNMUON_OK";
    case SIGNMUON_ERR_INVALID_ARG: return "SIGNMUON_ERR_INVALID_ARG";
    case SIGNMUON_ERR_ALIGNMENT: return "SIGNMUON_ERR_ALIGNMENT";
    case SIGNMUON_ERR_UNSUPPORTED: return "SIGNMUON_ERR_UNSUPPORTED";
    case SIGNMUON_ERR_WORKSPACE: return "SIGNMUON_ERR_WORKSPACE";
    case SIGNMUON_ERR_CUDA: return "SIGNMUON_ERR_CUDA";
    default: return "SIGNMUON_UNKNOWN_STATUS";
  }
}

int signmuon_abi_version(void) { return kAbiVersion; }

const char* signmuon_last_error_string(void) {
  return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

int32_t signmuon_x_ld(int32_t cols) { return cols <= 0 ? -1 : x_ld_of(cols); }

int64_t signmuon_packed_words(signmuon_shape shape) {
  if (shape.rows <= 0 || shape.cols <= 0) return -1;
  return packed_words_of(shape);
}

signmuon_status signmuon_device_error(void* workspace, uint32_t* code, void* stream) {
  if (!workspace || !code) return SIGNMUON_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_status(e);
  *code = v;
  if (v != 0 && (e = cudaMemsetAsync(workspace, 0, 4, st)) != cudaSuccess) return cuda_status(e);
  return SIGNMUON_OK;
}

// ------------------------------------------------------------------ momentum
static int mom_blocks(signmuon_shape s) {
  const int64_t n = (int64_t)s.rows * s.cols;
  return (int)((n + kMomElemsPerBlock - 1) / kMomElemsPerBlock);
}

size_t signmuon_momentum_workspace_bytes(const signmuon_shape* shapes, int n_mats, int n_workers) {
  if (validate_shapes(shapes, n_mats) != SIGNMUON_OK || n_workers <= 0) return 0;
  int64_t blocks = 0;
  for (int i = 0; i < n_mats; ++i) blocks += (int64_t)mom_blocks(shapes[i]) * n_workers;
  const int64_t units = (int64_t)n_mats * n_workers;
  return kWsHeaderBytes + align_up((size_t)units * sizeof(MomUnit), 256) + align_up((size_t)blocks * 4, 256);
}

// Momentum update with one of three outputs (kernel modes): the bf16 copy of
// M (0), or the signs of X0 = M / norm packed (1) or int8 (2).  Arguments
// other than the outputs are validated here.
static signmuon_status momentum_run(const signmuon_shape* shapes, int n_mats, int n_workers,
                                    signmuon_dtype grad_dtype, const void* const* grad, float* const* mom,
                                    float beta, void* const* out, int out_mode, float* inv_norm, void* workspace,
                                    size_t ws_bytes, void* stream) {
  signmuon_status st = validate_shapes(shapes, n_mats);
  if (st) return st;
  if (n_workers <= 0 || n_workers > SIGNMUON_MAX_WORKERS) return SIGNMUON_ERR_INVALID_ARG;
  if (grad_dtype != SIGNMUON_F32 && grad_dtype != SIGNMUON_BF16) return SIGNMUON_ERR_INVALID_ARG;
  const int units = n_mats * n_workers;
  if ((st = validate_ptrs(grad, units))) return st;
  if ((st = validate_ptrs(reinterpret_cast<const void* const*>(mom), units))) return st;
  if ((st = validate_ptrs(reinterpret_cast<const void* const*>(out), units))) return st;
  if (!inv_norm) return SIGNMUON_ERR_INVALID_ARG;
  if (!aligned16(inv_norm)) return SIGNMUON_ERR_ALIGNMENT;
  if ((st = check_workspace(workspace, ws_bytes, signmuon_momentum_workspace_bytes(shapes, n_mats, n_workers))))
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  std::vector<MomUnit> mu(units);
  int blocks = 0;
  for (int i = 0; i < n_mats; ++i) {
    for (int m = 0; m < n_workers; ++m) {
      MomUnit& u = mu[i * n_workers + m];
      u.grad = grad[i * n_workers + m];
      u.mom = mom[i * n_workers + m];
      u.x = static_cast<__nv_bfloat16*>(out[i * n_workers + m]);
      u.rows = shapes[i].rows;
      u.cols = shapes[i].cols;
      u.n = (int64_t)u.rows * u.cols;
      u.ld_x = x_ld_of(u.cols);
      u.block_begin = blocks;
      u.block_count = mom_blocks(shapes[i]);
      u.pad_ = 0;
      blocks += u.block_count;
    }
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  MomUnit* d_units = reinterpret_cast<MomUnit*>(ws + kWsHeaderBytes);
  float* partials = reinterpret_cast<float*>(ws + kWsHeaderBytes + align_up((size_t)units * sizeof(MomUnit), 256));
  cudaError_t e = upload_bytes(d_units, mu.data(), mu.size() * sizeof(MomUnit), s);
  if (e == cudaSuccess)
    e = launch_momentum(d_units, units, blocks, grad_dtype == SIGNMUON_BF16, beta, partials, out_mode, s);
  if (e == cudaSuccess) e = launch_momentum_finalize(d_units, units, partials, inv_norm, out_mode, s);
  return cuda_status(e);
}

signmuon_status signmuon_momentum_norm(const signmuon_shape* shapes, int n_mats, int n_workers,
                                       signmuon_dtype grad_dtype, const void* const* grad, float* const* mom,
                                       float beta, void* const* x_bf16, float* inv_norm, void* workspace,
                                       size_t ws_bytes, void* stream) {
  return momentum_run(shapes, n_mats, n_workers, grad_dtype, grad, mom, beta, x_bf16, 0, inv_norm, workspace,
                      ws_bytes, stream);
}

signmuon_status signmuon_momentum_sign(const signmuon_shape* shapes, int n_mats, int n_workers,
                                       signmuon_dtype grad_dtype, const void* const* grad, float* const* mom,
                                       float beta, int int8_out, void* const* signs, float* inv_norm,
                                       void* workspace, size_t ws_bytes, void* stream) {
  signmuon_status st = validate_shapes(shapes, n_mats);
  if (st) return st;
  // Packed words are written 32 consecutive elements at a time: whole words per row.
  if (!int8_out)
    for (int i = 0; i < n_mats; ++i)
      if (shapes[i].cols % 32) return SIGNMUON_ERR_UNSUPPORTED;
  return momentum_run(shapes, n_mats, n_workers, grad_dtype, grad, mom, beta, signs, int8_out ? 2 : 1, inv_norm,
                      workspace, ws_bytes, stream);
}

// ------------------------------------------------------------ spectral scaling
// Relative cost per byte of a segment in the segment pass: a row's teams of
// T warps leave 8 - (8 / T) T warps of the block idle (two for three-warp
// teams), and multi-warp teams read their rows twice from shared memory
// (3 % slower per byte than one warp per row on nanoGPT-small's shapes).
static double spec_cost_per_byte(int cols) {
  const int t = spec_team_warps(cols);
  return 8.0 / (spec_teams(cols) * t) * (t > 1 ? 1.03 : 1.0);
}
// Spectral workspace: header | units | seg_unit | blk_seg | v | partials.
struct SpecLayout {
  size_t units, seg_unit, blk_seg, vecs, parts, total;  // byte offsets (total = size)
  int segs;
};
// Partials of z per unit: one per row block, or per (segment, row subset).
static int spec_parts(signmuon_shape sh, int* segs) {
  if (spec_segmented(sh.cols)) {
    *segs = (sh.rows + kSpecSegRows - 1) / kSpecSegRows;
    return *segs * spec_zsplit(sh.cols);
  }
  *segs = 0;
  return (sh.rows + kSpecRows - 1) / kSpecRows;
}
static SpecLayout spec_layout(const signmuon_shape* shapes, int n_mats, int n_workers) {
  size_t vf = 0, pf = 0;
  int segs = 0;
  for (int i = 0; i < n_mats; ++i) {
    const size_t cols4 = align_up((size_t)shapes[i].cols, 4);
    int ns = 0;
    const size_t n_parts = (size_t)spec_parts(shapes[i], &ns);
    vf += cols4 * n_workers;
    pf += n_parts * cols4 * n_workers;
    segs += ns * n_workers;
  }
  const size_t units = (size_t)n_mats * n_workers;
  SpecLayout L;
  L.segs = segs;
  L.units = kWsHeaderBytes;
  L.seg_unit = L.units + align_up(units * sizeof(SpecUnit), 256);
  L.blk_seg = L.seg_unit + align_up((size_t)segs * 4, 256);
  L.vecs = L.blk_seg + align_up((size_t)(kSpecMaxGrid + 1) * 4, 256);
  L.parts = L.vecs + align_up(vf * 4, 256);
  L.total = L.parts + align_up(pf * 4, 256);
  return L;
}

size_t signmuon_spectral_workspace_bytes(const signmuon_shape* shapes, int n_mats, int n_workers) {
  if (validate_shapes(shapes, n_mats) != SIGNMUON_OK || n_workers <= 0) return 0;
  return spec_layout(shapes, n_mats, n_workers).total;
}

signmuon_status signmuon_spectral_norm(const signmuon_shape* shapes, int n_mats, int n_workers,
                                       const void* const* x_bf16, int iters, float* inv_norm, void* workspace,
                                       size_t ws_bytes, void* stream) {
  signmuon_status st = validate_shapes(shapes, n_mats);
  if (st) return st;
  if (n_workers <= 0 || n_workers > SIGNMUON_MAX_WORKERS) return SIGNMUON_ERR_INVALID_ARG;
  if (iters < 1 || iters > 1000) return SIGNMUON_ERR_INVALID_ARG;
  const int units = n_mats * n_workers;
  if ((st = validate_ptrs(x_bf16, units))) return st;
  if (!inv_norm) return SIGNMUON_ERR_INVALID_ARG;
  if (!aligned16(inv_norm)) return SIGNMUON_ERR_ALIGNMENT;
  const SpecLayout lay = spec_layout(shapes, n_mats, n_workers);
  if ((st = check_workspace(workspace, ws_bytes, lay.total))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // One host blob for the unit table and the segment tables (one upload).
  std::vector<uint8_t> blob(lay.vecs - lay.units, 0);
  SpecUnit* hu = reinterpret_cast<SpecUnit*>(blob.data());
  int32_t* seg_unit = reinterpret_cast<int32_t*>(blob.data() + (lay.seg_unit - lay.units));
  int32_t* blk_seg = reinterpret_cast<int32_t*>(blob.data() + (lay.blk_seg - lay.units));
  std::vector<double> seg_cost;  // estimated cost of each segment (bytes x cost per byte)
  seg_cost.reserve(lay.segs);
  int64_t voff = 0, poff = 0;
  int blocks = 0, segs = 0;
  for (int i = 0; i < n_mats; ++i) {
    const int64_t cols4 = (int64_t)align_up((size_t)shapes[i].cols, 4);
    int n_seg = 0;
    const int n_parts = spec_parts(shapes[i], &n_seg);
    for (int m = 0; m < n_workers; ++m) {
      const int ui = i * n_workers + m;
      SpecUnit& u = hu[ui];
      memset(&u, 0, sizeof(u));
      u.x = static_cast<const __nv_bfloat16*>(x_bf16[ui]);
      u.rows = shapes[i].rows;
      u.cols = shapes[i].cols;
      u.ld_x = x_ld_of(u.cols);
      u.n_parts = n_parts;
      u.v_off = voff;
      u.part_off = poff;
      // Each pass numbers only its own units' work (the others own an empty range).
      u.block_begin = blocks;
      u.seg_begin = segs;
      voff += cols4;
      poff += (int64_t)n_parts * cols4;
      if (n_seg > 0) {
        for (int k = 0; k < n_seg; ++k) {
          seg_unit[segs + k] = ui;
          seg_cost.push_back((double)std::min(kSpecSegRows, u.rows - k * kSpecSegRows) * u.cols * 2.0 *
                             spec_cost_per_byte(u.cols));
        }
        segs += n_seg;
      } else {
        blocks += n_parts;
      }
    }
  }
  // Segment-pass blocks (two per SM) take contiguous ranges of segments
  // holding about equal shares of the estimated cost.
  const int seg_grid = std::min(std::min(segs, 2 * sm_count()), kSpecMaxGrid);
  double total = 0.0;
  for (double c : seg_cost) total += c;
  int sgi = 0;
  double before = 0.0;
  blk_seg[0] = 0;
  for (int b = 1; b < seg_grid; ++b) {
    const double target = total * b / seg_grid;
    while (sgi < segs && before + seg_cost[sgi] / 2 < target) before += seg_cost[sgi++];
    blk_seg[b] = sgi;
  }
  if (seg_grid > 0) blk_seg[seg_grid] = segs;
  // SIGNMUON_SPECTRAL_INJECT_WAIT_TIMEOUT_US=<n> (1 <= n <= 2000000): fault
  // injection for testing the bounded waits.  The segment pass loads no rows
  // and every block gives up waiting for them after n microseconds, recording
  // a wait-timeout code in the workspace; the estimates are then meaningless.
  // Unset (the default): full 2 s limit, normal operation.
  uint64_t wait_limit_ns = kWaitTimeoutNs;
  int withhold = 0;
  if (const char* inj = getenv("SIGNMUON_SPECTRAL_INJECT_WAIT_TIMEOUT_US")) {
    const long us = strtol(inj, nullptr, 10);
    if (us >= 1 && us <= 2000000) {
      wait_limit_ns = (uint64_t)us * 1000ull;
      withhold = 1;
    }
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = upload_bytes(ws + lay.units, blob.data(), blob.size(), s);
  if (e == cudaSuccess)
    e = launch_spectral(reinterpret_cast<const SpecUnit*>(ws + lay.units), units, blocks,
                        reinterpret_cast<const int32_t*>(ws + lay.seg_unit),
                        reinterpret_cast<const int32_t*>(ws + lay.blk_seg), seg_grid,
                        reinterpret_cast<float*>(ws + lay.vecs), reinterpret_cast<float*>(ws + lay.parts), iters,
                        inv_norm, reinterpret_cast<uint32_t*>(ws), wait_limit_ns, withhold, s);
  return cuda_status(e);
}

// ------------------------------------------------------------ Newton-Schulz
size_t signmuon_newton_schulz_workspace_bytes(const signmuon_shape* shapes, int n_mats, int n_workers,
                                              int minimal) {
  if (validate_shapes(shapes, n_mats) != SIGNMUON_OK || n_workers <= 0) return 0;
  const int units = n_mats * n_workers;
  size_t arena = 0;
  for (int i = 0; i < n_mats; ++i) {
    const size_t b = ns_unit_bytes(shapes[i]).total;
    arena = minimal ? std::max(arena, b) : arena + b * n_workers;
  }
  return kWsHeaderBytes + ns_desc_bytes(units) + ns_rec_bytes(shapes, n_mats, n_workers) + arena;
}

}  // extern "C"

namespace {

// A Newton-Schulz plan: the wave schedule of one set of units whose unit
// table (tensor maps, buffer addresses, tile numbering) already sits in the
// workspace.  It lives in caller-owned host memory (plan_bytes() bytes).
struct NsPlanHeader {
  uint64_t magic;
  uint8_t* workspace;
  const float* scales;  // inv_norm
  int64_t max_elems;
  int32_t n_units, n_waves, out_mode, w_dtype;
};
struct NsPlanWave {
  int32_t u0, nu;
  int32_t total[3], pair[3];
  int64_t rec0[3];   // first tile record of each stage (index into the record table)
  int32_t long_k[3];  // CTA-pair stage whose every tile has K >= kLongK
  int32_t wide[3];    //   and which runs 256x512 tiles
};
constexpr uint64_t kNsPlanMagic = 0x314e4c50534e4d53ull;  // "SMNSPLN1"
constexpr size_t kNsPlanHeaderBytes = (sizeof(NsPlanHeader) + 63) / 64 * 64;

size_t ns_plan_bytes(int units) { return kNsPlanHeaderBytes + (size_t)units * sizeof(NsPlanWave); }
inline NsPlanWave* plan_waves(void* plan) { return reinterpret_cast<NsPlanWave*>(static_cast<uint8_t*>(plan) + kNsPlanHeaderBytes); }

signmuon_status ns_validate_buffers(const signmuon_shape* shapes, int n_mats, int n_workers,
                                    void* const* x_bf16, const float* inv_norm, signmuon_ns_out out_mode,
                                    void* const* out, signmuon_dtype w_dtype, void* const* w) {
  signmuon_status st = validate_shapes(shapes, n_mats);
  if (st) return st;
  if (n_workers <= 0 || n_workers > SIGNMUON_MAX_WORKERS) return SIGNMUON_ERR_INVALID_ARG;
  if (out_mode != SIGNMUON_OUT_PACK1 && out_mode != SIGNMUON_OUT_INT8 && out_mode != SIGNMUON_OUT_UPDATE_W &&
      out_mode != SIGNMUON_OUT_U_F32)
    return SIGNMUON_ERR_INVALID_ARG;
  const int units = n_mats * n_workers;
  if ((st = validate_ptrs(x_bf16, units))) return st;
  if (!inv_norm) return SIGNMUON_ERR_INVALID_ARG;
  // Read one float per unit: 4-byte alignment suffices (a caller may pass a
  // slice of a larger per-unit array).
  if (reinterpret_cast<uintptr_t>(inv_norm) & 3u) return SIGNMUON_ERR_ALIGNMENT;
  if (out_mode == SIGNMUON_OUT_UPDATE_W) {
    if (n_workers != 1) return SIGNMUON_ERR_INVALID_ARG;
    if (w_dtype != SIGNMUON_F32 && w_dtype != SIGNMUON_BF16) return SIGNMUON_ERR_INVALID_ARG;
    if ((st = validate_ptrs(w, n_mats))) return st;
  } else {
    if ((st = validate_ptrs(out, units))) return st;
  }
  return SIGNMUON_OK;
}

// Encodes the unit table, uploads it into the workspace (stream-ordered on s)
// and fills the plan.  Arguments are validated by the caller.
signmuon_status ns_make_plan(const signmuon_shape* shapes, int n_mats, int n_workers, void* const* x_bf16,
                             const float* inv_norm, signmuon_ns_out out_mode, void* const* out,
                             signmuon_dtype w_dtype, void* const* w, void* workspace, size_t ws_bytes,
                             void* plan, cudaStream_t s) {
  const int units = n_mats * n_workers;
  const size_t need_min = signmuon_newton_schulz_workspace_bytes(shapes, n_mats, n_workers, 1);
  signmuon_status st = check_workspace(workspace, ws_bytes, need_min);
  if (st) return st;
  if (!encode_fn()) return SIGNMUON_ERR_UNSUPPORTED;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  NsUnit* d_units = reinterpret_cast<NsUnit*>(ws + kWsHeaderBytes);
  NsTileRec* d_recs = reinterpret_cast<NsTileRec*>(ws + kWsHeaderBytes + ns_desc_bytes(units));
  const size_t tables = kWsHeaderBytes + ns_desc_bytes(units) + ns_rec_bytes(shapes, n_mats, n_workers);
  uint8_t* arena = ws + tables;
  const size_t arena_bytes = ws_bytes - tables;

  // Plan waves: consecutive units whose buffers fit the arena together.  The
  // fewest waves are those of a greedy fill; the units are then re-split into
  // that many waves of about equal bytes (so that the last is no small
  // remainder), unless a wave of that split would not fit.
  std::vector<size_t> ubytes(units);
  size_t total_bytes = 0;
  for (int i = 0; i < n_mats; ++i)
    for (int m = 0; m < n_workers; ++m) total_bytes += (ubytes[i * n_workers + m] = ns_unit_bytes(shapes[i]).total);
  std::vector<int> starts_new(units, 0);
  int n_greedy = 0;
  {
    size_t fill = arena_bytes;  // forces a new wave at unit 0
    for (int ui = 0; ui < units; ++ui) {
      if (fill + ubytes[ui] > arena_bytes) { starts_new[ui] = 1; ++n_greedy; fill = 0; }
      fill += ubytes[ui];
    }
  }
  {
    std::vector<int> even(units, 0);
    size_t before = 0, fill = 0;
    int wave = -1;
    bool fits = true;
    for (int ui = 0; ui < units && fits; ++ui) {
      // Wave of the unit's midpoint on the even split.
      const int w = (int)std::min<size_t>((size_t)n_greedy - 1,
                                          (before + ubytes[ui] / 2) * (size_t)n_greedy / std::max<size_t>(total_bytes, 1));
      if (w != wave) { even[ui] = 1; wave = w; fill = 0; }
      fill += ubytes[ui];
      fits = fill <= arena_bytes;
      before += ubytes[ui];
    }
    if (fits) starts_new = even;
  }
  std::vector<NsUnit> hu(units);
  std::vector<int> wave_begin;
  size_t used = 0;
  int64_t max_elems = 0;
  for (int i = 0; i < n_mats; ++i) {
    const UnitBytes ub = ns_unit_bytes(shapes[i]);
    const int rows = shapes[i].rows, cols = shapes[i].cols;
    const int32_t sdim = std::min(rows, cols);
    max_elems = std::max(max_elems, (int64_t)rows * cols);
    for (int m = 0; m < n_workers; ++m) {
      const int ui = i * n_workers + m;
      if (starts_new[ui]) {
        wave_begin.push_back(ui);
        used = 0;
      }
      NsUnit& u = hu[ui];
      memset(&u, 0, sizeof(NsUnit));
      u.rows = rows;
      u.cols = cols;
      u.ld_x = x_ld_of(cols);
      u.ld_s = x_ld_of(sdim);
      u.x = static_cast<__nv_bfloat16*>(x_bf16[ui]);
      u.a = arena + used;
      u.b = reinterpret_cast<__nv_bfloat16*>(arena + used + ub.a);
      u.xalt = reinterpret_cast<__nv_bfloat16*>(arena + used + 2 * ub.a);
      used += ub.total;
      u.out = out_mode == SIGNMUON_OUT_UPDATE_W ? w[i] : out[ui];
      u.scale = inv_norm + ui;
      if (!encode_bf16_2d(&u.map_x, u.x, cols, rows, u.ld_x) ||
          !encode_bf16_2d(&u.map_xalt, u.xalt, cols, rows, u.ld_x) ||
          !encode_bf16_2d(&u.map_a, u.a, sdim, sdim, u.ld_s, false, true) ||
          !encode_bf16_2d(&u.map_b, u.b, sdim, sdim, u.ld_s) ||
          !encode_bf16_2d(&u.st_x, u.x, cols, rows, u.ld_x, true) ||
          !encode_bf16_2d(&u.st_xalt, u.xalt, cols, rows, u.ld_x, true) ||
          !encode_bf16_2d(&u.st_a, u.a, sdim, sdim, u.ld_s, true, true) ||
          !encode_bf16_2d(&u.st_b, u.b, sdim, sdim, u.ld_s, true))
        return SIGNMUON_ERR_UNSUPPORTED;
    }
  }
  wave_begin.push_back(units);
  // SIGNMUON_NS_TILE_MODE=single|pair forces one tile mode (used by the tests
  // to compare the two modes on the same inputs); unset = automatic.
  int forced_mode = -1;
  if (const char* m = getenv("SIGNMUON_NS_TILE_MODE")) {
    if (!strcmp(m, "single")) forced_mode = 0;
    else if (!strcmp(m, "pair")) forced_mode = 1;
  }
  // SIGNMUON_NS_WIDE=0 keeps the long-reduction launches on 256x256 tiles
  // (the tests compare both layouts on the same inputs).
  bool wide_ok = true;
  if (const char* m = getenv("SIGNMUON_NS_WIDE")) wide_ok = strcmp(m, "0") != 0;
  // Per wave and stage, pick the tile mode with the least padded work (the
  // CTA-pair mode is preferred unless it pads more than 15 % extra), then
  // number the tiles; prefixes restart at each wave (a launch covers one
  // wave).
  NsPlanHeader* hdr = static_cast<NsPlanHeader*>(plan);
  NsPlanWave* waves = plan_waves(plan);
  const int n_waves = (int)wave_begin.size() - 1;
  std::vector<NsTileRec> recs;
  for (int wv = 0; wv < n_waves; ++wv) {
    NsPlanWave& W = waves[wv];
    W.u0 = wave_begin[wv];
    W.nu = wave_begin[wv + 1] - W.u0;
    for (int stg = 0; stg < 3; ++stg) {
      double single_area = 0, pair_area = 0;
      for (int ui = W.u0; ui < W.u0 + W.nu; ++ui) {
        single_area += (double)ns_tiles(hu[ui].rows, hu[ui].cols, stg, 0) * 128.0 * kBN;
        pair_area += (double)ns_tiles(hu[ui].rows, hu[ui].cols, stg, 1) * 256.0 * kBN;
      }
      int pair = pair_area <= 1.15 * single_area ? 1 : 0;
      if (forced_mode >= 0) pair = forced_mode;
      W.pair[stg] = pair;
      // The reduction length of a unit's tiles: the long side for the Gram
      // product, the short side for the other two.
      int min_k = INT32_MAX;
      for (int ui = W.u0; ui < W.u0 + W.nu; ++ui) {
        const int kr = stg == kStageGram ? std::max(hu[ui].rows, hu[ui].cols) : std::min(hu[ui].rows, hu[ui].cols);
        min_k = std::min(min_k, kr);
      }
      W.long_k[stg] = pair && min_k >= kLongK ? 1 : 0;
      W.wide[stg] = W.long_k[stg] && wide_ok ? 1 : 0;
      const int wide = W.wide[stg];
      int pre = 0;
      W.rec0[stg] = (int64_t)recs.size();
      for (int ui = W.u0; ui < W.u0 + W.nu; ++ui) {
        hu[ui].tile_begin[stg] = pre;
        hu[ui].tile_count[stg] = ns_tiles(hu[ui].rows, hu[ui].cols, stg, pair, wide);
        pre += hu[ui].tile_count[stg];
        if (stg == kStageApply && hu[ui].rows <= hu[ui].cols) {
          // Apply of a wide unit (X' = B'X): X is the B operand, so the tiles
          // go column by column -- consecutive tiles (running at the same
          // time on neighbouring CTA pairs) share one column block of X,
          // which is read from DRAM once instead of once per row of tiles.
          // (A tall unit's X is the A operand: row by row, the tile_of
          // numbering, already keeps its row blocks together.)
          const int bm = ns_tile_m(pair), bn = wide ? 2 * kBN : kBN;
          const int tiles_m = (hu[ui].rows + bm - 1) / bm, tiles_n = (hu[ui].cols + bn - 1) / bn;
          for (int tn = 0; tn < tiles_n; ++tn)
            for (int tm = 0; tm < tiles_m; ++tm)
              recs.push_back(NsTileRec{ui - W.u0, tm * tiles_n + tn, hu[ui].rows, hu[ui].cols});
        } else {
          for (int li = 0; li < hu[ui].tile_count[stg]; ++li)
            recs.push_back(NsTileRec{ui - W.u0, li, hu[ui].rows, hu[ui].cols});
        }
      }
      W.total[stg] = pre;
      // Launch order.  With few tiles per CTA (pair) the round-robin
      // assignment leaves CTAs unevenly loaded when tiles differ in length:
      // then the longest reductions go first (the Gram's K is the long side,
      // the other stages' the short one) so that the launch ends on short
      // tiles.  With many tiles per CTA the unit order stays, which keeps
      // the tiles running at the same time on few units (L2 reuse of their
      // operands).  The sort is stable: a unit's tiles stay together.
      const int workers = pair ? sm_count() / 2 : sm_count();
      if (W.total[stg] < 8 * workers) {
        auto k_of = [stg](const NsTileRec& r) {
          return stg == kStageGram ? std::max(r.rows, r.cols) : std::min(r.rows, r.cols);
        };
        std::stable_sort(recs.begin() + W.rec0[stg], recs.end(),
                         [&](const NsTileRec& x, const NsTileRec& y) { return k_of(x) > k_of(y); });
      }
    }
  }
  if (recs.size() * sizeof(NsTileRec) > ns_rec_bytes(shapes, n_mats, n_workers)) return SIGNMUON_ERR_WORKSPACE;
  cudaError_t e = upload_bytes(d_units, hu.data(), hu.size() * sizeof(NsUnit), s);
  if (e == cudaSuccess) e = upload_bytes(d_recs, recs.data(), recs.size() * sizeof(NsTileRec), s);
  if (e != cudaSuccess) return cuda_status(e);
  hdr->magic = kNsPlanMagic;
  hdr->workspace = ws;
  hdr->scales = inv_norm;
  hdr->max_elems = max_elems;
  hdr->n_units = units;
  hdr->n_waves = n_waves;
  hdr->out_mode = (int32_t)out_mode;
  hdr->w_dtype = (int32_t)w_dtype;
  return SIGNMUON_OK;
}

signmuon_status ns_run_plan(const void* plan, int k, float a, float b, float c, float eta, cudaStream_t s) {
  const NsPlanHeader* hdr = static_cast<const NsPlanHeader*>(plan);
  const NsPlanWave* waves = reinterpret_cast<const NsPlanWave*>(static_cast<const uint8_t*>(plan) + kNsPlanHeaderBytes);
  NsUnit* d_units = reinterpret_cast<NsUnit*>(hdr->workspace + kWsHeaderBytes);
  const NsTileRec* d_recs =
      reinterpret_cast<const NsTileRec*>(hdr->workspace + kWsHeaderBytes + ns_desc_bytes(hdr->n_units));
  // SIGNMUON_NS_INJECT_WAIT_TIMEOUT_US=<n> (1 <= n <= 2000000): fault
  // injection for testing the bounded waits.  Every Newton-Schulz GEMM
  // launch withholds its operand loads and gives up waiting after n
  // microseconds, recording a wait-timeout code in the workspace; its
  // outputs are left unwritten.  Unset (the default): full 2 s limit, normal
  // operation.
  uint64_t wait_limit_ns = kWaitTimeoutNs;
  int withhold = 0;
  if (const char* inj = getenv("SIGNMUON_NS_INJECT_WAIT_TIMEOUT_US")) {
    const long us = strtol(inj, nullptr, 10);
    if (us >= 1 && us <= 2000000) {
      wait_limit_ns = (uint64_t)us * 1000ull;
      withhold = 1;
    }
  }
  cudaError_t e = cudaSuccess;
  for (int wv = 0; wv < hdr->n_waves; ++wv) {
    const NsPlanWave& W = waves[wv];
    if (k == 0) {
      e = launch_ns_identity(d_units + W.u0, W.nu, hdr->max_elems, hdr->out_mode, hdr->w_dtype, eta, s);
      if (e != cudaSuccess) return cuda_status(e);
      continue;
    }
    for (int it = 0; it < k; ++it) {
      NsLaunch L;
      memset(&L, 0, sizeof(L));
      L.units = d_units + W.u0;
      L.scales = hdr->scales + W.u0;
      L.n_units = W.nu;
      L.parity = it & 1;
      L.first = it == 0;
      L.a = a;
      L.b = b;
      L.c = c;
      // The shifted form when the shift is moderate (Q's diagonal keeps fp16's
      // absolute precision near that of A): |b / 2c| <= 4.
      L.shift = c != 0.f && std::fabs((double)b) <= 8.0 * std::fabs((double)c);
      L.beta = L.shift ? (float)((double)b / (2.0 * (double)c)) : 0.f;
      L.a2 = L.shift ? (float)((double)a - (double)b * (double)b / (4.0 * (double)c)) : a;
      L.eta = eta;
      L.w_dtype = hdr->w_dtype;
      L.err = reinterpret_cast<uint32_t*>(hdr->workspace);
      L.wait_limit_ns = wait_limit_ns;
      L.withhold_loads = withhold;
      for (int stg = 0; stg < 3; ++stg) {
        L.stage = stg;
        L.recs = d_recs + W.rec0[stg];
        L.total_tiles = W.total[stg];
        L.pair = W.pair[stg];
        L.long_k = W.long_k[stg];
        L.wide = W.wide[stg];
        L.out_kind = (stg == kStageApply && it == k - 1) ? hdr->out_mode : (int)kOutIterate;
        e = launch_ns_gemm(L, s);
        if (e != cudaSuccess) return cuda_status(e);
      }
    }
  }
  return SIGNMUON_OK;
}

}  // namespace

extern "C" {

size_t signmuon_newton_schulz_plan_bytes(int n_mats, int n_workers) {
  if (n_mats <= 0 || n_workers <= 0 || n_workers > SIGNMUON_MAX_WORKERS) return 0;
  return ns_plan_bytes(n_mats * n_workers);
}

signmuon_status signmuon_newton_schulz_plan(const signmuon_shape* shapes, int n_mats, int n_workers,
                                            void* const* x_bf16, const float* inv_norm,
                                            signmuon_ns_out out_mode, void* const* out, signmuon_dtype w_dtype,
                                            void* const* w, void* workspace, size_t ws_bytes, void* plan,
                                            size_t plan_bytes, void* stream) {
  signmuon_status st = ns_validate_buffers(shapes, n_mats, n_workers, x_bf16, inv_norm, out_mode, out, w_dtype, w);
  if (st) return st;
  if (!plan) return SIGNMUON_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(plan) & 7u) return SIGNMUON_ERR_ALIGNMENT;
  if (plan_bytes < ns_plan_bytes(n_mats * n_workers)) return SIGNMUON_ERR_INVALID_ARG;
  static_cast<NsPlanHeader*>(plan)->magic = 0;  // invalid until fully built
  return ns_make_plan(shapes, n_mats, n_workers, x_bf16, inv_norm, out_mode, out, w_dtype, w, workspace,
                      ws_bytes, plan, static_cast<cudaStream_t>(stream));
}

signmuon_status signmuon_newton_schulz_run(const void* plan, int k, float a, float b, float c, float eta,
                                           void* stream) {
  if (!plan) return SIGNMUON_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(plan) & 7u) return SIGNMUON_ERR_ALIGNMENT;
  if (static_cast<const NsPlanHeader*>(plan)->magic != kNsPlanMagic) return SIGNMUON_ERR_INVALID_ARG;
  if (k < 0 || k > 64) return SIGNMUON_ERR_INVALID_ARG;
  return ns_run_plan(plan, k, a, b, c, eta, static_cast<cudaStream_t>(stream));
}

signmuon_status signmuon_newton_schulz_batched(const signmuon_shape* shapes, int n_mats, int n_workers,
                                               void* const* x_bf16, const float* inv_norm, int k, float a,
                                               float b, float c, signmuon_ns_out out_mode, void* const* out,
                                               signmuon_dtype w_dtype, void* const* w, float eta,
                                               void* workspace, size_t ws_bytes, void* stream) {
  signmuon_status st = ns_validate_buffers(shapes, n_mats, n_workers, x_bf16, inv_norm, out_mode, out, w_dtype, w);
  if (st) return st;
  if (k < 0 || k > 64) return SIGNMUON_ERR_INVALID_ARG;
  std::vector<uint64_t> plan((ns_plan_bytes(n_mats * n_workers) + 7) / 8);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = ns_make_plan(shapes, n_mats, n_workers, x_bf16, inv_norm, out_mode, out, w_dtype, w, workspace,
                         ws_bytes, plan.data(), s)))
    return st;
  return ns_run_plan(plan.data(), k, a, b, c, eta, s);
}

// ------------------------------------------------------------------ sign pack
signmuon_status signmuon_sign_pack(signmuon_shape shape, signmuon_dtype u_dtype, const void* u, int64_t ld_u,
                                   int int8_out, void* out, void* stream) {
  if (shape.rows <= 0 || shape.cols <= 0 || !u || !out || ld_u < shape.cols) return SIGNMUON_ERR_INVALID_ARG;
  if (u_dtype != SIGNMUON_F32 && u_dtype != SIGNMUON_BF16) return SIGNMUON_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(out)) return SIGNMUON_ERR_ALIGNMENT;
  return cuda_status(launch_sign_pack(shape, u_dtype == SIGNMUON_BF16, u, ld_u, int8_out != 0, out,
                                      packed_words_of(shape), static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ vote
size_t signmuon_vote_workspace_bytes(const signmuon_shape* shapes, int n_mats, int n_workers) {
  if (validate_shapes(shapes, n_mats) != SIGNMUON_OK || n_workers <= 0) return 0;
  return kWsHeaderBytes + align_up((size_t)n_mats * sizeof(VoteMat), 256) +
         align_up((size_t)n_mats * n_workers * sizeof(void*), 256);
}

signmuon_status signmuon_vote_update(const signmuon_shape* shapes, int n_mats, int n_workers, int int8_in,
                                     const void* const* signs, signmuon_dtype w_dtype, void* const* w, float eta,
                                     void* const* vote_bf16, int64_t* nnz, float* vote_inv_norm, void* workspace,
                                     size_t ws_bytes, void* stream) {
  signmuon_status st = validate_shapes(shapes, n_mats);
  if (st) return st;
  if (n_workers <= 0 || n_workers > SIGNMUON_MAX_WORKERS) return SIGNMUON_ERR_INVALID_ARG;
  if (w_dtype != SIGNMUON_F32 && w_dtype != SIGNMUON_BF16) return SIGNMUON_ERR_INVALID_ARG;
  const int units = n_mats * n_workers;
  if ((st = validate_ptrs(signs, units))) return st;
  const bool vote_out = vote_bf16 != nullptr;
  if (vote_out) {
    if ((st = validate_ptrs(vote_bf16, n_mats))) return st;
    if (!nnz || !vote_inv_norm) return SIGNMUON_ERR_INVALID_ARG;
    if (!aligned16(nnz) || !aligned16(vote_inv_norm)) return SIGNMUON_ERR_ALIGNMENT;
  } else {
    if ((st = validate_ptrs(w, n_mats))) return st;
  }
  if ((st = check_workspace(workspace, ws_bytes, signmuon_vote_workspace_bytes(shapes, n_mats, n_workers))))
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  std::vector<VoteMat> hm(n_mats);
  int blocks = 0;
  for (int i = 0; i < n_mats; ++i) {
    VoteMat& v = hm[i];
    memset(&v, 0, sizeof(v));
    v.w = vote_out ? nullptr : w[i];
    v.vote = vote_out ? vote_bf16[i] : nullptr;
    v.rows = shapes[i].rows;
    v.cols = shapes[i].cols;
    v.n = (int64_t)v.rows * v.cols;
    v.wpr = (int32_t)wpr_of(v.cols);
    v.n_words = (int64_t)v.rows * v.wpr;
    v.ld_x = x_ld_of(v.cols);
    v.block_begin = blocks;
    v.block_count = vote_blocks_for(int8_in != 0, w_dtype == SIGNMUON_BF16, vote_out, v.cols, v.n, v.n_words);
    v.sign_ptr_offset = i * n_workers;
    blocks += v.block_count;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  VoteMat* d_mats = reinterpret_cast<VoteMat*>(ws + kWsHeaderBytes);
  const void** d_table =
      reinterpret_cast<const void**>(ws + kWsHeaderBytes + align_up((size_t)n_mats * sizeof(VoteMat), 256));
  // The matrix table and the sign-pointer table are adjacent in the
  // workspace: one upload writes both.
  const size_t table_off = align_up((size_t)n_mats * sizeof(VoteMat), 256);
  std::vector<uint8_t> staged(table_off + (size_t)units * sizeof(void*), 0);
  memcpy(staged.data(), hm.data(), hm.size() * sizeof(VoteMat));
  memcpy(staged.data() + table_off, signs, (size_t)units * sizeof(void*));
  cudaError_t e = upload_bytes(d_mats, staged.data(), staged.size(), s);
  if (e == cudaSuccess && vote_out) e = cudaMemsetAsync(nnz, 0, (size_t)n_mats * sizeof(int64_t), s);
  if (e == cudaSuccess)
    e = launch_vote(d_mats, n_mats, blocks, d_table, n_workers, int8_in != 0, w_dtype == SIGNMUON_BF16, eta,
                    vote_out, reinterpret_cast<unsigned long long*>(nnz), s);
  if (e == cudaSuccess && vote_out) e = launch_vote_inv(nnz, vote_inv_norm, n_mats, s);
  return cuda_status(e);
}

}  // extern "C"
