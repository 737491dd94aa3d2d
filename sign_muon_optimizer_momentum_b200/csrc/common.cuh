// Internal definitions shared by the kernels and the C-ABI layer of
// libsignmuon.so.  Not part of the public interface (see include/signmuon.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "signmuon.h"

namespace signmuon {

// ---------------------------------------------------------------------------
// Device error codes recorded in the first word of a workspace.
// ---------------------------------------------------------------------------
enum DeviceError : uint32_t {
  kErrNone = 0,
  kErrWaitTimeoutProducer = 0x101,  // TMA producer gave up waiting for a free stage
  kErrWaitTimeoutMma = 0x102,       // MMA issuer gave up waiting for data / accumulator
  kErrWaitTimeoutEpilogue = 0x103,  // epilogue gave up waiting for an accumulator
  kErrWaitTimeoutDrain = 0x104,     // exit-time wait for in-flight copies ran out
  kErrWaitTimeoutSpectral = 0x105,  // spectral segment pass gave up waiting for its rows
};

// Workspace header: error word + padding.  Every workspace starts with it.
constexpr size_t kWsHeaderBytes = 256;

// Bounded waits: give up after this many nanoseconds of device time.
constexpr uint64_t kWaitTimeoutNs = 2000ull * 1000ull * 1000ull;  // 2 s

// ---------------------------------------------------------------------------
// Newton-Schulz GEMM tiling (tcgen05, one CTA per tile, cta_group::1).
// ---------------------------------------------------------------------------
constexpr int kBN = 256;          // MMA N (TMEM fp32 columns per accumulator)
constexpr int kBK = 64;           // K per stage: 64 bf16 = 128 B = one swizzle row
constexpr int kUmmaK = 16;        // K per tcgen05.mma for kind::f16
constexpr int kBoxRows = 64;      // every TMA box is 64 x 64 bf16 (8 KB)
constexpr int kBoxBytes = 64 * 64 * 2;
constexpr int kAccCols = kBN;                             // fp32 columns per accumulator
constexpr int kTmemCols = 2 * kAccCols;                   // double-buffered: 512
constexpr int kEpilogueThreads = 256;                     // warps 2-9
constexpr int kGemmThreads = 64 + kEpilogueThreads;       // warp 0 TMA, warp 1 MMA
constexpr int kBarrierBytes = 256;
// Epilogue output staging: two 32x32 bf16 blocks (2 KB each, 64-byte swizzle)
// per epilogue warp, written to global memory by TMA stores.
constexpr int kStageBlockBytes = 32 * 32 * 2;
constexpr int kStagingBytes = (kEpilogueThreads / 32) * 2 * kStageBlockBytes;  // 32 KB

// Row stride, in elements, of a bf16 Newton-Schulz buffer: cols rounded up
// to 8 (16 bytes, the TMA stride granule).  The public signmuon_x_ld.
inline int32_t x_ld_of(int32_t cols) { return (cols + 7) / 8 * 8; }

// Maps a CUDA error to a status; a failure is also recorded as the calling
// thread's last error (read back by signmuon_last_error_string).
signmuon_status cuda_status(cudaError_t e);

// Output rows per tile: 128 for one CTA, 256 for a CTA pair.
inline int ns_tile_m(int pair) { return pair ? 256 : 128; }

enum NsStage : int { kStageGram = 0, kStageSquare = 1, kStageApply = 2 };

// Final-iteration output kinds (mirror signmuon_ns_out) and the bf16 iterate.
enum NsOut : int {
  kOutPack1 = SIGNMUON_OUT_PACK1,
  kOutInt8 = SIGNMUON_OUT_INT8,
  kOutUpdateW = SIGNMUON_OUT_UPDATE_W,
  kOutUF32 = SIGNMUON_OUT_U_F32,
  kOutIterate = 100,
};

// One (matrix, worker) unit of a Newton-Schulz launch.  Tensor maps first so
// they stay 64-byte aligned (the struct is 64-byte aligned and a multiple
// of 64 bytes long).
struct alignas(64) NsUnit {
  // Load maps: 64x64 boxes, 128-byte swizzle (GEMM operands).
  CUtensorMap map_x;     // caller's bf16 X buffer  [rows, ld_x]
  CUtensorMap map_xalt;  // workspace bf16 X buffer [rows, ld_x]
  CUtensorMap map_a;     // workspace Gram A (fp16)  [s, ld_s]
  CUtensorMap map_b;     // workspace B' = aI + bA + cA^2 (bf16) [s, ld_s]
  // Store maps: 32x32 boxes, 64-byte swizzle (epilogue output blocks).
  CUtensorMap st_x;
  CUtensorMap st_xalt;
  CUtensorMap st_a;
  CUtensorMap st_b;
  __nv_bfloat16* x;
  __nv_bfloat16* xalt;
  void* a;               // fp16
  __nv_bfloat16* b;
  void* out;             // final output (packed / int8 / fp32 U / W)
  const float* scale;    // &inv_norm[u]
  int32_t rows, cols, ld_x, ld_s;
  int32_t tile_begin[3];  // host bookkeeping: first tile of the unit in unit order, per stage
  int32_t tile_count[3];  //   and its tile count (the kernels read the tile records)
  int32_t pad_[2];
};
static_assert(sizeof(NsUnit) % 64 == 0, "NsUnit must keep 64-byte alignment");

// One tile of a Newton-Schulz launch, laid out on the host in launch order,
// so that a CTA learns its next tile's unit and geometry from one 16-byte
// load issued a tile ahead (no search over the unit table).
struct NsTileRec {
  int32_t unit;   // index into the launch's unit table
  int32_t li;     // tile index within the unit (the tile_of numbering)
  int32_t rows, cols;
};
static_assert(sizeof(NsTileRec) == 16, "tile records are read as one 16-byte load");

struct NsLaunch {
  const NsUnit* units;
  const NsTileRec* recs;  // total_tiles records of this launch's stage
  const float* scales;    // scales[u] = 1 / norm of unit u (first iteration)
  int n_units;
  int stage;        // NsStage
  int parity;       // 0: X_in = x, X_out = xalt; 1: the reverse
  int first;        // scale X by *unit.scale (iteration 0)
  int out_kind;     // NsOut: kOutIterate for non-final APPLY
  int w_dtype;      // for kOutUpdateW
  int total_tiles;
  int pair;         // 1: CTA-pair (cta_group::2) 256x256 tiles; 0: one CTA, 128x256
  float a, b, c, eta;
  // shift (c != 0 and |b / 2c| <= 4): the Gram stage stores Q = A + beta I
  // (beta = b / 2c) in place of A, and the square stage forms
  // B' = c Q Q + a2 I (a2 = a - b^2 / 4c), which equals a I + b A + c A^2;
  // otherwise A itself, and the square's epilogue reads A back for b A.
  int shift;
  float beta, a2;
  uint32_t* err;
  uint64_t wait_limit_ns;  // every bounded wait gives up after this long
  // Fault injection for testing the bounded waits: the producer arms no
  // barrier and issues no copy, so the consumers' waits run out.
  int withhold_loads;
  int long_k;       // CTA pairs, every tile K >= kLongK: direct stores, no staging
  int wide;         // with long_k: 256x512 tiles, two N = 256 halves of one accumulator
};

// Reduction length from which a CTA-pair launch uses the long layout.
constexpr int kLongK = 2048;

// Momentum units.
struct MomUnit {
  const void* grad;
  float* mom;
  __nv_bfloat16* x;   // the bf16 copy of M; in the sign modes the packed / int8 sign buffer
  int64_t n;          // rows * cols
  int32_t rows, cols, ld_x;
  int32_t block_begin;  // first block of this unit in the flattened grid
  int32_t block_count;
  int32_t pad_;
};

// Vote matrices.
struct VoteMat {
  void* w;
  void* vote;          // bf16 vote-out buffer or null
  int64_t n;           // rows * cols
  int64_t n_words;     // rows * ceil(cols/32) (packed) -- logical words
  int32_t rows, cols, wpr, ld_x;
  int32_t block_begin, block_count;
  int32_t sign_ptr_offset;  // index into the sign pointer table (i * n_workers)
  int32_t pad_;
};

static_assert(sizeof(NsUnit) == 1152, "descriptor size is part of the launch-count bookkeeping");
static_assert(sizeof(MomUnit) == 56, "descriptor size is part of the launch-count bookkeeping");
static_assert(sizeof(VoteMat) == 64, "descriptor size is part of the launch-count bookkeeping");

// Spectral-scaling units (power iteration on X^T X).
// A unit is passed over either by the segment pass (spec_segmented(cols):
// rows streamed through shared memory, spec_zsplit(cols) partials of z per
// kSpecSegRows rows) or by the row-block pass (any other width: one partial
// of z per kSpecRows rows).
struct SpecUnit {
  const __nv_bfloat16* x;
  int64_t v_off;        // float offset of this unit's vector v (cols entries)
  int64_t part_off;     // float offset of its partial sums [n_parts][cols]
  int32_t rows, cols, ld_x;
  int32_t n_parts;      // its segment partials, or its row blocks
  int32_t block_begin;  // first row block of this unit in the row-block pass's grid (none if segmented)
  int32_t seg_begin;    // first segment of this unit in the segment pass's sequence (none if not)
};
static_assert(sizeof(SpecUnit) == 48, "descriptor size");
constexpr int kSpecRows = 32;
constexpr int kSpecSmemCols = 8192;  // v is staged in shared memory up to this many columns (32 KB)
constexpr int kSpecSegRows = 128;       // rows per segment
constexpr int kSpecSlotBytes = 24576;   // shared-memory ring slot: the rows of one group
constexpr int kSpecSlots = 4;
constexpr int kSpecSegMaxCols = 4096;   // at most six warps per row (below)
constexpr int kSpecScratchBytes = 16384;  // shared memory for the end-of-segment sums of z
constexpr int kSpecMaxGrid = 512;       // segment-pass blocks at most (two per SM)
// The segment pass takes each row with a team of T warps, lane l of the
// team's warp j holding the 8-column chunks 96 j + l + 32 i (i < 3) of v and
// z in registers; the block's 8 / T teams take the rows of a group round
// robin.
constexpr int kSpecLaneChunks = 3;
constexpr int kSpecTeamRows = 12;  // rows per group at most when T > 1 (15 fit 776 columns; 12 is 4 teams' multiple)
constexpr int kSpecWarpChunks = 32 * kSpecLaneChunks;  // 96 chunks: 768 columns per warp
__host__ __device__ inline bool spec_segmented(int cols) { return (cols & 7) == 0 && cols <= kSpecSegMaxCols; }
__host__ __device__ inline int spec_team_warps(int cols) { return (cols / 8 + kSpecWarpChunks - 1) / kSpecWarpChunks; }
__host__ __device__ inline int spec_teams(int cols) { return 8 / spec_team_warps(cols); }
// Rows per group (ring slot) of a segmented unit: the most rows that fit a
// slot, at most 32, rounded down to a multiple of the teams.
__host__ __device__ inline int spec_group_rows(int cols) {
  int g = kSpecSlotBytes / (2 * cols);
  if (g > 32) g = 32;
  const int t = spec_teams(cols);
  return g / t * t;
}
// Partials of z per segment of a segmented unit: each team sums z over its
// own rows, and the block adds the teams' sums in shared memory down to two
// (eight or four teams) or one.
__host__ __device__ inline int spec_zsplit(int cols) { return spec_teams(cols) >= 4 ? 2 : 1; }

// ---------------------------------------------------------------------------
// Launch helpers implemented in the .cu files (all enqueue on `stream`).
// ---------------------------------------------------------------------------
cudaError_t upload_bytes(void* dst_device, const void* src_host, size_t bytes, cudaStream_t stream);
cudaError_t launch_momentum(const MomUnit* units, int n_units, int total_blocks, int grad_bf16,
                            float beta, float* partials, int out_mode, cudaStream_t stream);
cudaError_t launch_momentum_finalize(const MomUnit* units, int n_units, const float* partials,
                                     float* inv_norm, int out_mode, cudaStream_t stream);
cudaError_t launch_sign_pack(signmuon_shape shape, int u_bf16, const void* u, int64_t ld_u,
                             int int8_out, void* out, int64_t out_words, cudaStream_t stream);
cudaError_t launch_vote(const VoteMat* mats, int n_mats, int total_blocks, const void* const* sign_table,
                        int n_workers, int int8_in, int w_bf16, float eta, int vote_out,
                        unsigned long long* nnz, cudaStream_t stream);
cudaError_t launch_vote_inv(const int64_t* nnz, float* inv, int n_mats, cudaStream_t stream);
int vote_blocks_for(int int8_in, int w_bf16, int vote_out, int cols, int64_t n, int64_t n_words);
cudaError_t launch_ns_gemm(const NsLaunch& p, cudaStream_t stream);
// seg_unit[s]: the unit of segment s (segments in unit order); the segment
// pass's block b takes segments [blk_seg[b], blk_seg[b + 1]) of seg_grid blocks.
cudaError_t launch_spectral(const SpecUnit* units, int n_units, int total_row_blocks, const int32_t* seg_unit,
                            const int32_t* blk_seg, int seg_grid, float* vecs, float* parts, int iters,
                            float* inv_norm, uint32_t* err, uint64_t wait_limit_ns, int withhold,
                            cudaStream_t stream);
cudaError_t launch_ns_identity(const NsUnit* units, int n_units, int64_t max_elems, int out_kind,
                               int w_dtype, float eta, cudaStream_t stream);

// Block-count helpers shared by host planning and kernels.
constexpr int kMomThreads = 256;
constexpr int kMomElemsPerThread = 16;
constexpr int kMomElemsPerBlock = kMomThreads * kMomElemsPerThread;  // 4096
constexpr int kVoteThreads = 256;

}  // namespace signmuon
