// signmuon_momentum_norm_noalloc: the momentum + Frobenius-norm call with its
// scratch in a fixed device array owned by the library instead of a
// caller-provided workspace.
//
// Who needs this: callers that cannot allocate device memory around the
// step -- for example an optimizer embedded in a runtime whose allocator has
// already reserved the whole device (a further cudaMalloc would fail or
// fragment it), or a loop that must not call cudaMalloc/cudaFree because
// those calls synchronise the device.  Such callers still pass their own
// inputs and outputs; only the scratch moves into the library.
//
// The scratch is one array, kNoAllocScratchBytes (1 MiB) of device memory on
// every GPU that loads the library, held until the process exits.  Its
// layout: the unit table (at most kNoAllocMaxUnits records) followed by the
// per-block partial sums of squares (at most kNoAllocMaxBlocks blocks of
// 4096 elements, i.e. about 1e9 elements over all units).  Every call
// rewrites the parts it reads, so nothing needs to start at zero.  All calls
// share the array: two calls whose kernels overlap on the GPU (different
// streams without ordering between them) race on it and must not be issued.
//
// The device address of the array is looked up once per device and cached
// for the life of the process.  It belongs to the device's primary context:
// after cudaDeviceReset (which destroys that context and the module's
// copy of the array) the cached address is stale, and this entry point must
// not be called again in that process.
#include <mutex>
#include <vector>

#include "common.cuh"

using namespace signmuon;

namespace {

constexpr size_t kNoAllocScratchBytes = 1u << 20;
constexpr size_t kNoAllocTableBytes = 64u << 10;
constexpr int kNoAllocMaxUnits = (int)(kNoAllocTableBytes / sizeof(MomUnit));  // 1170
constexpr int kNoAllocMaxBlocks = (int)((kNoAllocScratchBytes - kNoAllocTableBytes) / sizeof(float));

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  Host code
// cannot use the symbol itself (it names a host-side shadow), so the address
// is looked up once per device with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" signmuon_status signmuon_momentum_norm_noalloc(const signmuon_shape* shapes, int n_mats, int n_workers,
                                                          signmuon_dtype grad_dtype, const void* const* grad,
                                                          float* const* mom, float beta, void* const* x_bf16,
                                                          float* inv_norm, void* stream) {
  if (!shapes || n_mats <= 0 || n_workers <= 0 || n_workers > SIGNMUON_MAX_WORKERS) return SIGNMUON_ERR_INVALID_ARG;
  if (grad_dtype != SIGNMUON_F32 && grad_dtype != SIGNMUON_BF16) return SIGNMUON_ERR_INVALID_ARG;
  if (!grad || !mom || !x_bf16 || !inv_norm) return SIGNMUON_ERR_INVALID_ARG;
  const long long units = (long long)n_mats * n_workers;
  if (units > kNoAllocMaxUnits) return SIGNMUON_ERR_WORKSPACE;
  long long blocks = 0;
  for (int i = 0; i < n_mats; ++i) {
    if (shapes[i].rows <= 0 || shapes[i].cols <= 0) return SIGNMUON_ERR_INVALID_ARG;
    const long long n = (long long)shapes[i].rows * shapes[i].cols;
    blocks += (n + kMomElemsPerBlock - 1) / kMomElemsPerBlock * n_workers;
  }
  if (blocks > kNoAllocMaxBlocks) return SIGNMUON_ERR_WORKSPACE;
  for (long long u = 0; u < units; ++u) {
    if (!grad[u] || !mom[u] || !x_bf16[u]) return SIGNMUON_ERR_INVALID_ARG;
    if (!aligned16(grad[u]) || !aligned16(mom[u]) || !aligned16(x_bf16[u])) return SIGNMUON_ERR_ALIGNMENT;
  }
  if (!aligned16(inv_norm)) return SIGNMUON_ERR_ALIGNMENT;

  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_status(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  std::vector<MomUnit> mu((size_t)units);
  int b = 0;
  for (int i = 0; i < n_mats; ++i) {
    const int cnt = (int)(((long long)shapes[i].rows * shapes[i].cols + kMomElemsPerBlock - 1) / kMomElemsPerBlock);
    for (int m = 0; m < n_workers; ++m) {
      MomUnit& u = mu[(size_t)i * n_workers + m];
      u.grad = grad[i * n_workers + m];
      u.mom = mom[i * n_workers + m];
      u.x = static_cast<__nv_bfloat16*>(x_bf16[i * n_workers + m]);
      u.rows = shapes[i].rows;
      u.cols = shapes[i].cols;
      u.n = (int64_t)u.rows * u.cols;
      u.ld_x = x_ld_of(u.cols);
      u.block_begin = b;
      u.block_count = cnt;
      u.pad_ = 0;
      b += cnt;
    }
  }
  MomUnit* d_units = static_cast<MomUnit*>(scratch);
  float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + kNoAllocTableBytes);
  e = upload_bytes(d_units, mu.data(), mu.size() * sizeof(MomUnit), s);
  if (e == cudaSuccess) e = launch_momentum(d_units, (int)units, b, grad_dtype == SIGNMUON_BF16, beta, partials, 0, s);
  if (e == cudaSuccess) e = launch_momentum_finalize(d_units, (int)units, partials, inv_norm, 0, s);
  return cuda_status(e);
}
