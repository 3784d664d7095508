// cq_noalloc.cu -- cq_gemm_noalloc: cq_gemm for callers that cannot allocate
// device memory.  Its scratch (the stream-K tile counters and partial tiles)
// lives in one fixed, file-scope device array instead of a caller workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "cq.h"
#include "cq_host.h"

namespace cq {

// Largest scratch the fixed array provides: enough for every M <= 16
// (decode-sized) GEMM on a 148-SM part; larger problems are rejected.
constexpr size_t kFixedScratchBytes = static_cast<size_t>(4) << 20;

// Every GPU that loads libcq holds this array until the process exits.
static __device__ __align__(256) uint8_t g_fixed_scratch[kFixedScratchBytes];

// Device address of g_fixed_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is asked from the
// runtime (with the device current) and cached per device together with the
// context it belongs to: after a cudaDeviceReset the device has a new
// context, and the address is looked up again.
// cuCtxGetCurrent, fetched through the runtime (libcq does not link the
// driver library directly, so that it loads on a machine without one).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
static CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

static int fixed_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[128] = {};
  static CUcontext ctx_of[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return CQ_ERR_CUDA;
  // null on a thread that has not bound a context yet: then the lookup below
  // binds the device's primary context
  const CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (!get_ctx) return CQ_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ctx && addr[dev] && ctx_of[dev] == ctx) {
    *out = addr[dev];
    return CQ_OK;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess || !p) return CQ_ERR_CUDA;
  if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return CQ_ERR_CUDA;
  addr[dev] = p;
  ctx_of[dev] = ctx;
  *out = p;
  return CQ_OK;
}

}  // namespace cq

using namespace cq;

extern "C" int cq_gemm_noalloc(const uint16_t* x, int64_t M, const uint8_t* packed,
                               const float* scales, const uint16_t* ab, int64_t N, int64_t K,
                               int B, int G, int grid_mode, int epilogue, int out_dtype, void* y,
                               void* stream) {
  // every argument check first: a rejected call must not have touched the
  // shared array or queued anything on the stream
  int st = validate_gemm(x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype, y);
  if (st != CQ_OK) return st;
  if (M == 0 || N == 0) return CQ_OK;
  const int sms = num_sms();
  if (sms <= 0) return CQ_ERR_CUDA;
  size_t counter_bytes = 0, total = 0;
  gemm_scratch(M, N, K, B, G, epilogue, sms, &counter_bytes, &total);
  if (total > kFixedScratchBytes) return CQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = fixed_scratch_address(&scratch);
  if (st != CQ_OK) return st;
  // The array keeps the previous call's contents: the tile counters must
  // start at zero, the partial tiles are always written before being read.
  if (counter_bytes &&
      cudaMemsetAsync(scratch, 0, counter_bytes, static_cast<cudaStream_t>(stream)) !=
          cudaSuccess)
    return CQ_ERR_CUDA;
  return gemm_impl(x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype, y,
                   scratch, kFixedScratchBytes, static_cast<cudaStream_t>(stream),
                   kDefaultTimeoutNs, 0);
}
