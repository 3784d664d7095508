// cq_noalloc.cu -- cq_gemm_noalloc: cq_gemm for callers that cannot allocate
// device memory.  Its scratch (the stream-K tile counters and partial tiles)
// lives in one fixed, file-scope device array instead of a caller workspace.
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
// runtime once per device (with that device current) and cached.
static int fixed_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return CQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess || !p) return CQ_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return CQ_OK;
}

}  // namespace cq

using namespace cq;

extern "C" int cq_gemm_noalloc(const uint16_t* x, int64_t M, const uint8_t* packed,
                               const float* scales, const uint16_t* ab, int64_t N, int64_t K,
                               int B, int G, int grid_mode, int epilogue, int out_dtype, void* y,
                               void* stream) {
  int st = validate_matrix(packed, scales, ab, N, K, B, G, grid_mode);
  if (st != CQ_OK) return st;
  if (M < 0) return CQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return gemm_impl(x, M, packed, scales, ab, N, K, B, G, grid_mode,
                                         epilogue, out_dtype, y, nullptr, 0,
                                         static_cast<cudaStream_t>(stream), kDefaultTimeoutNs, 0);
  const int sms = num_sms();
  if (sms <= 0) return CQ_ERR_CUDA;
  if (K % kSlice != 0) return CQ_ERR_UNSUPPORTED;
  if (epilogue == CQ_EPI_SWIGLU && N % kRows != 0) return CQ_ERR_UNSUPPORTED;
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
