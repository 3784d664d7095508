// cq_api.cu -- libcq entry points that need no tensor core: version, status
// strings, the device error word, cq_pack and cq_decode.
#include <cuda_runtime.h>

#include "cq.h"
#include "cq_device.cuh"
#include "cq_host.h"

namespace cq {

// ---------------------------------------------------------------------------
// cq_pack: one thread per output byte.  Byte j of a row holds stream bits
// [8j, 8j+8); code k contributes its bits [kB, kB+B) shifted into place.
// ---------------------------------------------------------------------------
__global__ void pack_kernel(const uint8_t* __restrict__ codes, int64_t N, int64_t K, int B,
                            uint8_t* __restrict__ packed) {
  const int64_t row_bytes = K * B / 8;
  const int64_t total = N * row_bytes;
  const unsigned mask = (1u << B) - 1u;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = idx / row_bytes;
    const int64_t j = idx - n * row_bytes;
    const int64_t bit0 = 8 * j;
    const int64_t k_first = bit0 / B;
    const int64_t k_last = (bit0 + 7) / B;
    const uint8_t* row = codes + n * K;
    unsigned byte = 0;
    for (int64_t k = k_first; k <= k_last && k < K; ++k) {
      const int sh = static_cast<int>(k * B - bit0);   // may be negative
      const unsigned u = row[k] & mask;
      byte |= sh >= 0 ? (u << sh) : (u >> (-sh));
    }
    packed[idx] = static_cast<uint8_t>(byte & 0xFFu);
  }
}

// ---------------------------------------------------------------------------
// cq_decode: one thread per weight; levels in FP64, rounded once to FP32.
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void decode_kernel(const uint8_t* __restrict__ packed,
                              const float* __restrict__ scales,
                              const __half* __restrict__ ab, int64_t N, int64_t K, int B,
                              int G, int mode, void* __restrict__ out) {
  const int64_t total = N * K;
  const int64_t row_bytes = K * B / 8;
  const int64_t ng = K / G;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = idx / K;
    const int64_t k = idx - n * K;
    const int64_t bit = k * B;
    const uint8_t* row = packed + n * row_bytes;
    const unsigned lo = row[bit >> 3];
    const unsigned hi = ((bit >> 3) + 1 < row_bytes) ? row[(bit >> 3) + 1] : 0u;
    const unsigned u = (((hi << 8) | lo) >> (bit & 7)) & ((1u << B) - 1u);
    const int64_t g = n * ng + k / G;
    const double a = static_cast<double>(__half2float(ab[2 * g]));
    const double b = static_cast<double>(__half2float(ab[2 * g + 1]));
    const float L = static_cast<float>(level_f64(static_cast<int>(u), B, mode, scales[g], a, b));
    if (BF16)
      reinterpret_cast<uint16_t*>(out)[idx] = bf16_bits(L);
    else
      reinterpret_cast<float*>(out)[idx] = L;
  }
}

static int grid_for(int64_t total, int threads) {
  int64_t blocks = (total + threads - 1) / threads;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t cap = static_cast<int64_t>(sms) * 32;
  return static_cast<int>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace cq

using namespace cq;

extern "C" int cq_version(void) { return 100; }

extern "C" const char* cq_status_string(int status) {
  switch (status) {
    case CQ_OK: return "ok";
    case CQ_ERR_INVALID_ARG: return "invalid argument";
    case CQ_ERR_UNSUPPORTED: return "unsupported shape, width, group size or alignment";
    case CQ_ERR_CUDA: return "CUDA runtime error";
    case CQ_ERR_TIMEOUT: return "a bounded device wait ran out";
    case CQ_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

extern "C" int cq_get_device_error(void* stream, int* site) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return CQ_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return CQ_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess)
    return CQ_ERR_CUDA;
  if (site) *site = v;
  return v ? CQ_ERR_TIMEOUT : CQ_OK;
}

extern "C" int cq_pack(const uint8_t* codes, int64_t N, int64_t K, int B, uint8_t* packed,
                       void* stream) {
  if (!codes || !packed || N < 0 || K < 0) return CQ_ERR_INVALID_ARG;
  if (B < 1 || B > 8) return CQ_ERR_INVALID_ARG;
  if ((K * B) % 8 != 0) return CQ_ERR_UNSUPPORTED;
  const int64_t total = N * (K * B / 8);
  if (total == 0) return CQ_OK;
  pack_kernel<<<grid_for(total, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      codes, N, K, B, packed);
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

extern "C" int cq_decode(const uint8_t* packed, const float* scales, const uint16_t* ab,
                         int64_t N, int64_t K, int B, int G, int grid_mode, int out_dtype,
                         void* W_out, void* stream) {
  int st = validate_matrix(packed, scales, ab, N, K, B, G, grid_mode, 1, 8);
  if (st != CQ_OK) return st;
  if (!W_out) return CQ_ERR_INVALID_ARG;
  if (out_dtype != CQ_DTYPE_F32 && out_dtype != CQ_DTYPE_BF16) return CQ_ERR_INVALID_ARG;
  const int64_t total = N * K;
  if (total == 0) return CQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __half* abh = reinterpret_cast<const __half*>(ab);
  if (out_dtype == CQ_DTYPE_BF16)
    decode_kernel<true><<<grid_for(total, 256), 256, 0, s>>>(packed, scales, abh, N, K, B, G,
                                                             grid_mode, W_out);
  else
    decode_kernel<false><<<grid_for(total, 256), 256, 0, s>>>(packed, scales, abh, N, K, B, G,
                                                              grid_mode, W_out);
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}
