// cq_host.h -- host-side argument validation and TMA descriptor encoding
// shared by the libcq entry points.
#pragma once

#include <atomic>

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "cq.h"

namespace cq {

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Checks shared by every call that reads a packed CubicQuant matrix.
// Raise a kernel's dynamic shared-memory limit once per device: the
// attribute belongs to the device's context, so a process that drives
// several GPUs sets it on each (`done` holds one bit per device ordinal;
// ordinals >= 64 set it on every call).
template <typename Kernel>
inline bool ensure_smem_limit(Kernel* kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  if (bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

// Bit widths: cq_gemm and the format tools (pack, decode) take 1..8 (the
// midtread grid needs B >= 2: Kc = 2^(B-1) - 1 > 0); the grouped MoE GEMM and
// the Dynamic A8 path take {2, 3, 4}.
inline int validate_matrix(const uint8_t* packed, const float* scales, const uint16_t* ab,
                           int64_t N, int64_t K, int B, int G, int grid_mode, int b_min = 2,
                           int b_max = 4) {
  if (N < 0 || K < 0 || G <= 0) return CQ_ERR_INVALID_ARG;
  if (grid_mode != CQ_GRID_MIDRISE && grid_mode != CQ_GRID_MIDTREAD) return CQ_ERR_INVALID_ARG;
  if (B < b_min || B > b_max) return CQ_ERR_UNSUPPORTED;
  if (grid_mode == CQ_GRID_MIDTREAD && B < 2) return CQ_ERR_UNSUPPORTED;
  if (G % 128 != 0 || K % G != 0) return CQ_ERR_UNSUPPORTED;
  if (N * K == 0) return CQ_OK;
  if (!packed || !scales || !ab) return CQ_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(scales, 4) || !aligned(ab, 4)) return CQ_ERR_UNSUPPORTED;
  if (K > (int64_t)1 << 30 || N > (int64_t)1 << 30) return CQ_ERR_UNSUPPORTED;
  return CQ_OK;
}

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor map over a row-major bf16 matrix [rows][cols] loaded as boxes of
// 64 columns (128 bytes) x box_rows rows with the 128-byte swizzle.  Rows
// past `rows` read as zero.
inline int encode_bf16_rows_sw128(CUtensorMap* map, const void* base, int64_t rows,
                                  int64_t cols, int box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return CQ_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CQ_OK : CQ_ERR_CUDA;
}

// Tensor map over a packed CubicQuant matrix viewed as uint8 [rows][row_bytes],
// loaded as boxes of 16*B bytes (one 128-code slice) x 64 rows.  The swizzle
// (32-byte for B=2, 64-byte for B=4, 128-byte for B=8, none for the odd
// widths' 16*B-byte rows and for B=6) keeps the row-per-thread 16-byte
// shared-memory reads of the decoders conflict free (B=6: two-way).
inline int encode_packed_rows(CUtensorMap* map, const void* base, int64_t rows,
                              int64_t row_bytes, int B) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return CQ_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(16 * B), 64u};
  cuuint32_t estr[2] = {1u, 1u};
  CUtensorMapSwizzle sw = B == 2   ? CU_TENSOR_MAP_SWIZZLE_32B
                          : B == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : B == 8 ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CQ_OK : CQ_ERR_CUDA;
}

inline int num_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return sms;
}

}  // namespace cq
