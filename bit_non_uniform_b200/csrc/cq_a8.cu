// cq_a8.cu -- host side of the Dynamic-A8 GEMM: per-row activation
// quantization into the workspace, then the A8 engine.  Part of libcq's
// single translation unit.
#include <cuda_runtime.h>

#include "cq.h"
#include "cq_a8.cuh"
#include "cq_host.h"

namespace cq {

// Token-tile width of the A8 engine (three NT-column TMEM buffers: at most 128).
static int pick_nt_a8(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

struct A8Plan {
  int NT, n_tt, n_rt, spt, tiles, P;
  size_t off_amax, off_cnt, off_part, total;
};

static size_t round256(size_t v) { return (v + 255) / 256 * 256; }

static A8Plan plan_a8(int64_t M, int64_t N, int64_t K, int epilogue, int sms) {
  A8Plan g;
  g.n_rt = epilogue == CQ_EPI_SWIGLU ? static_cast<int>(N / kRows)
                                     : static_cast<int>((N + kRows - 1) / kRows);
  g.NT = pick_nt_a8(M);
  g.n_tt = static_cast<int>((M + g.NT - 1) / g.NT);
  g.spt = static_cast<int>(K / kSlice);
  g.tiles = g.n_rt * g.n_tt;
  const int64_t W = static_cast<int64_t>(g.tiles) * g.spt;
  g.P = static_cast<int>(W < sms ? W : sms);
  g.off_amax = round256(static_cast<size_t>(M) * K);                  // xq first
  g.off_cnt = g.off_amax + round256(static_cast<size_t>(M) * sizeof(float));
  g.off_part = g.off_cnt + round256(static_cast<size_t>(g.tiles) * sizeof(int));
  g.total = g.off_part + static_cast<size_t>(2) * g.P * g.NT * kRows * sizeof(float);
  return g;
}

// int8 [rows][cols] viewed as boxes of 128 columns x box_rows rows, 128-byte
// swizzle (the K-major operand layout of the MMA).  Rows past `rows` read 0.
static int encode_i8_rows_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                                int box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return CQ_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CQ_OK : CQ_ERR_CUDA;
}

static int quant_rows(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* absmax,
                      cudaStream_t s) {
  if (M == 0) return CQ_OK;
  quant_rows_kernel<<<static_cast<unsigned>(M), kQuantThreads, 0, s>>>(
      x, static_cast<int>(M), static_cast<int>(K), xq, absmax);
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

template <int NT, int TE>
static int launch_a8(const A8Params& p, const CUtensorMap& xmap, const CUtensorMap& wmap,
                     cudaStream_t s) {
  using C = A8Cfg<NT, TE>;
  static std::atomic<uint64_t> smem_set{0};
  if (!ensure_smem_limit(engine_a8_kernel<NT, TE>, C::SMEM, smem_set)) return CQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(p.e.P);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, engine_a8_kernel<NT, TE>, p, xmap, wmap) != cudaSuccess)
    return CQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

template <int NT>
static int launch_a8_te(const A8Params& p, const CUtensorMap& xmap, const CUtensorMap& wmap,
                        int B, cudaStream_t s) {
  if (B == 3) return launch_a8<NT, 64>(p, xmap, wmap, s);
  return launch_a8<NT, 16>(p, xmap, wmap, s);
}

static int gemm_a8_impl(const uint16_t* x, int64_t M, const uint8_t* packed, const float* scales,
                        const uint16_t* ab, int64_t N, int64_t K, int B, int G, int grid_mode,
                        int epilogue, int out_dtype, void* y, void* workspace, size_t ws_bytes,
                        cudaStream_t stream) {
  int st = validate_matrix(packed, scales, ab, N, K, B, G, grid_mode);
  if (st != CQ_OK) return st;
  if (M < 0) return CQ_ERR_INVALID_ARG;
  if (epilogue != CQ_EPI_NONE && epilogue != CQ_EPI_SWIGLU) return CQ_ERR_INVALID_ARG;
  if (out_dtype != CQ_DTYPE_F32 && out_dtype != CQ_DTYPE_BF16) return CQ_ERR_INVALID_ARG;
  if (epilogue == CQ_EPI_SWIGLU && N % kRows != 0) return CQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return CQ_OK;
  if (!x || !y || !workspace) return CQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(workspace, 256)) return CQ_ERR_UNSUPPORTED;
  if (M > (int64_t)1 << 24) return CQ_ERR_UNSUPPORTED;
  if (((M + 15) / 16) * ((N + kRows - 1) / kRows) >= ((int64_t)1 << 31)) return CQ_ERR_UNSUPPORTED;
  const int sms = num_sms();
  if (sms <= 0) return CQ_ERR_CUDA;
  const A8Plan g = plan_a8(M, N, K, epilogue, sms);
  if (ws_bytes < g.total) return CQ_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws);
  float* absmax = reinterpret_cast<float*>(ws + g.off_amax);
  st = quant_rows(x, M, K, xq, absmax, stream);
  if (st != CQ_OK) return st;

  CUtensorMap xmap, wmap;
  st = encode_i8_rows_sw128(&xmap, xq, M, K, g.NT);
  if (st != CQ_OK) return st;
  st = encode_packed_rows(&wmap, packed, N, K * B / 8, B);
  if (st != CQ_OK) return st;

  A8Params pa = {};
  EngineParams& p = pa.e;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = G;
  p.mode = grid_mode;
  p.epilogue = epilogue;
  p.out_bf16 = out_dtype == CQ_DTYPE_BF16;
  p.n_rt = g.n_rt;
  p.spt = g.spt;
  p.num_tiles = g.tiles;
  p.P = g.P;
  p.mat.packed = packed;
  p.mat.scales = scales;
  p.mat.ab = reinterpret_cast<const uint32_t*>(ab);
  p.mat.B = B;
  p.M = static_cast<int>(M);
  p.n_tt = g.n_tt;
  p.y = y;
  p.ldy = epilogue == CQ_EPI_SWIGLU ? N / 2 : N;
  p.y_rows = M;
  p.partial_slots = 2 * g.P;
  p.counter_len = g.tiles;
  p.counter = reinterpret_cast<int*>(ws + g.off_cnt);
  p.partial = reinterpret_cast<float*>(ws + g.off_part);
  p.timeout_ns = 2000000000ull;
  pa.absmax = absmax;
  // the stream-K counters start at zero (each finished tile resets its own)
  if (cudaMemsetAsync(p.counter, 0, static_cast<size_t>(g.tiles) * sizeof(int), stream) !=
      cudaSuccess)
    return CQ_ERR_CUDA;

  switch (g.NT) {
    case 16: return launch_a8_te<16>(pa, xmap, wmap, B, stream);
    case 32: return launch_a8_te<32>(pa, xmap, wmap, B, stream);
    case 64: return launch_a8_te<64>(pa, xmap, wmap, B, stream);
    default: return launch_a8_te<128>(pa, xmap, wmap, B, stream);
  }
}

}  // namespace cq

using namespace cq;

extern "C" CQ_API int cq_quant_rows(const uint16_t* x, int64_t M, int64_t K, int8_t* xq,
                                    float* absmax, void* stream) {
  if (M < 0 || K <= 0 || K > (int64_t)1 << 30 || M > (int64_t)1 << 31) return CQ_ERR_INVALID_ARG;
  if (M == 0) return CQ_OK;
  if (!x || !xq || !absmax) return CQ_ERR_INVALID_ARG;
  return quant_rows(x, M, K, xq, absmax, static_cast<cudaStream_t>(stream));
}

extern "C" CQ_API size_t cq_gemm_a8_workspace_size(int64_t M, int64_t N, int64_t K, int B,
                                                   int G, int epilogue) {
  if (M <= 0 || N <= 0 || K <= 0 || K % kSlice != 0 || G <= 0 || G % kSlice != 0 ||
      K % G != 0 || B < 2 || B > 4 || M > (int64_t)1 << 24)
    return 0;
  int sms = num_sms();
  if (sms <= 0) sms = 148;
  return plan_a8(M, N, K, epilogue, sms).total;
}

extern "C" CQ_API int cq_gemm_a8(const uint16_t* x, int64_t M, const uint8_t* packed,
                                 const float* scales, const uint16_t* ab, int64_t N, int64_t K,
                                 int B, int G, int grid_mode, int epilogue, int out_dtype,
                                 void* y, void* workspace, size_t ws_bytes, void* stream) {
  return gemm_a8_impl(x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype, y,
                      workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}
