// cq_gemm.cu -- host side of cq_gemm: argument checks, work partition,
// activation tensor map and the engine launch.
#include <cuda_runtime.h>

#include "cq.h"
#include "cq_engine.cuh"
#include "cq_gemv.cuh"
#include "cq_host.h"

namespace cq {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;   // 2 s per wait

static int pick_nt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

struct GemmPlan {
  int NT, n_tt, n_rt, spt, tiles, P;
  size_t ws_counter_bytes, ws_partial_bytes;
};

static GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int epilogue, int sms) {
  GemmPlan g;
  g.NT = pick_nt(M);
  g.n_tt = static_cast<int>((M + g.NT - 1) / g.NT);
  g.n_rt = epilogue == CQ_EPI_SWIGLU ? static_cast<int>(N / kRows)
                                     : static_cast<int>((N + kRows - 1) / kRows);
  g.spt = static_cast<int>(K / kSlice);
  g.tiles = g.n_rt * g.n_tt;
  const int64_t W = static_cast<int64_t>(g.tiles) * g.spt;
  g.P = static_cast<int>(W < sms ? W : sms);
  g.ws_counter_bytes = ((static_cast<size_t>(g.tiles) * sizeof(int) + 255) / 256) * 256;
  g.ws_partial_bytes = static_cast<size_t>(2) * g.P * g.NT * kRows * sizeof(float);
  return g;
}

// ---------------------------------------------------------------------------
// decode-sized path (M <= 2): gemv_kernel
// ---------------------------------------------------------------------------
struct GvPlan {
  bool use;
  int MT, ng, spc, gpair, n_rb, n_cols, rpc, P, x_bytes, smem, max_quads;
  size_t ws_counter_bytes, ws_partial_bytes;   // zero: the GEMV needs no workspace
};

static int gv_dynamic_smem(int B, int MT, int G, int spc, int x_bytes, int mq) {
  if (MT == 1) {
    if (B == 2) return GvCfg<2, 1>::smem_bytes(G, spc, x_bytes, mq);
    if (B == 3) return GvCfg<3, 1>::smem_bytes(G, spc, x_bytes, mq);
    return GvCfg<4, 1>::smem_bytes(G, spc, x_bytes, mq);
  }
  if (B == 2) return GvCfg<2, 2>::smem_bytes(G, spc, x_bytes, mq);
  if (B == 3) return GvCfg<3, 2>::smem_bytes(G, spc, x_bytes, mq);
  return GvCfg<4, 2>::smem_bytes(G, spc, x_bytes, mq);
}

static GvPlan plan_gemv(int64_t M, int64_t N, int64_t K, int B, int G, int epilogue, int sms) {
  GvPlan v = {};
  if (M < 1 || M > 2 || N < 1 || K < G || B < 2 || B > 4) return v;
  if (epilogue == CQ_EPI_SWIGLU && N % 16 != 0) return v;
  if (G / 8 * B > 256 || N >= (1 << 24) || K >= (1 << 24)) return v;   // a group row = one box row
  v.MT = M == 1 ? 1 : 2;
  v.ng = static_cast<int>(K / G);
  v.spc = G / 128;
  v.gpair = v.ng % 2 == 0 ? 2 : 1;
  v.n_rb = static_cast<int>(epilogue == CQ_EPI_SWIGLU ? N / 16 : (N + 15) / 16);
  const int64_t n_cols = static_cast<int64_t>(v.n_rb) * v.ng;
  if (n_cols >= (1 << 26)) return v;
  v.n_cols = static_cast<int>(n_cols);
  // every CTA owns whole row blocks
  v.rpc = (v.n_rb + sms - 1) / sms;
  v.P = (v.n_rb + v.rpc - 1) / v.rpc;
  if (v.rpc > kGvMaxRb) return v;
  for (int c = 0; c < v.P; ++c) {
    const int rb0 = c * v.rpc;
    const int rb1 = rb0 + v.rpc < v.n_rb ? rb0 + v.rpc : v.n_rb;
    const int nq = ((rb1 * v.ng - 1) >> 2) - ((rb0 * v.ng) >> 2) + 1;
    if (nq > v.max_quads) v.max_quads = nq;
  }
  if (v.max_quads > kGvMaxQuads) return v;
  v.x_bytes = static_cast<int>((M * K * 2 + 127) / 128 * 128);
  v.smem = gv_dynamic_smem(B, v.MT, G, v.spc, v.x_bytes, v.max_quads);
  if (v.smem > 227 * 1024) return v;
  v.use = true;
  return v;
}

template <int B, int MT>
static int launch_gemv(const GemvParams& p, const CUtensorMap& wmap, int smem, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(gemv_kernel<B, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess)
      return CQ_ERR_CUDA;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(p.P);
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, gemv_kernel<B, MT>, p, wmap) != cudaSuccess) return CQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

// Tensor map over the packed matrix for the GEMV, viewed as 4-D uint8
//   (byte of a group row [G*B/8], row [R], half [H], group [ng])
// with R x H = N rows (H = 2 separates the gate and up halves for SwiGLU).
// One box = gpair columns (consecutive groups of one row block) x 16 rows of
// whole group rows, landing in shared memory as [group][half][row][G*B/8]:
// the 16 row slots of a column are 8 * item + g for both epilogues.
static int encode_packed_gemv(CUtensorMap* map, const void* base, int64_t N, int64_t K, int B,
                              int G, int epilogue, int gpair) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return CQ_ERR_CUDA;
  const int64_t row_bytes = K * B / 8;
  const bool swiglu = epilogue == CQ_EPI_SWIGLU;
  const int64_t R = swiglu ? N / 2 : N;
  const int RG = G / 8 * B;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(RG), static_cast<cuuint64_t>(R),
                        swiglu ? 2u : 1u, static_cast<cuuint64_t>(K / G)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(row_bytes),
                           static_cast<cuuint64_t>(swiglu ? R * row_bytes : row_bytes),
                           static_cast<cuuint64_t>(RG)};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(RG), swiglu ? 8u : 16u, swiglu ? 2u : 1u,
                       static_cast<cuuint32_t>(gpair)};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CQ_OK : CQ_ERR_CUDA;
}

static int run_gemv(const GvPlan& v, const uint16_t* x, int64_t M, const uint8_t* packed,
                    const float* scales, const uint16_t* ab, int64_t N, int64_t K, int B, int G,
                    int grid_mode, int epilogue, int out_dtype, void* y, cudaStream_t stream,
                    uint64_t timeout_ns, uint64_t* trace) {
  CUtensorMap wmap;
  int st = encode_packed_gemv(&wmap, packed, N, K, B, G, epilogue, v.gpair);
  if (st != CQ_OK) return st;
  GemvParams p = {};
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = G;
  p.mode = grid_mode;
  p.epilogue = epilogue;
  p.out_bf16 = out_dtype == CQ_DTYPE_BF16;
  p.M = static_cast<int>(M);
  p.ng = v.ng;
  p.n_rb = v.n_rb;
  p.n_cols = v.n_cols;
  p.spc = v.spc;
  p.rpc = v.rpc;
  p.P = v.P;
  p.gpair = v.gpair;
  p.spc_magic = v.spc > 1 ? static_cast<uint32_t>(((1ull << 32) + v.spc - 1) / v.spc) : 0u;
  p.max_quads = v.max_quads;
  p.scales = scales;
  p.ab = reinterpret_cast<const uint32_t*>(ab);
  p.x = x;
  p.x_bytes = v.x_bytes;
  p.smem_bytes = v.smem;
  p.y = y;
  p.ldy = epilogue == CQ_EPI_SWIGLU ? N / 2 : N;
  p.timeout_ns = timeout_ns;
  p.trace = reinterpret_cast<unsigned long long*>(trace);
  if (v.MT == 1) {
    if (B == 2) return launch_gemv<2, 1>(p, wmap, v.smem, stream);
    if (B == 3) return launch_gemv<3, 1>(p, wmap, v.smem, stream);
    return launch_gemv<4, 1>(p, wmap, v.smem, stream);
  }
  if (B == 2) return launch_gemv<2, 2>(p, wmap, v.smem, stream);
  if (B == 3) return launch_gemv<3, 2>(p, wmap, v.smem, stream);
  return launch_gemv<4, 2>(p, wmap, v.smem, stream);
}

// Scratch bytes of whichever path gemm_impl takes for this problem.
static void gemm_scratch(int64_t M, int64_t N, int64_t K, int B, int G, int epilogue, int sms,
                         size_t* counter_bytes, size_t* total) {
  const GvPlan v = plan_gemv(M, N, K, B, G, epilogue, sms);
  if (v.use) {
    *counter_bytes = v.ws_counter_bytes;
    *total = v.ws_counter_bytes + v.ws_partial_bytes;
    return;
  }
  const GemmPlan g = plan_gemm(M, N, K, epilogue, sms);
  *counter_bytes = g.ws_counter_bytes;
  *total = g.ws_counter_bytes + g.ws_partial_bytes;
}

// ---------------------------------------------------------------------------
// tensor-core engine path
// ---------------------------------------------------------------------------
template <int NT>
static int launch_engine(const EngineParams& p, const CUtensorMap& map, const CUtensorMap& wmap,
                         cudaStream_t s) {
  using C = EngineCfg<NT>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(engine_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM) != cudaSuccess)
      return CQ_ERR_CUDA;
    attr_set = true;
  }
  engine_kernel<NT><<<p.P, kThreads, C::SMEM, s>>>(p, map, wmap);
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

int gemm_impl(const uint16_t* x, int64_t M, const uint8_t* packed, const float* scales,
              const uint16_t* ab, int64_t N, int64_t K, int B, int G, int grid_mode,
              int epilogue, int out_dtype, void* y, void* workspace, size_t ws_bytes,
              cudaStream_t stream, uint64_t timeout_ns, int debug_skip,
              uint64_t* trace = nullptr) {
  int st = validate_matrix(packed, scales, ab, N, K, B, G, grid_mode);
  if (st != CQ_OK) return st;
  if (M < 0) return CQ_ERR_INVALID_ARG;
  if (epilogue != CQ_EPI_NONE && epilogue != CQ_EPI_SWIGLU) return CQ_ERR_INVALID_ARG;
  if (out_dtype != CQ_DTYPE_F32 && out_dtype != CQ_DTYPE_BF16) return CQ_ERR_INVALID_ARG;
  if (epilogue == CQ_EPI_SWIGLU && N % kRows != 0) return CQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return CQ_OK;
  if (K == 0) return CQ_ERR_UNSUPPORTED;
  if (!x || !y) return CQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16)) return CQ_ERR_UNSUPPORTED;
  if (M > (int64_t)1 << 24) return CQ_ERR_UNSUPPORTED;
  const int sms = num_sms();
  if (sms <= 0) return CQ_ERR_CUDA;
  const GvPlan v = debug_skip ? GvPlan{} : plan_gemv(M, N, K, B, G, epilogue, sms);
  if (v.use)
    return run_gemv(v, x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype, y,
                    stream, timeout_ns, trace);
  const GemmPlan g = plan_gemm(M, N, K, epilogue, sms);
  const size_t need = g.ws_counter_bytes + g.ws_partial_bytes;
  if (ws_bytes < need || (need && !workspace)) return CQ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return CQ_ERR_UNSUPPORTED;

  CUtensorMap map, wmap;
  st = encode_bf16_rows_sw128(&map, x, M, K, g.NT);
  if (st != CQ_OK) return st;
  st = encode_packed_rows(&wmap, packed, N, K * B / 8, B);
  if (st != CQ_OK) return st;

  EngineParams p = {};
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
  p.counter = reinterpret_cast<int*>(workspace);
  p.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + g.ws_counter_bytes);
  p.timeout_ns = timeout_ns;
  p.debug_skip_first_stage = debug_skip;
  p.trace = trace;

  switch (g.NT) {
    case 16: return launch_engine<16>(p, map, wmap, stream);
    case 32: return launch_engine<32>(p, map, wmap, stream);
    case 64: return launch_engine<64>(p, map, wmap, stream);
    default: return launch_engine<128>(p, map, wmap, stream);
  }
}

size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K, int B, int G, int epilogue,
                           int sms) {
  if (M <= 0 || N <= 0 || K <= 0 || K % kSlice != 0 || G <= 0 || G % kSlice != 0 ||
      K % G != 0)
    return 0;
  size_t counters = 0, total = 0;
  gemm_scratch(M, N, K, B, G, epilogue, sms, &counters, &total);
  return total;
}

}  // namespace cq

using namespace cq;

extern "C" size_t cq_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int B, int G,
                                         int epilogue) {
  int sms = num_sms();
  if (sms <= 0) sms = 148;
  return gemm_workspace_size(M, N, K, B, G, epilogue, sms);
}

extern "C" int cq_gemm(const uint16_t* x, int64_t M, const uint8_t* packed, const float* scales,
                       const uint16_t* ab, int64_t N, int64_t K, int B, int G, int grid_mode,
                       int epilogue, int out_dtype, void* y, void* workspace, size_t ws_bytes,
                       void* stream) {
  return gemm_impl(x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype, y,
                   workspace, ws_bytes, static_cast<cudaStream_t>(stream), kDefaultTimeoutNs, 0);
}

// Profiling hook (not part of the public header): cq_gemm that also writes
// per-CTA event timestamps to trace ([grid][64] uint64, device memory, at
// least cq_gemm_workspace_size-independent 148*64 entries).
extern "C" CQ_API int cq_trace_gemm(const uint16_t* x, int64_t M, const uint8_t* packed,
                                    const float* scales, const uint16_t* ab, int64_t N,
                                    int64_t K, int B, int G, int epilogue, void* y,
                                    void* workspace, size_t ws_bytes, uint64_t* trace,
                                    void* stream) {
  return gemm_impl(x, M, packed, scales, ab, N, K, B, G, CQ_GRID_MIDRISE, epilogue,
                   CQ_DTYPE_F32, y, workspace, ws_bytes, static_cast<cudaStream_t>(stream),
                   kDefaultTimeoutNs, 0, trace);
}

// Test hook (not part of the public header): run cq_gemm with a chosen wait
// limit and, optionally, with the first stage load withheld so that the
// bounded waits run out; the caller then reads CQ_ERR_TIMEOUT from
// cq_get_device_error().
extern "C" CQ_API int cq_test_gemm_bounded(const uint16_t* x, int64_t M, const uint8_t* packed,
                                    const float* scales, const uint16_t* ab, int64_t N, int64_t K,
                                    int B, int G, void* y, void* workspace, size_t ws_bytes,
                                    uint64_t timeout_ns, int skip_first_stage, void* stream) {
  return gemm_impl(x, M, packed, scales, ab, N, K, B, G, CQ_GRID_MIDRISE, CQ_EPI_NONE,
                   CQ_DTYPE_F32, y, workspace, ws_bytes, static_cast<cudaStream_t>(stream),
                   timeout_ns, skip_first_stage);
}
