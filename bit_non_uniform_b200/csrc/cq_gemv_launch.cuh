// cq_gemv_launch.cuh -- host side of the decode-sized GEMM (M <= 2): the
// plan (row blocks per CTA, shared-memory layout), the 4-D tensor map over
// the packed matrix and the launch with programmatic dependent launch.
// Part of the single translation unit of libcq (included by cq_gemm.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "cq.h"
#include "cq_gemv.cuh"
#include "cq_host.h"

namespace cq {

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
  static std::atomic<uint64_t> smem_set{0};
  if (!ensure_smem_limit(gemv_kernel<B, MT>, 227 * 1024, smem_set)) return CQ_ERR_CUDA;
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

}  // namespace cq
