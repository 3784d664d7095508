// cq_narrow_launch.cuh -- host side of the narrow-row GEMM (M <= 16): the
// plan (units, CTA shares, ring depths, shared-memory layout), the tensor
// maps over the packed matrix and the activations, and the launch with
// programmatic dependent launch.  Part of the single translation unit of
// libcq (included by cq_gemm.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "cq.h"
#include "cq_host.h"
#include "cq_narrow.cuh"

namespace cq {

struct NrPlan {
  bool use;
  int MT, n_rb, Q, spc, ng, L, U, P, max_units, max_rbl, CS, XS, resident_x;
  int tbl_off, code_off, x_off, slot_off, smem;
  size_t ws_counter_bytes, ws_partial_bytes;
};

static int64_t nr_begin_host(int64_t U, int64_t P, int64_t c) { return (c * U) / P; }

static NrPlan plan_narrow(int64_t M, int64_t N, int64_t K, int B, int G, int epilogue, int sms) {
  NrPlan v = {};
  if (M < 1 || M > 16 || N < 1 || K < 512 || B < 2 || B > 4 || sms < 1) return v;
  if (K % 512 != 0 || G % 128 != 0 || K % G != 0) return v;
  if (epilogue == CQ_EPI_SWIGLU && N % 16 != 0) return v;
  if (N >= (1 << 24) || K >= (1 << 24)) return v;
  v.MT = M <= 8 ? 8 : 16;
  v.Q = static_cast<int>(K / 512);
  if (v.Q > kNrMaxJ) return v;
  v.spc = G / 128;
  v.ng = static_cast<int>(K / G);
  for (int c = 0; c < 4; ++c) {
    const int l = ((c + 1) * v.Q - 1) / v.spc - (c * v.Q) / v.spc + 1;
    if (l > v.L) v.L = l;
  }
  v.n_rb = static_cast<int>(epilogue == CQ_EPI_SWIGLU ? N / 16 : (N + 15) / 16);
  const int64_t U = static_cast<int64_t>(v.n_rb) * v.Q;
  if (U >= (1 << 30)) return v;
  v.U = static_cast<int>(U);
  v.P = static_cast<int>(U < sms ? U : sms);
  for (int c = 0; c < v.P; ++c) {
    const int64_t a = nr_begin_host(U, v.P, c), b = nr_begin_host(U, v.P, c + 1);
    const int units = static_cast<int>(b - a);
    const int rbl = static_cast<int>((b - 1) / v.Q - a / v.Q + 1);
    if (units > v.max_units) v.max_units = units;
    if (rbl > v.max_rbl) v.max_rbl = rbl;
  }
  if (v.max_units > kNrMaxUnits || v.max_rbl > kNrMaxRbl) return v;
  const int E = B == 3 ? 64 : 16;
  const int tbl_bytes = v.max_rbl * 2 * v.L * E * 128;
  const int code_stage = 1024 * B;
  const int x_stage = 1024 * static_cast<int>(M);
  const int slot_bytes = 512 * (v.MT / 8);
  auto align = [](int x, int a) { return (x + a - 1) / a * a; };
  auto layout = [&](int CS, int XS) {
    v.CS = CS;
    v.XS = XS;
    v.tbl_off = 0;
    v.code_off = align(tbl_bytes, 1024);
    v.x_off = align(v.code_off + CS * code_stage, 1024);
    v.slot_off = align(v.x_off + XS * x_stage, 128);
    // the table base is aligned up to a table block (E * 128 bytes) from the
    // 16-byte aligned start of the dynamic shared memory
    v.smem = E * 128 + v.slot_off + v.max_units * slot_bytes + kNrBarBytes + kNrOrderBytes;
    return v.smem <= 227 * 1024;
  };
  // preferred: every slice step's activations resident and every unit's codes
  // in flight at once; then fewer code stages; then an activation ring
  const int cs_all = v.max_units < kNrMaxCS ? v.max_units : kNrMaxCS;
  bool fits = false;
  if (v.Q <= kNrMaxXS) {
    v.resident_x = 1;
    for (int CS = cs_all; CS >= 1 && !fits; CS = CS > 8 ? CS - 4 : CS - 1)
      fits = layout(CS, v.Q);
  }
  if (!fits) {
    v.resident_x = 0;
    const int xs0 = v.Q < 4 ? v.Q : 4;
    for (int XS = xs0; XS >= 2 && !fits; --XS)
      for (int CS = cs_all; CS >= 1 && !fits; CS = CS > 8 ? CS - 4 : CS - 1)
        fits = layout(CS, XS);
  }
  if (!fits) return v;
  v.ws_counter_bytes = (static_cast<size_t>(v.n_rb) * sizeof(int) + 255) / 256 * 256;
  v.ws_partial_bytes = static_cast<size_t>(v.P) * 16 * v.MT * sizeof(float);
  v.use = true;
  return v;
}

// Packed codes for the narrow kernel: one box = one slice (16*B bytes) of each
// of the four quarters of 16 rows (SwiGLU: 8 gate rows and the 8 matching up
// rows), landing in shared memory as [row][quarter][16*B bytes].
static int encode_packed_narrow(CUtensorMap* map, const void* base, int64_t N, int64_t K, int B,
                                int epilogue) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return CQ_ERR_CUDA;
  const int64_t row_bytes = K * B / 8;
  const int64_t quarter = row_bytes / 4;
  const cuuint32_t slice = static_cast<cuuint32_t>(16 * B);
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r;
  if (epilogue == CQ_EPI_SWIGLU) {
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(quarter), 4u,
                          static_cast<cuuint64_t>(N / 2), 2u};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(quarter),
                             static_cast<cuuint64_t>(row_bytes),
                             static_cast<cuuint64_t>((N / 2) * row_bytes)};
    cuuint32_t box[4] = {slice, 4u, 8u, 2u};
    r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(quarter), 4u, static_cast<cuuint64_t>(N)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(quarter),
                             static_cast<cuuint64_t>(row_bytes)};
    cuuint32_t box[3] = {slice, 4u, 16u};
    r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS ? CQ_OK : CQ_ERR_CUDA;
}

// Activations for the narrow kernel, bf16 [M][K] viewed as 4-D
//   (8 values [16 bytes], quarter [stride K/4 values], token [stride K],
//    8-value chunk within the quarter [stride 8 values]);
// one box = the 16 chunks of one slice step of all tokens and quarters,
// landing as [chunk][token][quarter][8 values].
static int encode_x_narrow(CUtensorMap* map, const void* x, int64_t M, int64_t K) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return CQ_ERR_CUDA;
  cuuint64_t dims[4] = {8u, 4u, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(K / 32)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(K / 4 * 2), static_cast<cuuint64_t>(K * 2),
                           16u};
  cuuint32_t box[4] = {8u, 4u, static_cast<cuuint32_t>(M), 16u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CQ_OK : CQ_ERR_CUDA;
}

template <int B, int MT>
static int launch_narrow(const NarrowParams& p, const CUtensorMap& wmap, const CUtensorMap& xmap,
                         cudaStream_t s) {
  static std::atomic<uint64_t> smem_set{0};
  if (!ensure_smem_limit(narrow_kernel<B, MT>, 227 * 1024, smem_set)) return CQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(p.P);
  cfg.blockDim = dim3(kNrThreads);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, narrow_kernel<B, MT>, p, wmap, xmap) != cudaSuccess)
    return CQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

static int run_narrow(const NrPlan& v, const uint16_t* x, int64_t M, const uint8_t* packed,
                      const float* scales, const uint16_t* ab, int64_t N, int64_t K, int B,
                      int G, int grid_mode, int epilogue, int out_dtype, void* y,
                      void* workspace, cudaStream_t stream, uint64_t timeout_ns,
                      uint64_t* trace) {
  CUtensorMap wmap, xmap;
  int st = encode_packed_narrow(&wmap, packed, N, K, B, epilogue);
  if (st != CQ_OK) return st;
  st = encode_x_narrow(&xmap, x, M, K);
  if (st != CQ_OK) return st;
  NarrowParams p = {};
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = G;
  p.mode = grid_mode;
  p.epilogue = epilogue;
  p.out_bf16 = out_dtype == CQ_DTYPE_BF16;
  p.M = static_cast<int>(M);
  p.n_rb = v.n_rb;
  p.Q = v.Q;
  p.spc = v.spc;
  p.ng = v.ng;
  p.L = v.L;
  p.U = v.U;
  p.P = v.P;
  p.max_rbl = v.max_rbl;
  p.max_units = v.max_units;
  p.CS = v.CS;
  p.XS = v.XS;
  p.resident_x = v.resident_x;
  p.tbl_off = v.tbl_off;
  p.code_off = v.code_off;
  p.x_off = v.x_off;
  p.slot_off = v.slot_off;
  p.smem_bytes = v.smem;
  p.scales = scales;
  p.ab = reinterpret_cast<const uint32_t*>(ab);
  p.y = y;
  p.ldy = epilogue == CQ_EPI_SWIGLU ? N / 2 : N;
  p.counter = reinterpret_cast<int*>(workspace);
  p.partial =
      reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + v.ws_counter_bytes);
  p.counter_len = v.n_rb;
  p.partial_slots = v.P;
  p.timeout_ns = timeout_ns;
  p.trace = reinterpret_cast<unsigned long long*>(trace);
  if (v.MT == 8) {
    if (B == 2) return launch_narrow<2, 8>(p, wmap, xmap, stream);
    if (B == 3) return launch_narrow<3, 8>(p, wmap, xmap, stream);
    return launch_narrow<4, 8>(p, wmap, xmap, stream);
  }
  if (B == 2) return launch_narrow<2, 16>(p, wmap, xmap, stream);
  if (B == 3) return launch_narrow<3, 16>(p, wmap, xmap, stream);
  return launch_narrow<4, 16>(p, wmap, xmap, stream);
}

}  // namespace cq
