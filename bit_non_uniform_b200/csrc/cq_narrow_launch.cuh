// cq_narrow_launch.cuh -- host side of the narrow-row GEMM (M <= 16): the
// plan (units, CTA shares, shared-memory layout) and the launch with
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
  int MT, n_rb, Q, spc, ng, L, U, P, max_units, max_rbl;
  int tbl_off, x_off, slot_off, smem;
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
  const int64_t x_bytes = M * K * 2;              // every slice step of every token
  const int slot_bytes = 512 * (v.MT / 8);
  v.tbl_off = 0;
  v.x_off = (tbl_bytes + 1023) / 1024 * 1024;
  const int64_t slot_off = (v.x_off + x_bytes + 127) / 128 * 128;
  // the table base is aligned up to a table block (E * 128 bytes) from the
  // 16-byte aligned start of the dynamic shared memory
  const int64_t smem =
      E * 128 + slot_off + static_cast<int64_t>(v.max_units) * slot_bytes + kNrBarBytes +
      kNrOrderBytes;
  if (smem > 227 * 1024) return v;
  v.slot_off = static_cast<int>(slot_off);
  v.smem = static_cast<int>(smem);
  v.ws_counter_bytes = (static_cast<size_t>(v.n_rb) * sizeof(int) + 255) / 256 * 256;
  v.ws_partial_bytes = static_cast<size_t>(v.P) * 16 * v.MT * sizeof(float);
  v.use = true;
  return v;
}

template <int B, int MT>
static int launch_narrow(const NarrowParams& p, cudaStream_t s) {
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
  if (cudaLaunchKernelEx(&cfg, narrow_kernel<B, MT>, p) != cudaSuccess)
    return CQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

static int run_narrow(const NrPlan& v, const uint16_t* x, int64_t M, const uint8_t* packed,
                      const float* scales, const uint16_t* ab, int64_t N, int64_t K, int B,
                      int G, int grid_mode, int epilogue, int out_dtype, void* y,
                      void* workspace, cudaStream_t stream, uint64_t timeout_ns,
                      uint64_t* trace) {
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
  p.tbl_off = v.tbl_off;
  p.x_off = v.x_off;
  p.slot_off = v.slot_off;
  p.smem_bytes = v.smem;
  p.packed = packed;
  p.row_bytes = K * B / 8;
  p.scales = scales;
  p.ab = reinterpret_cast<const uint32_t*>(ab);
  p.x = x;
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
    if (B == 2) return launch_narrow<2, 8>(p, stream);
    if (B == 3) return launch_narrow<3, 8>(p, stream);
    return launch_narrow<4, 8>(p, stream);
  }
  if (B == 2) return launch_narrow<2, 16>(p, stream);
  if (B == 3) return launch_narrow<3, 16>(p, stream);
  return launch_narrow<4, 16>(p, stream);
}

}  // namespace cq
