// cq_moe.cu -- the grouped MoE layer: per-expert table preparation, device
// routing (route -> expert-sorted position), token gather, two grouped
// engine launches (gate/up + SwiGLU, down) and the weighted combine.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>
#include <vector>

#include "cq.h"
#include "cq_engine.cuh"
#include "cq_gemv.cuh"
#include "cq_host.h"

namespace cq {

constexpr int kRouteThreads = 1024;
constexpr int kMaxExperts = 16384;     // routing counters live in shared memory

// control words at the head of the workspace
enum Ctrl : int {
  CTRL_TT = 0, CTRL_TILES_GU = 1, CTRL_TILES_DN = 2, CTRL_BAD = 3,
  CTRL_CHUNKS = 8      // [2 stages][3 widths]: decode-path chunks per bit width
};

// Exclusive scan of v[0..n) in place with one CTA of kRouteThreads threads;
// returns the total (to every thread).  Each thread owns a contiguous chunk.
__device__ int block_exclusive_scan(int* v, int n, int* s_part) {
  const int tid = threadIdx.x;
  const int per = (n + kRouteThreads - 1) / kRouteThreads;
  const int b = tid * per;
  const int e = b + per < n ? b + per : n;
  int sum = 0;
  for (int i = b; i < e; ++i) sum += v[i];
  s_part[tid] = sum;
  __syncthreads();
  if (tid == 0) {                      // 1024 partial sums, scanned serially
    int run = 0;
    for (int i = 0; i < kRouteThreads; ++i) {
      const int t = s_part[i];
      s_part[i] = run;
      run += t;
    }
    s_part[kRouteThreads] = run;
  }
  __syncthreads();
  int run = s_part[tid];
  for (int i = b; i < e; ++i) {
    const int t = v[i];
    v[i] = run;
    run += t;
  }
  const int total = s_part[kRouteThreads];
  __syncthreads();
  return total;
}

// One CTA: count the routes of every expert, give each route its position in
// the expert-sorted order (experts ascending; inside an expert the order in
// which the atomics land, which no result depends on), the per-expert
// offsets, and the prefix of token tiles that the grouped launches walk.
__global__ void __launch_bounds__(kRouteThreads)
    moe_route_kernel(const int32_t* __restrict__ ids, int R, int E, int NT, int n_rt_gu,
                     int n_rt_dn, int* __restrict__ ctrl, int* __restrict__ cnt,
                     int* __restrict__ off, int* __restrict__ ttpre, int* __restrict__ rank,
                     int* __restrict__ perm, int* __restrict__ pos_of,
                     int* __restrict__ counters_gu, int* __restrict__ counters_dn,
                     const GvExpert* __restrict__ gvx, int* __restrict__ chunks, int max_chunks) {
  extern __shared__ int s_mem[];
  int* s_cnt = s_mem;                        // [E]
  int* s_tt = s_mem + E;                     // [E]
  int* s_part = s_mem + 2 * E;               // [kRouteThreads + 1]
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += kRouteThreads) s_cnt[e] = 0;
  if (tid == 0) ctrl[CTRL_BAD] = 0;
  __syncthreads();
  int bad = 0;
  for (int r = tid; r < R; r += kRouteThreads) {
    const int e = ids[r];
    if (e < 0 || e >= E) {
      rank[r] = -1;
      ++bad;
    } else {
      rank[r] = atomicAdd(&s_cnt[e], 1);
    }
  }
  if (bad) atomicAdd(&ctrl[CTRL_BAD], bad);
  __syncthreads();
  for (int e = tid; e < E; e += kRouteThreads) {
    cnt[e] = s_cnt[e];
    s_tt[e] = (s_cnt[e] + NT - 1) / NT;
  }
  __syncthreads();
  block_exclusive_scan(s_cnt, E, s_part);      // s_cnt now holds the offsets
  const int tt_total = block_exclusive_scan(s_tt, E, s_part);
  for (int e = tid; e < E; e += kRouteThreads) {
    off[e] = s_cnt[e];
    ttpre[e] = s_tt[e];
  }
  if (tid == 0) {
    ttpre[E] = tt_total;
    ctrl[CTRL_TT] = tt_total;
    ctrl[CTRL_TILES_GU] = n_rt_gu * tt_total;
    ctrl[CTRL_TILES_DN] = n_rt_dn * tt_total;
  }
  for (int r = tid; r < R; r += kRouteThreads) {
    const int rk = rank[r];
    if (rk >= 0) {
      const int pos = s_cnt[ids[r]] + rk;
      perm[pos] = r;
      pos_of[r] = pos;
    } else {
      pos_of[r] = -1;
    }
  }
  // stream-K tile counters of the two grouped launches start at zero
  for (int i = tid; i < n_rt_gu * tt_total; i += kRouteThreads) counters_gu[i] = 0;
  for (int i = tid; i < n_rt_dn * tt_total; i += kRouteThreads) counters_dn[i] = 0;
  if (!gvx) return;
  // decode path: chunks of at most two routes per expert, listed by bit width
  // (B = 2, 3, 4) and, within a width, by expert; per stage
  __syncthreads();
  for (int stage = 0; stage < 2; ++stage) {
    int* const ch_e = chunks + (stage * 3 + 0) * max_chunks;
    int* const ch_pos = chunks + (stage * 3 + 1) * max_chunks;
    int* const ch_m = chunks + (stage * 3 + 2) * max_chunks;
    int base = 0;
    for (int b = 2; b <= 4; ++b) {
      for (int e = tid; e < E; e += kRouteThreads)
        s_tt[e] = (gvx[stage * E + e].mat.B == b) ? (cnt[e] + 1) / 2 : 0;
      __syncthreads();
      const int n_b = block_exclusive_scan(s_tt, E, s_part);
      for (int e = tid; e < E; e += kRouteThreads) {
        if (gvx[stage * E + e].mat.B != b) continue;
        const int c = cnt[e];
        for (int j = 0; 2 * j < c; ++j) {
          const int idx = base + s_tt[e] + j;
          if (idx < max_chunks) {
            ch_e[idx] = e;
            ch_pos[idx] = off[e] + 2 * j;
            ch_m[idx] = c - 2 * j < 2 ? c - 2 * j : 2;
          }
        }
      }
      if (tid == 0) ctrl[CTRL_CHUNKS + stage * 3 + (b - 2)] = n_b;
      base += n_b;
      __syncthreads();
    }
  }
}

// Copy each routed token's activation row to its expert-sorted position.
__global__ void moe_gather_kernel(const uint4* __restrict__ tokens, int R, int k, int row16,
                                  const int* __restrict__ pos_of, uint4* __restrict__ xs) {
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < R; r += warps) {
    const int pos = pos_of[r];
    if (pos < 0) continue;
    const uint4* src = tokens + static_cast<int64_t>(r / k) * row16;
    uint4* dst = xs + static_cast<int64_t>(pos) * row16;
    for (int i = lane; i < row16; i += 32) dst[i] = src[i];
  }
}

// out[t] = sum_j w[t][j] * y[t*k + j] (j ascending, FP32); dropped routes
// contribute nothing and their per-route rows are cleared.
template <bool BF16>
__global__ void moe_combine_kernel(const float* __restrict__ y, int T, int k, int H,
                                   const float* __restrict__ w, const int* __restrict__ pos_of,
                                   float* __restrict__ route_rows, void* __restrict__ out) {
  const int t = blockIdx.x;
  if (t >= T) return;
  for (int j = 0; j < k; ++j) {
    if (pos_of[t * k + j] < 0 && route_rows) {
      float* row = route_rows + static_cast<int64_t>(t * k + j) * H;
      for (int h = threadIdx.x; h < H; h += blockDim.x) row[h] = 0.f;
    }
  }
  if (!out) return;
  for (int h4 = threadIdx.x; h4 < H / 4; h4 += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int r = t * k + j;
      if (pos_of[r] < 0) continue;
      const float wj = w[r];
      const float4 v = reinterpret_cast<const float4*>(y + static_cast<int64_t>(r) * H)[h4];
      acc.x += wj * v.x;
      acc.y += wj * v.y;
      acc.z += wj * v.z;
      acc.w += wj * v.w;
    }
    const int64_t o = static_cast<int64_t>(t) * H + 4 * h4;
    if (BF16) {
      __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(out) + o;
      ob[0] = __float2bfloat16_rn(acc.x);
      ob[1] = __float2bfloat16_rn(acc.y);
      ob[2] = __float2bfloat16_rn(acc.z);
      ob[3] = __float2bfloat16_rn(acc.w);
    } else {
      reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + o)[0] = acc;
    }
  }
}

}  // namespace cq

namespace cq {

static size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Token-tile width of both grouped launches, from the mean routes per expert.
static int moe_pick_nt(int64_t R, int E) {
  const int64_t mean = (R + E - 1) / (E > 0 ? E : 1);
  if (mean <= 16) return 16;
  if (mean <= 32) return 32;
  if (mean <= 64) return 64;
  return 128;
}

struct MoePlan {
  int NT, n_rt_gu, n_rt_dn, P;
  int64_t R, max_tt, max_chunks;
  size_t o_ctrl, o_cnt, o_off, o_ttpre, o_rank, o_perm, o_pos, o_x, o_h, o_y, o_cgu, o_cdn,
      o_part, o_chunks, total;
};

static MoePlan moe_plan(int64_t T, int k, int E, int64_t H, int64_t I, int sms) {
  MoePlan m;
  m.R = T * k;
  m.NT = moe_pick_nt(m.R, E);
  m.n_rt_gu = static_cast<int>(2 * I / kRows);
  m.n_rt_dn = static_cast<int>((H + kRows - 1) / kRows);
  m.P = sms;
  // sum over experts of ceil(cnt/NT) <= active experts + R/NT
  m.max_tt = (m.R < E ? m.R : E) + m.R / m.NT + 1;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += align256(bytes);
    return at;
  };
  m.o_ctrl = take(64 * sizeof(int));
  m.o_cnt = take(static_cast<size_t>(E) * sizeof(int));
  m.o_off = take(static_cast<size_t>(E + 1) * sizeof(int));
  m.o_ttpre = take(static_cast<size_t>(E + 1) * sizeof(int));
  m.o_rank = take(static_cast<size_t>(m.R) * sizeof(int));
  m.o_perm = take(static_cast<size_t>(m.R) * sizeof(int));
  m.o_pos = take(static_cast<size_t>(m.R) * sizeof(int));
  m.o_x = take(static_cast<size_t>(m.R) * H * 2);
  m.o_h = take(static_cast<size_t>(m.R) * I * 2);
  m.o_y = take(static_cast<size_t>(m.R) * H * 4);
  m.o_cgu = take(static_cast<size_t>(m.n_rt_gu) * m.max_tt * sizeof(int));
  m.o_cdn = take(static_cast<size_t>(m.n_rt_dn) * m.max_tt * sizeof(int));
  m.o_part = take(static_cast<size_t>(2) * m.P * m.NT * kRows * sizeof(float));
  // decode path: sum over experts of ceil(cnt/2) <= (R + active experts) / 2
  m.max_chunks = (m.R + (m.R < E ? m.R : E)) / 2 + 1;
  m.o_chunks = take(static_cast<size_t>(6) * m.max_chunks * sizeof(int));
  m.total = o;
  return m;
}

static int validate_moe_shape(int64_t T, int k, int E, int64_t H, int64_t I, int G) {
  if (T < 0 || k <= 0 || E <= 0 || H <= 0 || I <= 0 || G <= 0) return CQ_ERR_INVALID_ARG;
  if (E > kMaxExperts) return CQ_ERR_UNSUPPORTED;
  if (G % 128 != 0 || H % G != 0 || I % G != 0 || I % 64 != 0) return CQ_ERR_UNSUPPORTED;
  if (T * k > (int64_t)1 << 28 || H > (int64_t)1 << 20 || I > (int64_t)1 << 20)
    return CQ_ERR_UNSUPPORTED;
  return CQ_OK;
}

// Decode-sized grouped path: usable when experts see few routes on average
// and the GEMV kernel fits every bit width's work item in shared memory.
static bool moe_gemv_plan(const MoePlan& m, int64_t T, int k, int E, int64_t H, int64_t I, int G,
                          int grid_mode, int sms, MoeGvParams* q) {
  const int64_t active = m.R < E ? m.R : E;
  if (m.R > 4 * active || G / 8 * 4 > 256) return false;
  for (int stage = 0; stage < 2; ++stage) {
    const int64_t N = stage == 0 ? 2 * I : H;
    const int64_t K = stage == 0 ? H : I;
    MoeGvParams& p = q[stage];
    memset(&p, 0, sizeof(p));
    GemvParams& b = p.base;
    b.N = static_cast<int>(N);
    b.K = static_cast<int>(K);
    b.G = G;
    b.mode = grid_mode;
    b.epilogue = stage == 0 ? CQ_EPI_SWIGLU : CQ_EPI_NONE;
    b.out_bf16 = stage == 0 ? 1 : 0;
    b.M = 2;
    b.ng = static_cast<int>(K / G);
    b.n_rb = static_cast<int>(stage == 0 ? N / 16 : (N + 15) / 16);
    b.n_cols = b.n_rb * b.ng;
    b.spc = G / 128;
    b.gpair = b.ng % 2 == 0 ? 2 : 1;
    b.spc_magic = b.spc > 1 ? static_cast<uint32_t>(((1ull << 32) + b.spc - 1) / b.spc) : 0u;
    b.x_bytes = static_cast<int>((2 * K * 2 + 127) / 128 * 128);
    b.ldy = stage == 0 ? I : H;
    b.timeout_ns = kDefaultTimeoutNs;
    int smem = 0;
    for (int bi = 0; bi < 3; ++bi) {
      const int B = bi + 2;
      int rpc = (b.n_rb + sms - 1) / sms;
      if (rpc > kGvMaxRb) rpc = kGvMaxRb;
      int sm = 0, mq = 0;
      for (; rpc >= 1; --rpc) {
        mq = (rpc * b.ng + 3) / 4 + 1;
        if (mq > kGvMaxQuads) continue;
        sm = gv_dynamic_smem(B, 2, G, b.spc, b.x_bytes, mq);
        if (sm <= 227 * 1024) break;
      }
      if (rpc < 1) return false;
      p.rpc[bi] = rpc;
      p.max_quads[bi] = mq;
      p.ipi[bi] = (b.n_rb + rpc - 1) / rpc;
      if (sm > smem) smem = sm;
    }
    b.smem_bytes = smem;
  }
  return true;
}

// Experts may mix bit widths: 64-entry pair tables (any of 2, 3, 4 bits), or
// the wide-code decoder when the layer has a width outside {2, 3, 4}.
template <int NT>
static int launch_grouped(const EngineParams& p, const CUtensorMap& xmap, bool wide,
                          cudaStream_t s) {
  CUtensorMap unused;
  memset(&unused, 0, sizeof(unused));
  if (wide) return launch_engine<NT, 0>(p, xmap, unused, s);
  return launch_engine<NT, 64>(p, xmap, unused, s);
}

static int launch_grouped_nt(int NT, const EngineParams& p, const CUtensorMap& xmap, bool wide,
                             cudaStream_t s) {
  switch (NT) {
    case 16: return launch_grouped<16>(p, xmap, wide, s);
    case 32: return launch_grouped<32>(p, xmap, wide, s);
    case 64: return launch_grouped<64>(p, xmap, wide, s);
    default: return launch_grouped<128>(p, xmap, wide, s);
  }
}

// The code widths of every layer table cq_moe_prepare_layer wrote, by the
// table's device address: the grouped launches pick their decoder from it
// without reading the table back.  A table it does not know is taken to hold
// widths 2..4 only (a wider expert in it is flagged on the device).
struct LayerWidths {
  int bmin, bmax;
};
static std::mutex g_layer_mu;
static std::unordered_map<const void*, LayerWidths> g_layer_widths;

static void remember_layer(const void* layer, LayerWidths w) {
  std::lock_guard<std::mutex> lock(g_layer_mu);
  g_layer_widths[layer] = w;
}

static void forget_layer(const void* layer) {
  std::lock_guard<std::mutex> lock(g_layer_mu);
  g_layer_widths.erase(layer);
}

static LayerWidths layer_widths(const void* layer) {
  std::lock_guard<std::mutex> lock(g_layer_mu);
  const auto it = g_layer_widths.find(layer);
  return it == g_layer_widths.end() ? LayerWidths{2, 4} : it->second;
}

}  // namespace cq

using namespace cq;

// Layer table: [E] LayerEntry (engine) followed by [2][E] GvExpert (the
// decode-sized path's per-expert tensor maps; a B whose group rows do not fit
// one box row leaves the map zero and the layer on the engine).
static size_t gv_table_offset(int E) { return static_cast<size_t>(E) * sizeof(LayerEntry); }

extern "C" size_t cq_moe_layer_bytes(int E) {
  return E > 0 ? gv_table_offset(E) + static_cast<size_t>(2) * E * sizeof(GvExpert) : 0;
}

extern "C" int cq_moe_prepare_layer(const cq_expert_desc* experts, int E, int64_t H, int64_t I,
                                    int G, void* layer) {
  int st = validate_moe_shape(1, 1, E, H, I, G);
  if (st != CQ_OK) return st;
  if (!experts || !layer) return CQ_ERR_INVALID_ARG;
  if (!aligned(layer, 64)) return CQ_ERR_UNSUPPORTED;
  forget_layer(layer);
  LayerWidths lw = {8, 1};
  std::vector<LayerEntry> host(static_cast<size_t>(E));
  memset(host.data(), 0, host.size() * sizeof(LayerEntry));
  std::vector<GvExpert> gvx(static_cast<size_t>(2) * E);
  memset(gvx.data(), 0, gvx.size() * sizeof(GvExpert));
  for (int e = 0; e < E; ++e) {
    const cq_matrix_desc* d[2] = {&experts[e].gate_up, &experts[e].down};
    const int64_t rows[2] = {2 * I, H};
    const int64_t cols[2] = {H, I};
    for (int w = 0; w < 2; ++w) {
      if (d[w]->reserved != 0) return CQ_ERR_INVALID_ARG;
      st = validate_matrix(d[w]->packed, d[w]->scales, d[w]->ab, rows[w], cols[w], d[w]->B, G,
                           CQ_GRID_MIDRISE, 1, 8);
      if (st != CQ_OK) return st;
      lw.bmin = d[w]->B < lw.bmin ? d[w]->B : lw.bmin;
      lw.bmax = d[w]->B > lw.bmax ? d[w]->B : lw.bmax;
      st = encode_packed_rows(&host[e].map[w], d[w]->packed, rows[w], cols[w] * d[w]->B / 8,
                              d[w]->B);
      if (st != CQ_OK) return st;
      host[e].mat[w].packed = d[w]->packed;
      host[e].mat[w].scales = d[w]->scales;
      host[e].mat[w].ab = reinterpret_cast<const uint32_t*>(d[w]->ab);
      host[e].mat[w].B = d[w]->B;
      host[e].mat[w].reserved = 0;
      GvExpert& g = gvx[static_cast<size_t>(w) * E + e];
      g.mat.packed = d[w]->packed;
      g.mat.scales = d[w]->scales;
      g.mat.ab = reinterpret_cast<const uint32_t*>(d[w]->ab);
      g.mat.B = d[w]->B;
      if (d[w]->B >= 2 && d[w]->B <= 4 && G / 8 * d[w]->B <= 256) {
        const int ng = static_cast<int>(cols[w] / G);
        st = encode_packed_gemv(&g.map, d[w]->packed, rows[w], cols[w], d[w]->B, G,
                                w == 0 ? CQ_EPI_SWIGLU : CQ_EPI_NONE, ng % 2 == 0 ? 2 : 1);
        if (st != CQ_OK) return st;
      }
    }
  }
  if (cudaMemcpy(layer, host.data(), host.size() * sizeof(LayerEntry),
                 cudaMemcpyHostToDevice) != cudaSuccess)
    return CQ_ERR_CUDA;
  if (cudaMemcpy(static_cast<uint8_t*>(layer) + gv_table_offset(E), gvx.data(),
                 gvx.size() * sizeof(GvExpert), cudaMemcpyHostToDevice) != cudaSuccess)
    return CQ_ERR_CUDA;
  remember_layer(layer, lw);
  return CQ_OK;
}

extern "C" size_t cq_moe_workspace_size(int64_t T, int k, int E, int64_t H, int64_t I, int G) {
  if (validate_moe_shape(T, k, E, H, I, G) != CQ_OK) return 0;
  int sms = num_sms();
  if (sms <= 0) sms = 148;
  return moe_plan(T, k, E, H, I, sms).total;
}

extern "C" int cq_moe_grouped_gemm(const uint16_t* tokens, int64_t T, const int32_t* topk_ids,
                                   const float* topk_w, int k, int E, const void* layer,
                                   int64_t H, int64_t I, int G, int grid_mode, int out_dtype,
                                   void* route_out, void* out, void* workspace, size_t ws_bytes,
                                   void* stream) {
  int st = validate_moe_shape(T, k, E, H, I, G);
  if (st != CQ_OK) return st;
  if (grid_mode != CQ_GRID_MIDRISE && grid_mode != CQ_GRID_MIDTREAD) return CQ_ERR_INVALID_ARG;
  if (out_dtype != CQ_DTYPE_F32 && out_dtype != CQ_DTYPE_BF16) return CQ_ERR_INVALID_ARG;
  if (T == 0) return CQ_OK;
  if (!tokens || !topk_ids || !layer || !workspace) return CQ_ERR_INVALID_ARG;
  if (out && !topk_w) return CQ_ERR_INVALID_ARG;
  if (!aligned(tokens, 16) || !aligned(layer, 64) || !aligned(workspace, 256) ||
      (route_out && !aligned(route_out, 16)) || (out && !aligned(out, 16)))
    return CQ_ERR_UNSUPPORTED;
  const LayerWidths lw = layer_widths(layer);
  const bool wide = lw.bmin < 2 || lw.bmax > 4;
  if (grid_mode == CQ_GRID_MIDTREAD && lw.bmin < 2) return CQ_ERR_UNSUPPORTED;
  const int sms = num_sms();
  if (sms <= 0) return CQ_ERR_CUDA;
  const MoePlan m = moe_plan(T, k, E, H, I, sms);
  if (ws_bytes < m.total) return CQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* ctrl = reinterpret_cast<int*>(ws + m.o_ctrl);
  int* cnt = reinterpret_cast<int*>(ws + m.o_cnt);
  int* off = reinterpret_cast<int*>(ws + m.o_off);
  int* ttpre = reinterpret_cast<int*>(ws + m.o_ttpre);
  int* rank = reinterpret_cast<int*>(ws + m.o_rank);
  int* perm = reinterpret_cast<int*>(ws + m.o_perm);
  int* pos_of = reinterpret_cast<int*>(ws + m.o_pos);
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + m.o_x);
  uint16_t* hs = reinterpret_cast<uint16_t*>(ws + m.o_h);
  float* ybuf = route_out ? static_cast<float*>(route_out) : reinterpret_cast<float*>(ws + m.o_y);
  int* cgu = reinterpret_cast<int*>(ws + m.o_cgu);
  int* cdn = reinterpret_cast<int*>(ws + m.o_cdn);
  float* part = reinterpret_cast<float*>(ws + m.o_part);
  const int R = static_cast<int>(m.R);

  // 1. routing
  const size_t route_smem = (2 * static_cast<size_t>(E) + kRouteThreads + 1) * sizeof(int);
  static std::atomic<uint64_t> route_smem_set{0};
  if (!ensure_smem_limit(moe_route_kernel,
                         static_cast<int>((2 * kMaxExperts + kRouteThreads + 1) * sizeof(int)),
                         route_smem_set))
    return CQ_ERR_CUDA;
  // decode-sized layers (few routes per expert) take the grouped GEMV path
  MoeGvParams gvp[2];
  const bool gv = !wide && moe_gemv_plan(m, T, k, E, H, I, G, grid_mode, sms, gvp);
  const GvExpert* gvx = reinterpret_cast<const GvExpert*>(
      static_cast<const uint8_t*>(layer) + gv_table_offset(E));
  int* chunks = reinterpret_cast<int*>(ws + m.o_chunks);
  moe_route_kernel<<<1, kRouteThreads, route_smem, s>>>(
      topk_ids, R, E, m.NT, m.n_rt_gu, m.n_rt_dn, ctrl, cnt, off, ttpre, rank, perm, pos_of,
      cgu, cdn, gv ? gvx : nullptr, chunks, static_cast<int>(m.max_chunks));
  if (cudaGetLastError() != cudaSuccess) return CQ_ERR_CUDA;
  // 2. expert-sorted activations
  const int row16 = static_cast<int>(H * 2 / 16);
  moe_gather_kernel<<<sms * 4, 256, 0, s>>>(reinterpret_cast<const uint4*>(tokens), R, k, row16,
                                            pos_of, reinterpret_cast<uint4*>(xs));
  if (cudaGetLastError() != cudaSuccess) return CQ_ERR_CUDA;
  // 3. gate/up + SwiGLU -> h (BF16, sorted order);  4. down -> y (FP32, route order)
  CUtensorMap xmap_gu, xmap_dn;
  if (gv) {
    for (int stage = 0; stage < 2; ++stage) {
      MoeGvParams& q = gvp[stage];
      q.experts = gvx + static_cast<size_t>(stage) * E;
      q.E = E;
      q.n_chunks = ctrl + CTRL_CHUNKS + 3 * stage;
      q.chunk_e = chunks + (stage * 3 + 0) * m.max_chunks;
      q.chunk_pos = chunks + (stage * 3 + 1) * m.max_chunks;
      q.chunk_m = chunks + (stage * 3 + 2) * m.max_chunks;
      q.xs = stage == 0 ? xs : hs;
      q.y = stage == 0 ? static_cast<void*>(hs) : static_cast<void*>(ybuf);
      q.base.y = q.y;                  // the per-CTA body writes through the stage shape
      q.out_rows = stage == 0 ? nullptr : perm;
      q.y_rows = m.R;
      q.R = m.R;
      static std::atomic<uint64_t> smem_set{0};
      if (!ensure_smem_limit(moe_gemv_kernel<2>, 227 * 1024, smem_set)) return CQ_ERR_CUDA;
      moe_gemv_kernel<2><<<sms, kGvThreads, q.base.smem_bytes, s>>>(q);
      if (cudaGetLastError() != cudaSuccess) return CQ_ERR_CUDA;
    }
  }
  st = encode_bf16_rows_sw128(&xmap_gu, xs, R, H, m.NT);
  if (st != CQ_OK) return st;
  st = encode_bf16_rows_sw128(&xmap_dn, hs, R, I, m.NT);
  if (st != CQ_OK) return st;
  for (int which = 0; which < 2 && !gv; ++which) {
    EngineParams p = {};
    p.N = static_cast<int>(which == 0 ? 2 * I : H);
    p.K = static_cast<int>(which == 0 ? H : I);
    p.G = G;
    p.mode = grid_mode;
    p.epilogue = which == 0 ? CQ_EPI_SWIGLU : CQ_EPI_NONE;
    p.out_bf16 = which == 0 ? 1 : 0;
    p.n_rt = which == 0 ? m.n_rt_gu : m.n_rt_dn;
    p.spt = p.K / kSlice;
    p.P = m.P;
    p.grouped = 1;
    p.which = which;
    p.layer = static_cast<const LayerEntry*>(layer);
    p.g_ttpre = ttpre;
    p.g_cnt = cnt;
    p.g_off = off;
    p.g_num_tiles = ctrl + (which == 0 ? CTRL_TILES_GU : CTRL_TILES_DN);
    p.out_rows = which == 0 ? nullptr : perm;
    p.E = E;
    p.y = which == 0 ? static_cast<void*>(hs) : static_cast<void*>(ybuf);
    p.ldy = which == 0 ? I : H;
    p.partial = part;
    p.counter = which == 0 ? cgu : cdn;
    p.y_rows = m.R;
    p.partial_slots = 2 * m.P;
    p.counter_len = static_cast<int>((which == 0 ? m.n_rt_gu : m.n_rt_dn) * m.max_tt);
    p.timeout_ns = kDefaultTimeoutNs;
    st = launch_grouped_nt(m.NT, p, which == 0 ? xmap_gu : xmap_dn, wide, s);
    if (st != CQ_OK) return st;
  }
  // 5. weighted combine (and clearing of dropped routes' rows)
  if (out || route_out) {
    if (out_dtype == CQ_DTYPE_BF16)
      moe_combine_kernel<true><<<static_cast<int>(T), 256, 0, s>>>(
          ybuf, static_cast<int>(T), k, static_cast<int>(H), topk_w, pos_of,
          route_out ? static_cast<float*>(route_out) : nullptr, out);
    else
      moe_combine_kernel<false><<<static_cast<int>(T), 256, 0, s>>>(
          ybuf, static_cast<int>(T), k, static_cast<int>(H), topk_w, pos_of,
          route_out ? static_cast<float*>(route_out) : nullptr, out);
    if (cudaGetLastError() != cudaSuccess) return CQ_ERR_CUDA;
  }
  return CQ_OK;
}
