// cq_gemv.cuh -- decode-sized CubicQuant GEMM (M <= 2 activation rows) for
// sm_100a.
//
// At one or two tokens the weight-only GEMM streams the packed weights once
// and is bound by how fast they can be decoded: every pair of codes becomes a
// BF16x2 operand word through a per-(row, group) lookup table in shared
// memory, and those lookups set the pace.  This kernel keeps everything else
// off that path: the decoded words go straight into the register operands
// of the warp-level tensor-core MMA (m16n8k16, FP32 accumulate), no decoded
// weight is ever stored, and the CTA runs in four phases with no
// producer/consumer hand-offs inside the hot loop.
//
// Work decomposition.  A row block is 16 weight rows (with the SwiGLU
// epilogue: 8 gate rows and the 8 matching up rows, i.e. 8 output columns).
// A column is (row block, group); columns are numbered row-block-major and
// taken four at a time ("quads").  A task is (quad, slice step s): lane
// (g, c) of a warp decodes the whole 128-code slice (s + c) mod spc of
// column c for rows g and g+8 (32 MMA steps).  The four lanes of an MMA row
// therefore work on four different columns, so every lane reads its own
// table (conflict free) and the MMA's N dimension keeps the columns apart:
// only lane (c, c) feeds activations into operand column c (for two tokens,
// lanes (2c+m, c) feed column 2c+m), so D[g][c] is exactly column c's
// partial dot product.  Rotating the slice by c also makes the 16-byte code
// reads conflict free.  A task is 8192 weights for every B.
//
// Each CTA owns whole row blocks (ceil(row blocks / SMs) of them), so no
// result ever crosses CTAs: the launch uses fewer CTAs than SMs when the
// row blocks do not divide evenly, and a quad that straddles two CTAs' row
// blocks is decoded by both (each keeps its own columns).
//
// Phases of a CTA:
//   A  one thread sets up the barriers; every thread waits for the
//      preceding grid (programmatic dependent launch).
//   B  one warp issues the TMA loads (one box per pair of columns: 16 rows x
//      whole group rows) and the activation copy; the compute warps build
//      every level table of the CTA's quads (FP64 levels -> FP32 -> BF16
//      pairs).
//   C  the compute warps decode and multiply their tasks; a task's partial
//      results go to a shared slot.
//   D  row-block sums in a fixed order (deterministic) and the output, with
//      the SwiGLU epilogue.
//
// Follows the article's A16 path (decode in the tile, model-dtype operand,
// FP32 accumulation; the group scale folded into the BF16 level as in the
// tensor-core engine).
#pragma once

#include "cq.h"
#include "cq_device.cuh"

namespace cq {

constexpr int kGvCompute = 12;            // warps that build tables and decode
constexpr int kGvTmaWarp = 12;            // issues the TMA loads
constexpr int kGvWarps = 13;
constexpr int kGvThreads = kGvWarps * 32;
constexpr int kGvMaxQuads = 24;         // quads one CTA may touch
constexpr int kGvMaxRb = 16;            // row blocks one CTA may own
// barriers and flags: a fixed block at the end of the dynamic shared memory
// (the same place for every work item of a persistent CTA)
constexpr int kGvBarBytes = 8 * (kGvMaxQuads + 1) + 64;

struct GemvParams {
  int N, K, G;
  int mode, epilogue, out_bf16;
  int M;               // activation rows (1..MT)
  int ng;              // groups per row, K / G
  int n_rb;            // row blocks
  int n_cols;          // n_rb * ng
  int spc;             // 128-code slices per group, G / 128
  int rpc;             // row blocks per CTA
  int P;               // CTAs, ceil(n_rb / rpc)
  int gpair;           // columns per TMA box (2 when ng is even, else 1)
  uint32_t spc_magic;  // ceil(2^32 / spc) when spc > 1
  int max_quads;       // largest number of quads of one CTA (shared layout)
  const float* scales;
  const uint32_t* ab;  // (a | b << 16), fp16 bits
  const uint16_t* x;   // [M][K] bf16
  int x_bytes;         // shared bytes reserved for x (>= M*K*2, multiple of 128)
  int smem_bytes;      // dynamic shared memory of the launch
  void* y;
  int64_t ldy;
  uint64_t timeout_ns;
  unsigned long long* trace;   // optional [P][64] clock64 stamps, or null
};

// The share of one CTA: row blocks [rb_first, rb_first + n_rbl) of one
// matrix, multiplied with M activation rows; output row m goes to element
// offset y_off[m] of y.
struct GvCta {
  int rb_first, n_rbl, M;
  const uint16_t* x;       // [M][K] bf16
  const float* scales;
  const uint32_t* ab;
  int64_t y_off[2];
};

#define GV_STAMP(k)                                                                 \
  do {                                                                              \
    if (p.trace) p.trace[blockIdx.x * 64 + (k)] = clock64();                        \
  } while (0)

template <int B, int MT>
struct GvCfg {
  static constexpr int E = (B == 3) ? 64 : 16;         // table entries per (row, group)
  static constexpr int SET_BYTES = 2 * E * 32 * 4;     // tables of one quad (both items)
  static constexpr int SLICE_BYTES = 16 * B;           // one 128-code slice of a row
  static constexpr int NV = 64 * MT;                   // values of one task partial
  // dynamic shared memory (the first 16 KB are alignment slack: the tables
  // start on a 16 KB boundary)
  static int smem_bytes(int G, int spc, int x_bytes, int max_quads) {
    const int quad_bytes = 64 * (G / 8 * B);
    return 16384 + max_quads * (SET_BYTES + quad_bytes) + x_bytes + max_quads * spc * NV * 4 +
           kGvMaxRb * 16 * MT * 4 + kGvBarBytes;
  }
};

// Row of item `it` (0: rows g, 1: rows g+8 of the MMA) of row block rb.
__device__ __forceinline__ int gv_row(int N, int epilogue, int rb, int it, int g) {
  if (epilogue == CQ_EPI_SWIGLU) return (it == 0 ? 0 : (N >> 1)) + rb * 8 + g;
  return rb * 16 + it * 8 + g;
}

// BF16 bits of the 2^B levels of one (row, group), by the same arithmetic as
// the engine's tables and the cq_decode kernel: q(t) in FP64 from the exact
// FP16 a, b, times s, rounded once to FP32 and then to BF16.  Levels are odd
// in k, so the positive side is evaluated and mirrored.
template <int B>
__device__ __forceinline__ void gv_levels(bool valid, float s, uint32_t abw, int mode,
                                          uint32_t (&L)[1 << B]) {
  constexpr int H = 1 << (B - 1);
  if (!valid) {
#pragma unroll
    for (int u = 0; u < (1 << B); ++u) L[u] = 0u;
    return;
  }
  const double a = static_cast<double>(__half2float(__ushort_as_half(abw & 0xFFFFu)));
  const double b = static_cast<double>(__half2float(__ushort_as_half(abw >> 16)));
  if (mode == CQ_GRID_MIDRISE) {
#pragma unroll
    for (int j = 0; j < H; ++j) {
      const uint32_t m = bf16_bits(static_cast<float>(level_f64(H + j, B, 0, s, a, b)));
      L[H + j] = m;
      L[H - 1 - j] = m ^ 0x8000u;
    }
  } else {
#pragma unroll
    for (int m = 0; m <= H; ++m) {
      const uint32_t v = bf16_bits(static_cast<float>(level_f64(H - 1 + m, B, 1, s, a, b)));
      L[H - 1 + m] = v;
      if (m >= 1 && m <= H - 1) L[H - 1 - m] = v ^ 0x8000u;
    }
  }
}

// Bits [sh, ...) of w moved to bit 7 (a table entry is 128 bytes away from
// the next: 32 lanes' words).
__device__ __forceinline__ uint32_t gv_at7(uint32_t w, int sh) {
  return sh >= 7 ? (w >> (sh - 7)) : (w << (7 - sh));
}

// Table word for pair q (codes 2q, 2q+1) of a 128-code slice held in c[].
// tl = byte address of this lane's word of entry 0 of the table.
template <int B>
__device__ __forceinline__ uint32_t gv_pair(const uint32_t (&c)[4 * B], int q, uint32_t tl) {
  if constexpr (B == 2) {
    const uint32_t v = gv_at7(c[q >> 3], 4 * (q & 7));
    return lds32((v & (15u << 7)) | tl);
  } else if constexpr (B == 3) {
    const int o = 6 * q;
    const int wi = o >> 5, sh = o & 31;
    uint32_t v;
    if (sh <= 26)
      v = gv_at7(c[wi], sh);
    else
      v = __funnelshift_r(c[wi], c[wi + 1 < 12 ? wi + 1 : 11], sh - 7);
    return lds32((v & (63u << 7)) | tl);
  } else {
    const uint32_t w = c[q >> 2];
    const int sh = 8 * (q & 3);
    const uint32_t lo = lds32((gv_at7(w, sh) & (15u << 7)) | tl);
    const uint32_t hi = lds32((gv_at7(w, sh + 4) & (15u << 7)) | tl);
    return __byte_perm(lo, hi, 0x7610);
  }
}

__device__ __forceinline__ bool gv_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                        uint64_t timeout_ns, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait(bar, parity, abort, timeout_ns, site);
}

// Warp-wide wait: every lane waits, then the warp reconverges (lanes leave
// the bounded spin at different iterations; without the reconvergence the
// code after the wait would run lane group by lane group).
__device__ __forceinline__ bool gv_wait_warp(uint32_t bar, uint32_t parity, volatile int* abort,
                                             uint64_t timeout_ns, int site) {
  const bool ok = gv_wait(bar, parity, abort, timeout_ns, site);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ float gv_silu(float g) { return g / (1.0f + expf(-g)); }

// n / spc (n < 2^26, spc <= 64).
__device__ __forceinline__ int gv_div_spc(const GemvParams& p, int n) {
  return p.spc == 1 ? n : static_cast<int>(__umulhi(static_cast<uint32_t>(n), p.spc_magic));
}

// Part `sub` (0..3) of the sum of one output (entry e0 of column 0, row
// block rb) over the row block's columns and their slice steps: the groups
// gi = sub, sub + 4, ... in order, each group's slice steps in order
// (task k of the CTA = its k-th quad-slice).  Four threads build the four
// parts, which are then added in a fixed order.
template <int NV, int MT>
__device__ __forceinline__ float gv_rb_sum_part(const GemvParams& p, uint32_t slots, int rb,
                                                int e0, int q_first, int sub) {
  float v = 0.f;
  for (int gi = sub; gi < p.ng; gi += 4) {
    const int chi = rb * p.ng + gi;
    const int kb = ((chi >> 2) - q_first) * p.spc;
    const uint32_t src = slots + 4u * static_cast<uint32_t>((chi & 3) * (16 * MT) + e0);
    float t[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      t[u] = u < p.spc ? __uint_as_float(lds32(src + 4u * static_cast<uint32_t>(NV * (kb + u))))
                       : 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) v += t[u];
    for (int st = 4; st < p.spc; ++st)
      v += __uint_as_float(lds32(src + 4u * static_cast<uint32_t>(NV * (kb + st))));
  }
  return v;
}

template <int B, int MT>
__device__ __forceinline__ void gemv_cta(const GemvParams& p, const CUtensorMap* wmap,
                                         const GvCta& w, int max_quads, bool reuse) {
  using C = GvCfg<B, MT>;
  constexpr int E = C::E;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 16383u) & ~16383u;
  uint8_t* const gbase = smem_raw + (base - raw);
  const int RG = p.G / 8 * B;                  // bytes of one group of one row
  const int quad_bytes = 64 * RG;              // 4 columns x 16 rows
  const uint32_t tbl0 = base;                                          // [quads][2][E][32]
  const uint32_t codes0 = tbl0 + max_quads * C::SET_BYTES;            // [quads][4][16][RG]
  const uint32_t xs = codes0 + max_quads * quad_bytes;                // [M][K] bf16
  const uint32_t slots = xs + static_cast<uint32_t>(p.x_bytes);       // [tasks][NV] f32
  const uint32_t outs = slots + max_quads * p.spc * C::NV * 4;        // [rb][16][MT] f32
  const uint32_t bars = raw + static_cast<uint32_t>(p.smem_bytes - kGvBarBytes);
  const uint32_t bar_quad = bars;                                     // [kGvMaxQuads]
  const uint32_t bar_x = bar_quad + 8 * kGvMaxQuads;
  volatile int* const flags = reinterpret_cast<volatile int*>(gbase + (bar_x + 8 - base));
  float* const slot_f = reinterpret_cast<float*>(gbase + (slots - base));
  float* const out_f = reinterpret_cast<float*>(gbase + (outs - base));
  uint32_t* const tblw = reinterpret_cast<uint32_t*>(gbase);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint64_t tmo = p.timeout_ns;

  // this CTA's row blocks, columns, quads and tasks (quad-slices)
  const int rb_first = w.rb_first;
  const int n_rbl = w.n_rbl;
  const int col0 = rb_first * p.ng;
  const int col1 = (rb_first + n_rbl) * p.ng;
  const int q_first = col0 >> 2;
  const int n_quads = ((col1 - 1) >> 2) - q_first + 1;
  const int n_loc = n_quads * p.spc;

  // ------------------------------------------------------------------ phase A
  if (tid == 0) {
    GV_STAMP(0);
    griddep_launch_dependents();
    if (reuse) {
      // a persistent CTA's previous item: every phase of these barriers has
      // completed and nothing waits on them any more
      for (int q = 0; q < kGvMaxQuads; ++q) mbar_inval(bar_quad + 8 * q);
      mbar_inval(bar_x);
    }
    for (int q = 0; q < kGvMaxQuads; ++q) mbar_init(bar_quad + 8 * q, 1);
    mbar_init(bar_x, 1);
    int bad = 0;
    if (n_rbl <= 0 || n_quads > max_quads || n_rbl > kGvMaxRb || n_quads > kGvMaxQuads ||
        w.M < 1 || w.M > MT)
      bad = 32;
    flags[0] = bad;
    if (bad) atomicCAS(&g_device_error, 0, bad);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  if (tid == 0) GV_STAMP(2);
  if (flags[0]) return;

  // ------------------------------------------------------------------ phase B
  if (warp == kGvTmaWarp && lane == 0) {
    prefetch_tensormap(wmap);
    const uint32_t xbytes = static_cast<uint32_t>(w.M) * p.K * 2u;
    mbar_arrive_expect_tx(bar_x, xbytes);
    for (int m = 0; m < w.M; ++m)
      bulk_g2s(xs + m * p.K * 2, w.x + static_cast<int64_t>(m) * p.K, p.K * 2u, bar_x);
    const int box_bytes = p.gpair * 16 * RG;
    const int nbox = 4 / p.gpair;
    for (int qq = 0; qq < n_quads; ++qq) {
      const int Q = q_first + qq;
      // boxes holding none of this CTA's columns are not loaded
      uint32_t bytes = 0;
      for (int bx = 0; bx < nbox; ++bx) {
        const int chi = 4 * Q + bx * p.gpair;
        if (chi + p.gpair > col0 && chi < col1) bytes += static_cast<uint32_t>(box_bytes);
      }
      mbar_arrive_expect_tx(bar_quad + 8 * qq, bytes);
      for (int bx = 0; bx < nbox; ++bx) {
        const int chi = 4 * Q + bx * p.gpair;
        if (!(chi + p.gpair > col0 && chi < col1)) continue;
        const int rb = chi / p.ng;
        const int gi = chi - rb * p.ng;
        const int y0 = p.epilogue == CQ_EPI_SWIGLU ? rb * 8 : rb * 16;
        tma_load_4d(codes0 + qq * quad_bytes + bx * box_bytes, wmap, 0, y0, 0, gi,
                    bar_quad + 8 * qq);
      }
    }
    GV_STAMP(3);
  }
  if (warp == kGvTmaWarp) __syncwarp();
  // level tables: one (quad, item, lane) table per thread and round; columns
  // of other CTAs' row blocks get zero tables
  for (int id = tid; warp < kGvCompute && id < n_quads * 64; id += kGvCompute * 32) {
    const int qq = id >> 6, it = (id >> 5) & 1, ln = id & 31;
    const int g = ln >> 2, c = ln & 3;
    const int chi = 4 * (q_first + qq) + c;
    bool valid = chi >= col0 && chi < col1;
    float s = 0.f;
    uint32_t abw = 0u;
    if (valid) {
      const int rb = chi / p.ng;
      const int gi = chi - rb * p.ng;
      const int row = gv_row(p.N, p.epilogue, rb, it, g);
      valid = row < p.N;
      if (valid) {
        const int64_t mi = static_cast<int64_t>(row) * p.ng + gi;
        s = __ldg(w.scales + mi);
        abw = __ldg(w.ab + mi);
      }
    }
    uint32_t L[1 << B];
    gv_levels<B>(valid, s, abw, p.mode, L);
    uint32_t* const tb = tblw + (qq * C::SET_BYTES) / 4 + it * (E * 32) + ln;
    if constexpr (B == 4) {
#pragma unroll
      for (int e = 0; e < 16; ++e) tb[e * 32] = L[e] | (L[e] << 16);
    } else {
      constexpr int NL = 1 << B;
#pragma unroll
      for (int e = 0; e < E; ++e) tb[e * 32] = L[e & (NL - 1)] | (L[e / NL] << 16);
    }
  }
  if (warp < kGvCompute) asm volatile("bar.sync 1, %0;" ::"n"(kGvCompute * 32) : "memory");
  if (tid == 0) GV_STAMP(4);

  // ------------------------------------------------------------------ phase C
  if (warp < kGvCompute) {
    const int g = lane >> 2, c = lane & 3;
    const bool x_role = MT == 1 ? (g == c) : ((g >> 1) == c);
    const int xm = MT == 1 ? 0 : (g & 1);
    // 16-byte chunk order of the code reads (keeps them conflict free)
    const int rot = B == 2 ? (g & 1) : (B == 4 ? 2 * (c >> 1) + (g & 1) : 0);
    bool ok = gv_wait_warp(bar_x, 0, flags, tmo, SITE_GV_X);
    for (int k = warp; ok && k < n_loc; k += kGvCompute) {
      const int qq = gv_div_spc(p, k);
      const int Q = q_first + qq;
      const int sstep = k - qq * p.spc;
      if (!gv_wait_warp(bar_quad + 8 * qq, 0, flags, tmo, SITE_GV_STAGE_FULL)) break;
      const int chi = 4 * Q + c;
      const bool cv = chi >= col0 && chi < col1;
      int sc = sstep + c;
      while (sc >= p.spc) sc -= p.spc;
      const int gi = cv ? chi - (chi / p.ng) * p.ng : 0;
      // the lane's two rows of slice sc of column c (stale data for columns
      // of other CTAs: their tables are zero)
      const uint32_t cb = codes0 + qq * quad_bytes + c * 16 * RG + g * RG + sc * C::SLICE_BYTES;
      uint32_t c0[4 * B], c1[4 * B];
#pragma unroll
      for (int v = 0; v < B; ++v) {
        int vv = v + rot;
        while (vv >= B) vv -= B;
        const uint4 q0 = lds128(cb + 16 * vv);
        const uint4 q1 = lds128(cb + 8 * RG + 16 * vv);
#pragma unroll
        for (int w = 0; w < B; ++w)
          if (w == vv) {
            c0[4 * w + 0] = q0.x;
            c0[4 * w + 1] = q0.y;
            c0[4 * w + 2] = q0.z;
            c0[4 * w + 3] = q0.w;
            c1[4 * w + 0] = q1.x;
            c1[4 * w + 1] = q1.y;
            c1[4 * w + 2] = q1.z;
            c1[4 * w + 3] = q1.w;
          }
      }
      const uint32_t tl0 = tbl0 + qq * C::SET_BYTES + lane * 4;
      const uint32_t tl1 = tl0 + E * 128;
      const bool xh = x_role && cv && xm < w.M;
      const uint32_t xa = xs + (static_cast<uint32_t>(xm) * p.K + gi * p.G + sc * 128) * 2u;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        // activations of this 32-code piece (zero for lanes without a role)
        uint32_t xv[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 q = make_uint4(0u, 0u, 0u, 0u);
          if (xh) q = lds128(xa + pc * 64 + 16 * v);
          xv[4 * v + 0] = q.x;
          xv[4 * v + 1] = q.y;
          xv[4 * v + 2] = q.z;
          xv[4 * v + 3] = q.w;
        }
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int q = 16 * pc + 2 * s;      // pair index within the slice
          const uint32_t a0 = gv_pair<B>(c0, q, tl0);
          const uint32_t a1 = gv_pair<B>(c1, q, tl1);
          const uint32_t a2 = gv_pair<B>(c0, q + 1, tl0);
          const uint32_t a3 = gv_pair<B>(c1, q + 1, tl1);
          mma_16816_bf16(acc[s & 3], a0, a1, a2, a3, xv[2 * s], xv[2 * s + 1]);
        }
      }
      float d[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) d[b] = ((acc[0][b] + acc[1][b]) + acc[2][b]) + acc[3][b];
      float* const sl = slot_f + k * C::NV;
      if (MT == 1) {
        if (c < 2) {
          sl[((2 * c) * 2 + 0) * 8 + g] = d[0];
          sl[((2 * c + 1) * 2 + 0) * 8 + g] = d[1];
          sl[((2 * c) * 2 + 1) * 8 + g] = d[2];
          sl[((2 * c + 1) * 2 + 1) * 8 + g] = d[3];
        }
      } else {
        sl[((c * 2 + 0) * 8 + g) * 2 + 0] = d[0];
        sl[((c * 2 + 0) * 8 + g) * 2 + 1] = d[1];
        sl[((c * 2 + 1) * 8 + g) * 2 + 0] = d[2];
        sl[((c * 2 + 1) * 8 + g) * 2 + 1] = d[3];
      }
    }
  }
  __syncthreads();
  if (tid == 0) GV_STAMP(5);
  if (flags[0]) {
    // a wait gave up: no copy may still be landing in shared memory at exit
    if (tid == 0) {
      volatile int dummy = 0;
      mbar_wait(bar_x, 0, &dummy, tmo, SITE_TEARDOWN);
      for (int qq = 0; qq < n_quads; ++qq) mbar_wait(bar_quad + 8 * qq, 0, &dummy, tmo, SITE_TEARDOWN);
    }
    __syncthreads();
    return;
  }

  // ------------------------------------------------------------------ phase D
  // out_f[rbl][r][m]: row slot r = 8 * item + g of row block rb_first + rbl
  // four lanes per output, whole warps at a time (the shuffles need them)
  const int n_out = n_rbl * 16 * MT;
  for (int base4 = warp * 32; base4 < n_out * 4; base4 += kGvThreads) {
    const int o4 = base4 + lane;
    const int o = o4 >> 2;
    float v = 0.f;
    if (o < n_out) {
      const int m = o % MT;
      const int r = (o / MT) & 15;
      const int rb = rb_first + o / (16 * MT);
      v = gv_rb_sum_part<C::NV, MT>(p, slots, rb, r * MT + m, q_first, o4 & 3);
    }
    v += __shfl_xor_sync(0xffffffffu, v, 1);     // (part 0 + part 1), (part 2 + part 3)
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    if (o < n_out && (o4 & 3) == 0) out_f[o] = v;
  }
  __syncthreads();
  if (tid == 0) GV_STAMP(6);
  if (p.epilogue == CQ_EPI_SWIGLU) {
    for (int o = tid; o < n_rbl * 8 * MT; o += kGvThreads) {
      const int m = o % MT;
      const int g = (o / MT) & 7;
      const int rbl = o / (8 * MT);
      const int rb = rb_first + rbl;
      if (m >= w.M) continue;
      const float gate = out_f[(rbl * 16 + g) * MT + m];
      const float up = out_f[(rbl * 16 + 8 + g) * MT + m];
      const float h = gv_silu(gate) * up;
      const int64_t off = w.y_off[m] + rb * 8 + g;
      if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(h);
      else
        reinterpret_cast<float*>(p.y)[off] = h;
    }
  } else {
    for (int o = tid; o < n_out; o += kGvThreads) {
      const int m = o % MT;
      const int r = (o / MT) & 15;
      const int rb = rb_first + o / (16 * MT);
      const int row = rb * 16 + r;
      if (m >= w.M || row >= p.N) continue;
      const int64_t off = w.y_off[m] + row;
      if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(out_f[o]);
      else
        reinterpret_cast<float*>(p.y)[off] = out_f[o];
    }
  }
  if (tid == 0) GV_STAMP(1);
}

// cq_gemm's decode-sized path: CTA c owns row blocks [c * rpc, (c+1) * rpc).
template <int B, int MT>
__global__ void __launch_bounds__(kGvThreads, 1)
    gemv_kernel(const __grid_constant__ GemvParams p, const __grid_constant__ CUtensorMap wmap) {
  GvCta w;
  w.rb_first = blockIdx.x * p.rpc;
  w.n_rbl = min(p.rpc, p.n_rb - w.rb_first);
  w.M = p.M;
  w.x = p.x;
  w.scales = p.scales;
  w.ab = p.ab;
  w.y_off[0] = 0;
  w.y_off[1] = p.ldy;
  gemv_cta<B, MT>(p, &wmap, w, p.max_quads, false);
}

// ---------------------------------------------------------------------------
// Grouped (MoE) form: the decode-sized products of one MoE stage, one work
// item per (expert, chunk of at most MT routed tokens, range of row blocks).
// Items are ordered by bit width (all B = 2, then 3, then 4) so that items of
// one width are uniform; a persistent CTA walks items item, item + grid, ...
// ---------------------------------------------------------------------------
struct GvMatrix {        // one expert matrix (device pointers)
  const uint8_t* packed;
  const float* scales;
  const uint32_t* ab;
  int B;
  int reserved;
};

struct alignas(64) GvExpert {   // what the grouped kernel needs of one expert and stage
  CUtensorMap map;               // the 4-D GEMV tensor map of the matrix
  GvMatrix mat;
};

struct MoeGvParams {
  GemvParams base;             // shape of the stage's matrices (x, scales, ab, y unused)
  int rpc[3];                  // row blocks per item, B = 2, 3, 4
  int max_quads[3];
  int ipi[3];                  // items per chunk: ceil(n_rb / rpc)
  const GvExpert* experts;     // [E] (64-byte aligned)
  int E;
  const int* n_chunks;         // [3] chunks of width B (device, written by the router)
  const int* chunk_e;          // [chunks] expert of each chunk, ordered by width
  const int* chunk_pos;        // [chunks] sorted position of its first route
  const int* chunk_m;          // [chunks] routes in the chunk (1..MT)
  const uint16_t* xs;          // [R][K] bf16 activations in sorted order
  void* y;                     // output rows
  const int* out_rows;         // sorted position -> output row, or null (identity)
  int64_t y_rows;              // rows of y
  int64_t R;                   // routes (rows of xs)
};

// Resolve work item `item` of a grouped stage: width, chunk and row blocks.
struct GvItem {
  int bi, ck, part;
};
__device__ __forceinline__ bool gv_item(const MoeGvParams& q, int item, int n2, int n3, int s3,
                                        int s4, int total, GvItem& it) {
  if (item >= total) return false;
  int local, chunk0;
  if (item < s3) {
    it.bi = 0; local = item; chunk0 = 0;
  } else if (item < s4) {
    it.bi = 1; local = item - s3; chunk0 = n2;
  } else {
    it.bi = 2; local = item - s4; chunk0 = n2 + n3;
  }
  it.ck = chunk0 + local / q.ipi[it.bi];
  it.part = local % q.ipi[it.bi];
  return true;
}

template <int MT>
__global__ void __launch_bounds__(kGvThreads, 1) moe_gemv_kernel(const __grid_constant__ MoeGvParams q) {
  if (!q.base.y || !q.xs) {
    if (threadIdx.x == 0) atomicCAS(&g_device_error, 0, 38);
    return;
  }
  const int n2 = ld_guarded(q.n_chunks + 0), n3 = ld_guarded(q.n_chunks + 1),
            n4 = ld_guarded(q.n_chunks + 2);
  const int s3 = n2 * q.ipi[0];
  const int s4 = s3 + n3 * q.ipi[1];
  const int total = s4 + n4 * q.ipi[2];
  bool reuse = false;
  GvItem cur;
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    gv_item(q, item, n2, n3, s3, s4, total, cur);
    const int bi = cur.bi, ck = cur.ck, part = cur.part;
    const int e = ld_guarded(q.chunk_e + ck);
    const int pos = ld_guarded(q.chunk_pos + ck);
    const int M = ld_guarded(q.chunk_m + ck);
    if (e < 0 || e >= q.E || pos < 0 || M < 1 || M > MT || pos + M > q.R) {
      if (threadIdx.x == 0) atomicCAS(&g_device_error, 0, 36);
      continue;
    }
    const GvExpert* ex = q.experts + e;
    GvCta w;
    w.rb_first = part * q.rpc[bi];
    w.n_rbl = min(q.rpc[bi], q.base.n_rb - w.rb_first);
    w.M = M;
    w.x = q.xs + static_cast<int64_t>(pos) * q.base.K;
    w.scales = ex->mat.scales;
    w.ab = ex->mat.ab;
    bool rows_ok = true;
    for (int m = 0; m < 2; ++m) {
      const int pm = pos + (m < M ? m : 0);
      const int64_t row = q.out_rows ? static_cast<int64_t>(ld_guarded(q.out_rows + pm)) : pm;
      if (row < 0 || row >= q.y_rows) rows_ok = false;
      w.y_off[m] = row * q.base.ldy;
    }
    if (!rows_ok || ex->mat.B != bi + 2) {
      if (threadIdx.x == 0) atomicCAS(&g_device_error, 0, 37);
      continue;
    }
    if (bi == 0)
      gemv_cta<2, MT>(q.base, &ex->map, w, q.max_quads[0], reuse);
    else if (bi == 1)
      gemv_cta<3, MT>(q.base, &ex->map, w, q.max_quads[1], reuse);
    else
      gemv_cta<4, MT>(q.base, &ex->map, w, q.max_quads[2], reuse);
    reuse = true;
    __syncthreads();
  }
}

}  // namespace cq
