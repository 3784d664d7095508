// cq_a8.cuh -- Dynamic-A8 CubicQuant GEMM for sm_100a (the article's second
// execution mode, section "一份 checkpoint，同时服务 A16 与 Dynamic A8"):
// activations quantized per row to INT8, weight codes decoded to their INT8
// carriers inside the tile, integer dot products on the tensor cores
// (tcgen05.mma kind::i8, INT32 accumulators in TMEM) drained once per group
// through the FP32 group scale.
//
//   xq[m][k]   = RNE(x[m][k] * RN(127 / absmax[m])), saturated to +-127
//   carrier(u) = RNE(127 sign(k) q(t)), saturated to +-127
//   y[m][n]    = (absmax[m] / 127^2) * sum_g s[n][g] * sum_{k in g} xq[m][k] carrier(u[n][k])
//
// The engine is the A16 engine's structure (persistent CTAs, stream-K over
// (tile, slice), decoder / producer / MMA / epilogue warps) with three
// differences: a decoded slice is 128 INT8 carriers per row (32 TMEM
// columns), the MMA is kind::i8 with K = 32 per instruction, and the
// accumulator is handed to the epilogue at every group boundary, where it
// is scaled by the row's s and added to FP32 running sums kept in TMEM.
#pragma once

#include "cq_engine.cuh"

namespace cq {

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::i8 (S8 inputs, S32 accumulate).
__device__ __forceinline__ void mma_ts_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor: kind::i8, A = B = S8, D = S32, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
  return (2u << 4)                                   // D format S32
         | (1u << 7)                                 // A format S8
         | (1u << 10)                                // B format S8
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Store 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
      "%10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// INT8 carrier of code u: q(t) = a t + b t^2 + c t^3 term by term with
// c = (1 - a) - b, times 127 sign(k), rounded to the nearest integer (ties
// to even) and saturated.  The operation order is that of the definition,
// so the integer decision is the same as any other FP64 evaluation of it in
// that order.
__device__ __forceinline__ int carrier_i8(int u, int B, int mode, double a, double b) {
  int sg;
  double t;
  coord(u, B, mode, sg, t);
  const double c = __dsub_rn(__dsub_rn(1.0, a), b);
  const double at = __dmul_rn(a, t);
  const double bt2 = __dmul_rn(__dmul_rn(b, t), t);
  const double ct3 = __dmul_rn(__dmul_rn(__dmul_rn(c, t), t), t);
  const double q = __dadd_rn(__dadd_rn(at, bt2), ct3);
  double v = rint(__dmul_rn(127.0 * static_cast<double>(sg), q));
  v = v > 127.0 ? 127.0 : (v < -127.0 ? -127.0 : v);
  return static_cast<int>(v);
}

// Carrier tables, laid out like the A16 pair tables (entry e of tile row i
// is the 32-bit word at tbl + e*128 + i):
//   B=2: e = u0 | u1<<2 -> C[u0] | C[u1] << 8
//   B=3: e = u0 | u1<<3 -> C[u0] | C[u1] << 8
//   B=4: e = u          -> C[u]
// with C the carrier bytes.  The carrier is odd in k, so the positive side
// is evaluated and mirrored (round-to-nearest-even is symmetric).
template <int B>
__device__ __forceinline__ void build_table_a8(uint32_t* tbl, int i, bool valid, uint32_t abw,
                                               int mode) {
  constexpr int NC = 1 << B;
  constexpr int H = NC / 2;
  uint32_t C[NC];
#pragma unroll
  for (int u = 0; u < NC; ++u) C[u] = 0u;
  if (valid) {
    const double a = static_cast<double>(__half2float(__ushort_as_half(abw & 0xFFFFu)));
    const double b = static_cast<double>(__half2float(__ushort_as_half(abw >> 16)));
    if (mode == CQ_GRID_MIDRISE) {
#pragma unroll
      for (int j = 0; j < H; ++j) {
        const int c = carrier_i8(H + j, B, 0, a, b);
        C[H + j] = static_cast<uint32_t>(c) & 0xFFu;
        C[H - 1 - j] = static_cast<uint32_t>(-c) & 0xFFu;
      }
    } else {
#pragma unroll
      for (int m = 0; m <= H; ++m) {
        const int c = carrier_i8(H - 1 + m, B, 1, a, b);
        C[H - 1 + m] = static_cast<uint32_t>(c) & 0xFFu;
        if (m >= 1 && m <= H - 1) C[H - 1 - m] = static_cast<uint32_t>(-c) & 0xFFu;
      }
    }
  }
  if constexpr (B == 2) {
#pragma unroll
    for (int e = 0; e < 16; ++e) tbl[e * kRows + i] = C[e & 3] | (C[e >> 2] << 8);
  } else if constexpr (B == 3) {
#pragma unroll
    for (int e = 0; e < 64; ++e) tbl[e * kRows + i] = C[e & 7] | (C[e >> 3] << 8);
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) tbl[e * kRows + i] = C[e];
  }
}

// One 128-code slice of tile row i -> 32 words of four INT8 carriers each
// (word w holds codes 4w .. 4w+3, lowest code in the lowest byte).
template <int B>
__device__ __forceinline__ void decode_slice_a8(const uint4* codes, uint32_t swz,
                                                const uint32_t* tbl, uint32_t i,
                                                uint32_t (&r)[32]) {
  uint32_t c[4 * B];
#pragma unroll
  for (int v = 0; v < B; ++v) {
    const uint4 q = codes[v ^ swz];
    c[4 * v + 0] = q.x;
    c[4 * v + 1] = q.y;
    c[4 * v + 2] = q.z;
    c[4 * v + 3] = q.w;
  }
#pragma unroll
  for (int w = 0; w < 32; ++w) {
    if constexpr (B == 2) {
      const int p0 = 2 * w, p1 = 2 * w + 1;
      const uint32_t lo = tbl[(at_bit7(c[p0 >> 3], 4 * (p0 & 7)) & (15u << 7)) | i];
      const uint32_t hi = tbl[(at_bit7(c[p1 >> 3], 4 * (p1 & 7)) & (15u << 7)) | i];
      r[w] = __byte_perm(lo, hi, 0x5410);
    } else if constexpr (B == 3) {
      uint32_t pr[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int o = 6 * (2 * w + h);
        const int wi = o >> 5, sh = o & 31;
        uint32_t v;
        if (sh <= 26)
          v = at_bit7(c[wi], sh);
        else
          v = __funnelshift_r(c[wi], c[wi + 1 < 4 * B ? wi + 1 : 4 * B - 1], sh - 7);
        pr[h] = tbl[(v & (63u << 7)) | i];
      }
      r[w] = __byte_perm(pr[0], pr[1], 0x5410);
    } else {
      uint32_t l[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int n = 4 * w + h;
        l[h] = tbl[(at_bit7(c[n >> 3], 4 * (n & 7)) & (15u << 7)) | i];
      }
      r[w] = __byte_perm(__byte_perm(l[0], l[1], 0x0040), __byte_perm(l[2], l[3], 0x0040),
                         0x5410);
    }
  }
}

// Dynamic per-row INT8 quantization: one CTA per row.
constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads)
    quant_rows_kernel(const uint16_t* __restrict__ x, int M, int K, int8_t* __restrict__ xq,
                      float* __restrict__ absmax) {
  __shared__ float red[kQuantThreads / 32];
  const int row = blockIdx.x;
  if (row >= M) return;
  const uint16_t* xr = x + static_cast<int64_t>(row) * K;
  int8_t* qr = xq + static_cast<int64_t>(row) * K;
  float mx = 0.f;
  for (int k = threadIdx.x; k < K; k += kQuantThreads)
    mx = fmaxf(mx, fabsf(__uint_as_float(static_cast<uint32_t>(xr[k]) << 16)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) mx = fmaxf(mx, red[w]);
  const float inv = mx > 0.f ? __fdiv_rn(127.0f, mx) : 0.f;
  for (int k = threadIdx.x; k < K; k += kQuantThreads) {
    const float v = __uint_as_float(static_cast<uint32_t>(xr[k]) << 16);
    float r = rintf(__fmul_rn(v, inv));
    r = r > 127.f ? 127.f : (r < -127.f ? -127.f : r);
    qr[k] = static_cast<int8_t>(static_cast<int>(r));
  }
  if (threadIdx.x == 0) absmax[row] = mx;
}

// Shapes of the A8 engine: decoded slices of 32 TMEM columns, two INT32
// accumulators and one buffer of FP32 running sums of NT columns each.
template <int NT, int TE>
struct A8Cfg {
  static constexpr int SPS = NT <= 32 ? 4 : (NT == 64 ? 2 : 1);   // slices per stage
  static constexpr int SCOL = 32;                                  // TMEM columns per slice
  static constexpr int FREE = (kTmemCols - 3 * NT) / SCOL;
  static constexpr int RING = FREE >= kTmemRing ? kTmemRing : FREE;
  static constexpr int DCOL = RING * SCOL;                         // accumulators
  static constexpr int RCOL = DCOL + 2 * NT;                       // running sums
  static constexpr int SLICE_W_BYTES = kRows * 16 * 4;
  static constexpr int W_STAGE = SPS * SLICE_W_BYTES;
  static constexpr int X_STAGE = 128 * SPS * NT;                   // SPS boxes of NT x 128 int8
  static constexpr int XCHG_BYTES = 16 * 64 * 4;
  static constexpr int MISC_BYTES = 1024;
  static constexpr int TBL_BYTES = 2 * TE * kRows * 4;
  static constexpr int BUDGET = 226 * 1024;
  static constexpr int AVAIL = BUDGET - 1024 - TBL_BYTES - XCHG_BYTES - MISC_BYTES;
  static constexpr int SX_RAW = (AVAIL - 2 * W_STAGE) / X_STAGE;
  static constexpr int SX = SX_RAW > 4 ? 4 : SX_RAW;
  static constexpr int SW_RAW = (AVAIL - SX * X_STAGE) / W_STAGE;
  static constexpr int SW = SW_RAW > 8 ? 8 : SW_RAW;
  static constexpr int SMEM =
      1024 + SX * X_STAGE + SW * W_STAGE + TBL_BYTES + XCHG_BYTES + MISC_BYTES;
  static_assert(NT <= 128, "the A8 engine keeps three NT-column buffers in TMEM");
  static_assert(RING >= 2, "TMEM ring too small");
  static_assert(RCOL + NT <= kTmemCols, "TMEM budget exceeded");
  static_assert(SX >= 2 && SW >= 2, "not enough shared memory for two stages per ring");
  static_assert(SMEM <= 227 * 1024, "shared memory budget exceeded");
};

struct A8Params {
  EngineParams e;          // plain mode only
  const float* absmax;     // [M] row absmax of the activations
};

template <int NT, int TE>
__global__ void __launch_bounds__(kThreads, 1)
    engine_a8_kernel(const __grid_constant__ A8Params pa,
                     const __grid_constant__ CUtensorMap xmap,
                     const __grid_constant__ CUtensorMap wmap) {
  using C = A8Cfg<NT, TE>;
  const EngineParams& p = pa.e;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t xring = base;
  const uint32_t wring = xring + C::SX * C::X_STAGE;
  const uint32_t tbl_s = wring + C::SW * C::W_STAGE;
  const uint32_t xchg_s = tbl_s + C::TBL_BYTES;
  const uint32_t misc = xchg_s + C::XCHG_BYTES;
  uint8_t* const gbase = smem_raw + (base - raw);
  float* const xchg = reinterpret_cast<float*>(gbase + (xchg_s - base));
  uint32_t* const tbl = reinterpret_cast<uint32_t*>(gbase + (tbl_s - base));
  const uint32_t bar_wfull = misc;
  const uint32_t bar_wfree = bar_wfull + 8 * C::SW;
  const uint32_t bar_xfull = bar_wfree + 8 * C::SW;
  const uint32_t bar_xfree = bar_xfull + 8 * C::SX;
  const uint32_t bar_aready = bar_xfree + 8 * C::SX;      // [4]
  const uint32_t bar_tfree = bar_aready + 8 * kTmemRing;  // [4]
  const uint32_t bar_dfull = bar_tfree + 8 * kTmemRing;   // [2]
  const uint32_t bar_dfree = bar_dfull + 16;              // [2]
  const uint32_t bar_fin = bar_dfree + 16;
  const uint32_t slot_tmem = bar_fin + 8;
  volatile int* const abort_flag =
      reinterpret_cast<volatile int*>(gbase + (slot_tmem + 8 - base));
  volatile int* const last_flag =
      reinterpret_cast<volatile int*>(gbase + (slot_tmem + 12 - base));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int cta = blockIdx.x;

  if (tid == 0) {
    griddep_launch_dependents();
    for (int s = 0; s < C::SW; ++s) {
      mbar_init(bar_wfull + 8 * s, 1);
      mbar_init(bar_wfree + 8 * s, kDecoders);
    }
    for (int s = 0; s < C::SX; ++s) {
      mbar_init(bar_xfull + 8 * s, 1);
      mbar_init(bar_xfree + 8 * s, 1);
    }
    for (int s = 0; s < kTmemRing; ++s) {
      mbar_init(bar_aready + 8 * s, kRows);
      mbar_init(bar_tfree + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_dfull + 8 * s, 1);
      mbar_init(bar_dfree + 8 * s, kEpilogue);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(slot_tmem, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&xmap);
    prefetch_tensormap(&wmap);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base =
      *reinterpret_cast<volatile uint32_t*>(gbase + (slot_tmem - base));
  griddep_wait();

  const int num_tiles = p.num_tiles;
  const int64_t W = static_cast<int64_t>(num_tiles) * p.spt;
  const int Pe = W < p.P ? static_cast<int>(W) : p.P;
  const int64_t r0 = cta < Pe ? range_begin(W, Pe, cta) : W;
  const int64_t r1 = cta < Pe ? range_begin(W, Pe, cta + 1) : W;
  const uint64_t tmo = p.timeout_ns;
  const int ng = p.K / p.G;
  const int spc = p.G / kSlice;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane < 2) {
      const bool wl = lane == 0;
      const int NS = wl ? C::SW : C::SX;
      const uint32_t full0 = wl ? bar_wfull : bar_xfull;
      const uint32_t free0 = wl ? bar_wfree : bar_xfree;
      int st = 0;
      uint32_t round = 0;
      int load_no = 0;
      bool ok = true;
      for (int64_t x = r0; ok && x < r1 && !*abort_flag;) {
        const Segment sg = segment_at(x, r1, p.spt);
        const TileInfo ti = resolve_tile(p, sg.t, NT, 2, 4);
        const int Bw = ti.mat.B;
        const int row_a = tile_row(p, ti.rt, 0);
        const int row_b = tile_row(p, ti.rt, 64);
        for (int sb = sg.s0; ok && sb < sg.s1; sb += C::SPS) {
          const int ns = (sg.s1 - sb) < C::SPS ? (sg.s1 - sb) : C::SPS;
          if (!wait_phase(free0 + 8 * st, (round & 1u) ^ 1u, abort_flag, tmo,
                          SITE_PRODUCER_EMPTY)) {
            ok = false;
            break;
          }
          if (wl) {
            const uint32_t wbox = 64u * 16u * Bw;
            const uint32_t wdst = wring + st * C::W_STAGE;
            mbar_arrive_expect_tx(bar_wfull + 8 * st, static_cast<uint32_t>(ns) * 2u * wbox);
            for (int j = 0; j < ns; ++j) {
              const int cb = (sb + j) * 16 * Bw;
              const uint32_t sdst = wdst + j * C::SLICE_W_BYTES;
              tma_load_2d(sdst, &wmap, cb, row_a, bar_wfull + 8 * st);
              tma_load_2d(sdst + wbox, &wmap, cb, row_b, bar_wfull + 8 * st);
            }
          } else {
            const uint32_t xdst = xring + st * C::X_STAGE;
            mbar_arrive_expect_tx(bar_xfull + 8 * st, static_cast<uint32_t>(ns * NT * 128));
            for (int j = 0; j < ns; ++j)
              tma_load_2d(xdst + j * (NT * 128), &xmap, (sb + j) * kSlice, ti.x_row0,
                          bar_xfull + 8 * st);
          }
          ++load_no;
          if (++st == NS) {
            st = 0;
            ++round;
          }
        }
        if (ok) x = sg.end;
      }
      if (*abort_flag) {
        const int armed = load_no < NS ? load_no : NS;
        for (int k = 1; k <= armed; ++k) {
          const int idx = load_no - k;
          const int sl = idx % NS;
          const uint32_t rd = static_cast<uint32_t>(idx / NS);
          volatile int dummy = 0;
          mbar_wait(full0 + 8 * sl, rd & 1u, &dummy, tmo, SITE_TEARDOWN);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The INT32 accumulator is handed to the epilogue at the end of every
    // group (or segment end), so buffers alternate per drain.
    if (lane == 0) {
      const uint32_t idesc = idesc_s8_s32(kRows, NT);
      int st = 0, ts = 0;
      uint32_t round = 0, tround = 0, dcount = 0;
      bool ok = true;
      for (int64_t x = r0; ok && x < r1;) {
        const Segment sg = segment_at(x, r1, p.spt);
        uint32_t acc = 0, db = 0, d_tmem = 0;
        for (int sb = sg.s0; sb < sg.s1 && ok; sb += C::SPS) {
          const int ns = (sg.s1 - sb) < C::SPS ? (sg.s1 - sb) : C::SPS;
          if (!wait_phase(bar_xfull + 8 * st, round & 1u, abort_flag, tmo, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t desc0 = smem_desc_sw128(xring + st * C::X_STAGE);
          for (int j = 0; j < ns; ++j) {
            const int s = sb + j;
            const bool first = s == sg.s0 || s % spc == 0;
            const bool last = s == sg.s1 - 1 || (s + 1) % spc == 0;
            if (first) {
              db = dcount & 1u;
              const uint32_t duse = dcount >> 1;
              if (!wait_phase(bar_dfree + 8 * db, (duse & 1u) ^ 1u, abort_flag, tmo,
                              SITE_MMA_DFREE)) {
                ok = false;
                break;
              }
              tc_fence_after();
              d_tmem = tmem_base + C::DCOL + db * NT;
              acc = 0;
            }
            if (!wait_phase(bar_aready + 8 * ts, tround & 1u, abort_flag, tmo,
                            SITE_MMA_AREADY)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = tmem_base + ts * C::SCOL;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // box j of the stage, 32-byte K step inside its 128-byte rows
              const uint64_t off = static_cast<uint64_t>((j * NT * 128 + kk * 32) >> 4);
              mma_ts_i8(d_tmem, a0 + kk * 8, desc0 + off, idesc, acc);
              acc = 1;
            }
            mma_commit(bar_tfree + 8 * ts);
            if (++ts == C::RING) {
              ts = 0;
              ++tround;
            }
            if (last) {
              mma_commit(bar_dfull + 8 * db);
              ++dcount;
            }
          }
          if (!ok) break;
          mma_commit(bar_xfree + 8 * st);
          if (++st == C::SX) {
            st = 0;
            ++round;
          }
        }
        if (!ok) break;
        x = sg.end;
      }
      mma_commit(bar_fin);
      volatile int dummy = 0;
      mbar_wait(bar_fin, 0, &dummy, tmo, SITE_TEARDOWN);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ decoders
    const int q = warp & 3;
    const int h = warp >> 2;
    const int i = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t* const mytbl = tbl + h * (TE * kRows);
    int st = 0, ts = 0;
    uint32_t round = 0, tround = 0;
    bool ok = true;
    for (int64_t x = r0; ok && x < r1;) {
      const Segment sg = segment_at(x, r1, p.spt);
      const TileInfo ti = resolve_tile(p, sg.t, NT, 2, 4);
      const int Bw = ti.mat.B;
      const int grow = tile_row(p, ti.rt, i);
      const uint32_t swz = Bw == 2 ? ((i >> 2) & 1u) : (Bw == 4 ? ((i >> 1) & 3u) : 0u);
      const bool valid = grow < p.N;
      int cur_g = -1;
      for (int sb = sg.s0; sb < sg.s1 && ok; sb += C::SPS) {
        const int ns = (sg.s1 - sb) < C::SPS ? (sg.s1 - sb) : C::SPS;
        if (!wait_phase(bar_wfull + 8 * st, round & 1u, abort_flag, tmo, SITE_DECODER_FULL)) {
          ok = false;
          break;
        }
        const uint32_t wrow = wring + st * C::W_STAGE + i * 16 * Bw;
        for (int j = 0; j < ns; ++j) {
          const int sl = sb + j;
          if ((sl & 1) == h) {
            const int g = sl / spc;
            if (TE < 64 && Bw == 3) {
              if (g != cur_g && i == 0) bad_access(27);
              cur_g = g;
            }
            if (g != cur_g) {
              cur_g = g;
              uint32_t abw = 0;
              if (valid && g < ng)
                abw = __ldg(ti.mat.ab + static_cast<int64_t>(grow) * ng + g);
              else if (valid)
                bad_access(22);
              if (Bw == 2)
                build_table_a8<2>(mytbl, i, valid, abw, p.mode);
              else if (Bw == 3)
                build_table_a8<3>(mytbl, i, valid, abw, p.mode);
              else
                build_table_a8<4>(mytbl, i, valid, abw, p.mode);
            }
            if (!wait_phase(bar_tfree + 8 * ts, (tround & 1u) ^ 1u, abort_flag, tmo,
                            SITE_DECODER_TFREE)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + lane_off + ts * C::SCOL;
            const uint4* caddr =
                reinterpret_cast<const uint4*>(gbase + (wrow + j * C::SLICE_W_BYTES - base));
            uint32_t r[32];
            if (Bw == 2)
              decode_slice_a8<2>(caddr, swz, mytbl, i, r);
            else if (Bw == 3)
              decode_slice_a8<3>(caddr, swz, mytbl, i, r);
            else
              decode_slice_a8<4>(caddr, swz, mytbl, i, r);
            tmem_st32(taddr, r);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_aready + 8 * ts);
          }
          if (++ts == C::RING) {
            ts = 0;
            ++tround;
          }
        }
        if (!ok) break;
        mbar_arrive(bar_wfree + 8 * st);
        if (++st == C::SW) {
          st = 0;
          ++round;
        }
      }
      x = sg.end;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Per group drain: running[n][m] += s[n][g] * acc[n][m] (FP32, TMEM).
    // At the end of a segment: times absmax[m] / 127^2, then the output or
    // the stream-K partial, as in the A16 engine.
    const int q = warp & 3;
    const int i = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t rbase = tmem_base + lane_off + C::RCOL;
    uint32_t dcount = 0;
    bool ok = true;
    for (int64_t x = r0; ok && x < r1;) {
      const Segment sg = segment_at(x, r1, p.spt);
      const TileInfo ti = resolve_tile(p, sg.t, NT, 2, 4);
      const int grow = tile_row(p, ti.rt, i);
      const int nchunks = (ti.m_valid + 15) >> 4;
      const int g0 = sg.s0 / spc, g1 = (sg.s1 - 1) / spc;
      for (int g = g0; g <= g1; ++g) {
        const uint32_t db = dcount & 1u;
        const uint32_t duse = dcount >> 1;
        if (!wait_phase(bar_dfull + 8 * db, duse & 1u, abort_flag, tmo, SITE_DECODER_DFULL))
          ok = false;
        if (!vote_all_epilogue(ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float sgs = 0.f;
        if (grow < p.N && g < ng) sgs = __ldg(ti.mat.scales + static_cast<int64_t>(grow) * ng + g);
        const uint32_t daddr = tmem_base + lane_off + C::DCOL + db * NT;
        for (int cc = 0; cc < nchunks; ++cc) {
          uint32_t ra[16], rr[16];
          tmem_ld16(daddr + cc * 16, ra);
          if (g != g0) tmem_ld16(rbase + cc * 16, rr);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float run = g != g0 ? __uint_as_float(rr[k]) : 0.f;
            rr[k] = __float_as_uint(
                fmaf(sgs, static_cast<float>(static_cast<int32_t>(ra[k])), run));
          }
          tmem_st16(rbase + cc * 16, rr);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_dfree + 8 * db);
        ++dcount;
      }
      if (!ok) break;
      // per-token factor absmax / 127^2 of the chunk's columns
      auto load_chunk = [&](int cc, float (&v)[16]) {
        uint32_t rr[16];
        tmem_ld16(rbase + cc * 16, rr);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int m = ti.x_row0 + cc * 16 + k;
          const float f = m < p.M ? __ldg(pa.absmax + m) * (1.0f / 16129.0f) : 0.f;
          v[k] = __uint_as_float(rr[k]) * f;
        }
      };
      if (sg.s0 == 0 && sg.s1 == p.spt) {
        for (int cc = 0; cc < nchunks; ++cc) {
          float v[16];
          load_chunk(cc, v);
          finalize16(p, ti, i, grow, v, cc, xchg);
        }
      } else {
        const int first_tile = static_cast<int>(r0 / p.spt);
        const int slot = 2 * cta + (sg.t == first_tile ? 0 : 1);
        const bool slot_ok = slot < p.partial_slots && sg.t < p.counter_len;
        if (!slot_ok && i == 0) bad_access(24);
        float* const mine = p.partial + static_cast<int64_t>(slot_ok ? slot : 0) * NT * kRows;
        for (int cc = 0; cc < nchunks; ++cc) {
          float v[16];
          load_chunk(cc, v);
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (slot_ok && cc * 16 + k < ti.m_valid) mine[(cc * 16 + k) * kRows + i] = v[k];
        }
        __threadfence();
        named_bar_epilogue();
        const int c_lo = owner_of(W, Pe, static_cast<int64_t>(sg.t) * p.spt);
        const int c_hi = owner_of(W, Pe, static_cast<int64_t>(sg.t) * p.spt + p.spt - 1);
        if (i == 0) {
          const int old = slot_ok ? atomicAdd(p.counter + sg.t, 1) : -1;
          *last_flag = (old == c_hi - c_lo) ? 1 : 0;
        }
        named_bar_epilogue();
        const bool last = *last_flag != 0;
        if (last) {
          __threadfence();
          for (int cc = 0; cc < nchunks; ++cc) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = 0.f;
            for (int c = c_lo; c <= c_hi; ++c) {
              const int ft = static_cast<int>(range_begin(W, Pe, c) / p.spt);
              const int sl = 2 * c + (sg.t == ft ? 0 : 1);
              if (sl >= p.partial_slots) {
                bad_access(25);
                continue;
              }
              const float* src = p.partial + static_cast<int64_t>(sl) * NT * kRows;
#pragma unroll
              for (int k = 0; k < 16; ++k)
                if (cc * 16 + k < ti.m_valid) v[k] += __ldcg(src + (cc * 16 + k) * kRows + i);
            }
            finalize16(p, ti, i, grow, v, cc, xchg);
          }
          if (i == 0 && slot_ok) p.counter[sg.t] = 0;
        }
        named_bar_epilogue();
      }
      x = sg.end;
    }
  }

  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace cq
