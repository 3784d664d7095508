// cq_engine.cuh -- the fused CubicQuant GEMM tile engine for sm_100a.
//
// One CTA per SM, persistent.  A tile is 128 weight rows x NT tokens; the K
// dimension is cut into 128-code "slices" (one slice never crosses a group
// because G is a multiple of 128).  The launch's work is the list of
// (tile, slice) pairs, split evenly over the CTAs (stream-K); a tile whose
// slices are spread over several CTAs is finished by the last of them, which
// sums the partial tiles in CTA order (deterministic) and applies the
// epilogue.
//
// Warp roles (192 threads):
//   warps 0-3  decoders: thread i owns weight row i of the tile and TMEM
//              lane i.  Per group it builds a private BF16 pair table
//              (two codes -> two levels, one 32-bit word per entry, the
//              entries of all 128 threads interleaved so that every lookup
//              hits the thread's own bank), then turns each slice of packed
//              codes into 64 BF16x2 words written to TMEM with tcgen05.st
//              (the A operand of the MMA).  They also run the epilogue.
//   warp 4     producer: 1-D bulk copies of the packed rows and 2-D TMA
//              loads of the activation tile (128-byte swizzle) into a ring
//              of shared-memory stages.
//   warp 5     TMEM owner and MMA issuer: tcgen05.mma kind::f16 with A from
//              TMEM (decoded weights) and B from shared memory
//              (activations), FP32 accumulators in TMEM.
//
// This follows the article's fused A16 path ("压缩权重必须“边解码、边计算”"):
// packed codes + group parameters -> unpack and generate the levels inside
// the tile -> temporary model-dtype (BF16) weights -> immediate tile dot
// product with FP32 accumulation -> output dtype; the full weight matrix is
// never materialised.  The group scale s is folded into the BF16 level
// (BF16(s q) has the same relative rounding as BF16(q)).
#pragma once

#include "cq.h"
#include "cq_device.cuh"

namespace cq {

constexpr int kRows = 128;            // weight rows per tile (MMA M)
constexpr int kSlice = 128;           // codes per slice along K
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kTmemRing = 4;          // TMEM slice buffers (64 columns each)
constexpr int kDCol = 256;            // first TMEM column of the accumulator
constexpr int kDecoders = 128;

template <int NT>
struct EngineCfg {
  static constexpr int SPS = NT <= 32 ? 4 : (NT == 64 ? 2 : 1);   // slices per stage
  static constexpr int pitch(int B) {                           // smem row pitch, odd # of 16B
    return ((SPS * B) % 2 ? SPS * B : SPS * B + 1) * 16;
  }
  static constexpr int W_BYTES = ((kRows * pitch(4) + 1023) / 1024) * 1024;
  static constexpr int X_BYTES = 256 * SPS * NT;                // 2*SPS boxes of 64 x NT bf16
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  static constexpr int TBL_BYTES = 64 * 512;                    // largest pair table (W3)
  static constexpr int XCHG_BYTES = 16 * 64 * 4;
  static constexpr int MISC_BYTES = 1024;
  static constexpr int BUDGET = 224 * 1024;
  static constexpr int S_RAW = (BUDGET - 1024 - TBL_BYTES - XCHG_BYTES - MISC_BYTES) / STAGE_BYTES;
  static constexpr int S = S_RAW > 6 ? 6 : S_RAW;
  static constexpr int SMEM = 1024 + S * STAGE_BYTES + TBL_BYTES + XCHG_BYTES + MISC_BYTES;
  static_assert(S >= 2, "not enough shared memory for two stages");
  static_assert(SMEM <= 227 * 1024, "shared memory budget exceeded");
};

// One quantized matrix operand.
struct MatrixRef {
  const uint8_t* packed;
  const float* scales;
  const uint32_t* ab;     // (a | b << 16), fp16 bits
  int B;
};

struct EngineParams {
  // common shape of every tile in the launch
  int N;                 // weight rows
  int K;                 // reduction length
  int G;                 // group size
  int mode;              // grid mode
  int epilogue;          // CQ_EPI_NONE / CQ_EPI_SWIGLU
  int out_bf16;          // output dtype
  int n_rt;              // row tiles per matrix
  int spt;               // slices per tile = K / 128
  int num_tiles;         // tiles in the launch (plain mode)
  int P;                 // CTAs
  // plain GEMM
  MatrixRef mat;
  int M;                 // tokens
  int n_tt;              // token tiles
  void* y;
  int64_t ldy;           // row stride of y in elements
  // workspace
  float* partial;        // [2P][NT][128]
  int* counter;          // [num_tiles]
  // control
  uint64_t timeout_ns;
  int debug_skip_first_stage;   // test hook: never issue stage load 0
};

struct TileInfo {
  MatrixRef mat;
  int rt, tt;
  int x_row0;       // first activation row of the token tile (tensor map row)
  int m_valid;      // valid tokens in this tile (<= NT)
};

__device__ __forceinline__ TileInfo resolve_tile(const EngineParams& p, int t, int NT) {
  TileInfo ti;
  ti.mat = p.mat;
  ti.rt = t / p.n_tt;
  ti.tt = t - ti.rt * p.n_tt;
  ti.x_row0 = ti.tt * NT;
  const int rem = p.M - ti.x_row0;
  ti.m_valid = rem < NT ? rem : NT;
  return ti;
}

// Global weight row of tile row i.
__device__ __forceinline__ int tile_row(const EngineParams& p, int rt, int i) {
  if (p.epilogue == CQ_EPI_SWIGLU)
    return i < 64 ? rt * 64 + i : (p.N >> 1) + rt * 64 + (i - 64);
  return rt * kRows + i;
}

// Stream-K partition: CTA c owns linear slices [r(c), r(c+1)).
__device__ __forceinline__ int64_t range_begin(int64_t W, int P, int c) {
  return (static_cast<int64_t>(c) * W) / P;
}
// CTA that owns linear slice x.
__device__ __forceinline__ int owner_of(int64_t W, int P, int64_t x) {
  return static_cast<int>(((x + 1) * P - 1) / W);
}

// ---------------------------------------------------------------------------
// decoder helpers
// ---------------------------------------------------------------------------

// Build this thread's pair table for one group: 2^B levels
// L_u = BF16(FP32(s sign q(t_u))) and the entries
//   B=2: e = u0 | u1<<2 (16 entries)  ->  L[u0] | L[u1] << 16
//   B=3: e = u0 | u1<<3 (64 entries)  ->  L[u0] | L[u1] << 16
//   B=4: e = u        (16 entries)   ->  L[u]  | L[u]  << 16
// Entry e of thread i lives at tbl + e*512 + 4*i.
template <int B>
__device__ __forceinline__ void build_table(uint32_t tbase, bool valid, float s, uint32_t abw,
                                            int mode) {
  uint32_t L[1 << B];
  if (valid) {
    const double a = static_cast<double>(__half2float(__ushort_as_half(abw & 0xFFFFu)));
    const double b = static_cast<double>(__half2float(__ushort_as_half(abw >> 16)));
#pragma unroll
    for (int u = 0; u < (1 << B); ++u)
      L[u] = bf16_bits(static_cast<float>(level_f64(u, B, mode, s, a, b)));
  } else {
#pragma unroll
    for (int u = 0; u < (1 << B); ++u) L[u] = 0u;
  }
  if constexpr (B == 2) {
#pragma unroll
    for (int e = 0; e < 16; ++e) sts32(tbase + e * 512, L[e & 3] | (L[e >> 2] << 16));
  } else if constexpr (B == 3) {
#pragma unroll
    for (int e = 0; e < 64; ++e) sts32(tbase + e * 512, L[e & 7] | (L[e >> 3] << 16));
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) sts32(tbase + e * 512, L[e] | (L[e] << 16));
  }
}

// Decode pairs [P0, P0+32) of one 128-code slice (codes in c[]) into r[].
template <int B, int P0>
__device__ __forceinline__ void decode_half(const uint32_t (&c)[4 * B], uint32_t tbase,
                                            uint32_t (&r)[32]) {
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int p = P0 + q;
    if constexpr (B == 2) {
      const uint32_t idx = (c[p >> 3] >> (4 * (p & 7))) & 15u;
      r[q] = lds32(tbase + (idx << 9));
    } else if constexpr (B == 3) {
      const int o = 6 * p;
      const int wi = o >> 5, sh = o & 31;
      uint32_t v;
      if (sh <= 26)
        v = c[wi] >> sh;
      else
        v = __funnelshift_r(c[wi], c[wi + 1 < 4 * B ? wi + 1 : 4 * B - 1], sh);
      r[q] = lds32(tbase + ((v & 63u) << 9));
    } else {
      const uint32_t byte = (c[p >> 2] >> (8 * (p & 3))) & 0xFFu;
      const uint32_t lo = lds32(tbase + ((byte & 15u) << 9));
      const uint32_t hi = lds32(tbase + ((byte >> 4) << 9));
      r[q] = __byte_perm(lo, hi, 0x7610);
    }
  }
}

template <int B>
__device__ __forceinline__ void decode_slice_to_tmem(uint32_t codes_addr, uint32_t tbase,
                                                     uint32_t taddr) {
  uint32_t c[4 * B];
#pragma unroll
  for (int v = 0; v < B; ++v) {
    const uint4 q = lds128(codes_addr + 16 * v);
    c[4 * v + 0] = q.x;
    c[4 * v + 1] = q.y;
    c[4 * v + 2] = q.z;
    c[4 * v + 3] = q.w;
  }
  uint32_t r[32];
  decode_half<B, 0>(c, tbase, r);
  tmem_st32(taddr, r);
  decode_half<B, 32>(c, tbase, r);
  tmem_st32(taddr + 32, r);
}

__device__ __forceinline__ void named_bar_decoders() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// All-decoders AND-vote at named barrier 1.  Every decoder reaches it once
// per segment, whether or not one of its waits gave up, so the named
// barriers of the epilogue are only entered when all 128 agree.
__device__ __forceinline__ bool vote_all_decoders(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(ok))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

// Store 16 accumulator columns (tokens m0..m0+15) of tile row i.
__device__ __forceinline__ void finalize16(const EngineParams& p, const TileInfo& ti, int i,
                                           int grow, const float (&v)[16], int cc,
                                           float* xchg) {
  const int m0 = cc * 16;
  if (p.epilogue == CQ_EPI_SWIGLU) {
    if (i >= 64) {
#pragma unroll
      for (int q = 0; q < 16; ++q) xchg[q * 64 + (i - 64)] = v[q];
    }
    named_bar_decoders();
    if (i < 64) {
      const int col = ti.rt * 64 + i;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int m = m0 + q;
        if (m < ti.m_valid) {
          const float h = silu_f(v[q]) * xchg[q * 64 + i];
          const int64_t off = static_cast<int64_t>(ti.x_row0 + m) * p.ldy + col;
          if (p.out_bf16)
            reinterpret_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(h);
          else
            reinterpret_cast<float*>(p.y)[off] = h;
        }
      }
    }
    named_bar_decoders();
  } else {
    if (grow < p.N) {
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int m = m0 + q;
        if (m < ti.m_valid) {
          const int64_t off = static_cast<int64_t>(ti.x_row0 + m) * p.ldy + grow;
          if (p.out_bf16)
            reinterpret_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(v[q]);
          else
            reinterpret_cast<float*>(p.y)[off] = v[q];
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    engine_kernel(const __grid_constant__ EngineParams p,
                  const __grid_constant__ CUtensorMap xmap) {
  using C = EngineCfg<NT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-align the working area (swizzled TMA destinations need it)
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t stage0 = base;
  const uint32_t tbl = stage0 + C::S * C::STAGE_BYTES;
  const uint32_t xchg_s = tbl + C::TBL_BYTES;
  const uint32_t misc = xchg_s + C::XCHG_BYTES;
  uint8_t* const gbase = smem_raw + (base - raw);
  float* const xchg = reinterpret_cast<float*>(gbase + (xchg_s - base));
  // barriers and flags
  const uint32_t bar_full = misc;                         // [S]
  const uint32_t bar_wempty = bar_full + 8 * C::S;        // [S]
  const uint32_t bar_aready = bar_wempty + 8 * C::S;      // [4]
  const uint32_t bar_tfree = bar_aready + 8 * kTmemRing;  // [4]
  const uint32_t bar_dfull = bar_tfree + 8 * kTmemRing;
  const uint32_t bar_dfree = bar_dfull + 8;
  const uint32_t bar_fin = bar_dfree + 8;
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
    for (int s = 0; s < C::S; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_wempty + 8 * s, kDecoders + 1);
    }
    for (int s = 0; s < kTmemRing; ++s) {
      mbar_init(bar_aready + 8 * s, kDecoders);
      mbar_init(bar_tfree + 8 * s, 1);
    }
    mbar_init(bar_dfull, 1);
    mbar_init(bar_dfree, kDecoders);
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(slot_tmem, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 4 && lane == 0) prefetch_tensormap(&xmap);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base =
      *reinterpret_cast<volatile uint32_t*>(gbase + (slot_tmem - base));

  const int64_t W = static_cast<int64_t>(p.num_tiles) * p.spt;
  const int64_t r0 = range_begin(W, p.P, cta);
  const int64_t r1 = range_begin(W, p.P, cta + 1);
  const uint64_t tmo = p.timeout_ns;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    int st = 0;
    uint32_t round = 0;
    int load_no = 0;
    int64_t x = r0;
    while (x < r1 && !*abort_flag) {
      const int t = static_cast<int>(x / p.spt);
      const int s0 = static_cast<int>(x - static_cast<int64_t>(t) * p.spt);
      const int64_t seg_end = static_cast<int64_t>(t + 1) * p.spt < r1
                                  ? static_cast<int64_t>(t + 1) * p.spt
                                  : r1;
      const int s1 = static_cast<int>(seg_end - static_cast<int64_t>(t) * p.spt);
      const TileInfo ti = resolve_tile(p, t, NT);
      const int Bw = ti.mat.B;
      const int pitch = C::pitch(Bw);
      const int64_t row_bytes = static_cast<int64_t>(p.K) * Bw / 8;
      int valid_rows = 0;
      if (p.epilogue == CQ_EPI_SWIGLU) {
        valid_rows = kRows;
      } else {
        const int rem = p.N - ti.rt * kRows;
        valid_rows = rem < kRows ? rem : kRows;
      }
      for (int sb = s0; sb < s1; sb += C::SPS) {
        const int ns = (s1 - sb) < C::SPS ? (s1 - sb) : C::SPS;
        if (!mbar_wait(bar_wempty + 8 * st, (round & 1u) ^ 1u, abort_flag, tmo,
                       SITE_PRODUCER_EMPTY))
          break;
        const bool skip = p.debug_skip_first_stage && load_no == 0;
        if (!skip) {
          const uint32_t wb = static_cast<uint32_t>(ns * 16 * Bw);
          const uint32_t bytes =
              static_cast<uint32_t>(valid_rows) * wb + static_cast<uint32_t>(2 * ns * NT * 128);
          const uint32_t wdst = stage0 + st * C::STAGE_BYTES;
          const uint32_t xdst = wdst + C::W_BYTES;
          if (lane == 0) mbar_arrive_expect_tx(bar_full + 8 * st, bytes);
          __syncwarp();
          for (int r = lane; r < valid_rows; r += 32) {
            const int grow = tile_row(p, ti.rt, r);
            const uint8_t* src = ti.mat.packed + static_cast<int64_t>(grow) * row_bytes +
                                 static_cast<int64_t>(sb) * 16 * Bw;
            bulk_g2s(wdst + r * pitch, src, wb, bar_full + 8 * st);
          }
          if (lane == 0) {
            for (int b = 0; b < 2 * ns; ++b)
              tma_load_2d(xdst + b * (NT * 128), &xmap, sb * kSlice + b * 64, ti.x_row0,
                          bar_full + 8 * st);
          }
        }
        ++load_no;
        if (++st == C::S) {
          st = 0;
          ++round;
        }
      }
      x = seg_end;
    }
    // make sure no copy is still landing in shared memory before exit
    __syncwarp();
    if (lane == 0 && *abort_flag) {
      // the ring positions armed last are the only ones that may be in flight
      const int armed = load_no < C::S ? load_no : C::S;
      for (int k = 1; k <= armed; ++k) {
        const int idx = load_no - k;
        if (p.debug_skip_first_stage && idx == 0) continue;
        const int s = idx % C::S;
        const uint32_t rd = static_cast<uint32_t>(idx / C::S);
        volatile int dummy = 0;
        mbar_wait(bar_full + 8 * s, rd & 1u, &dummy, tmo, SITE_TEARDOWN);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kRows, NT);
      int st = 0, ts = 0;
      uint32_t round = 0, tround = 0, seg = 0;
      int64_t x = r0;
      bool ok = true;
      while (ok && x < r1) {
        const int t = static_cast<int>(x / p.spt);
        const int s0 = static_cast<int>(x - static_cast<int64_t>(t) * p.spt);
        const int64_t seg_end = static_cast<int64_t>(t + 1) * p.spt < r1
                                    ? static_cast<int64_t>(t + 1) * p.spt
                                    : r1;
        const int s1 = static_cast<int>(seg_end - static_cast<int64_t>(t) * p.spt);
        if (!mbar_wait(bar_dfree, (seg & 1u) ^ 1u, abort_flag, tmo, SITE_MMA_DFREE)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t acc = 0;
        for (int sb = s0; sb < s1 && ok; sb += C::SPS) {
          const int ns = (s1 - sb) < C::SPS ? (s1 - sb) : C::SPS;
          if (!mbar_wait(bar_full + 8 * st, round & 1u, abort_flag, tmo, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xs = stage0 + st * C::STAGE_BYTES + C::W_BYTES;
          for (int j = 0; j < ns; ++j) {
            if (!mbar_wait(bar_aready + 8 * ts, tround & 1u, abort_flag, tmo, SITE_MMA_AREADY)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const int kin = j * kSlice + kk * 16;           // k offset inside the stage
              const uint32_t baddr = xs + (kin >> 6) * (NT * 128) + (kin & 63) * 2;
              mma_ts_bf16(tmem_base + kDCol, tmem_base + ts * 64 + kk * 8,
                          smem_desc_sw128(baddr), idesc, acc);
              acc = 1;
            }
            mma_commit(bar_tfree + 8 * ts);
            if (++ts == kTmemRing) {
              ts = 0;
              ++tround;
            }
          }
          if (!ok) break;
          mma_commit(bar_wempty + 8 * st);
          if (++st == C::S) {
            st = 0;
            ++round;
          }
        }
        if (!ok) break;
        mma_commit(bar_dfull);
        ++seg;
        x = seg_end;
      }
      // all issued MMAs have completed before TMEM is released
      mma_commit(bar_fin);
      volatile int dummy = 0;
      mbar_wait(bar_fin, 0, &dummy, tmo, SITE_TEARDOWN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ decoders
    const int i = tid;                                   // tile row / TMEM lane
    const uint32_t tbase = tbl + 4u * i;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    int st = 0, ts = 0;
    uint32_t round = 0, tround = 0, seg = 0;
    int64_t x = r0;
    bool ok = true;
    const int ng = p.K / p.G;
    while (ok && x < r1) {
      const int t = static_cast<int>(x / p.spt);
      const int s0 = static_cast<int>(x - static_cast<int64_t>(t) * p.spt);
      const int64_t seg_end = static_cast<int64_t>(t + 1) * p.spt < r1
                                  ? static_cast<int64_t>(t + 1) * p.spt
                                  : r1;
      const int s1 = static_cast<int>(seg_end - static_cast<int64_t>(t) * p.spt);
      const TileInfo ti = resolve_tile(p, t, NT);
      const int Bw = ti.mat.B;
      const int pitch = C::pitch(Bw);
      const int grow = tile_row(p, ti.rt, i);
      const bool valid = grow < p.N;
      // group metadata: the current group and a prefetch of the next one
      int cur_g = -1;
      int g_next = (s0 * kSlice) / p.G;
      float s_next = 0.f;
      uint32_t ab_next = 0;
      if (valid) {
        s_next = __ldg(ti.mat.scales + static_cast<int64_t>(grow) * ng + g_next);
        ab_next = __ldg(ti.mat.ab + static_cast<int64_t>(grow) * ng + g_next);
      }
      for (int sb = s0; sb < s1 && ok; sb += C::SPS) {
        const int ns = (s1 - sb) < C::SPS ? (s1 - sb) : C::SPS;
        if (!mbar_wait(bar_full + 8 * st, round & 1u, abort_flag, tmo, SITE_DECODER_FULL)) {
          ok = false;
          break;
        }
        const uint32_t wrow = stage0 + st * C::STAGE_BYTES + i * pitch;
        for (int j = 0; j < ns; ++j) {
          const int g = ((sb + j) * kSlice) / p.G;
          if (g != cur_g) {
            // g == g_next here: slices visit groups in order
            const float s_cur = s_next;
            const uint32_t ab_cur = ab_next;
            cur_g = g;
            g_next = g + 1;
            if (valid && g_next < ng) {
              s_next = __ldg(ti.mat.scales + static_cast<int64_t>(grow) * ng + g_next);
              ab_next = __ldg(ti.mat.ab + static_cast<int64_t>(grow) * ng + g_next);
            }
            if (Bw == 2)
              build_table<2>(tbase, valid, s_cur, ab_cur, p.mode);
            else if (Bw == 3)
              build_table<3>(tbase, valid, s_cur, ab_cur, p.mode);
            else
              build_table<4>(tbase, valid, s_cur, ab_cur, p.mode);
          }
          if (!mbar_wait(bar_tfree + 8 * ts, (tround & 1u) ^ 1u, abort_flag, tmo,
                         SITE_DECODER_TFREE)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t taddr = tmem_base + lane_off + ts * 64;
          const uint32_t caddr = wrow + j * 16 * Bw;
          if (Bw == 2)
            decode_slice_to_tmem<2>(caddr, tbase, taddr);
          else if (Bw == 3)
            decode_slice_to_tmem<3>(caddr, tbase, taddr);
          else
            decode_slice_to_tmem<4>(caddr, tbase, taddr);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar_aready + 8 * ts);
          if (++ts == kTmemRing) {
            ts = 0;
            ++tround;
          }
        }
        if (!ok) break;
        mbar_arrive(bar_wempty + 8 * st);
        if (++st == C::S) {
          st = 0;
          ++round;
        }
      }
      // ---------------------------------------------------------- epilogue
      if (ok && !mbar_wait(bar_dfull, seg & 1u, abort_flag, tmo, SITE_DECODER_DFULL))
        ok = false;
      if (!vote_all_decoders(ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t daddr = tmem_base + lane_off + kDCol;
      const int nchunks = (ti.m_valid + 15) >> 4;
      if (s0 == 0 && s1 == p.spt) {
        // whole tile in this CTA: straight to the output
        for (int cc = 0; cc < nchunks; ++cc) {
          uint32_t rr[16];
          tmem_ld16(daddr + cc * 16, rr);
          tmem_wait_ld();
          float v[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(rr[q]);
          finalize16(p, ti, i, grow, v, cc, xchg);
        }
        tc_fence_before();
        mbar_arrive(bar_dfree);
      } else {
        // partial tile: park it in the workspace, the last contributor reduces
        const int first_tile = static_cast<int>(r0 / p.spt);
        const int slot = 2 * cta + (t == first_tile ? 0 : 1);
        float* const mine = p.partial + static_cast<int64_t>(slot) * NT * kRows;
        for (int cc = 0; cc < nchunks; ++cc) {
          uint32_t rr[16];
          tmem_ld16(daddr + cc * 16, rr);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q)
            if (cc * 16 + q < ti.m_valid) mine[(cc * 16 + q) * kRows + i] = __uint_as_float(rr[q]);
        }
        tc_fence_before();
        mbar_arrive(bar_dfree);
        __threadfence();
        named_bar_decoders();
        const int64_t W_ = W;
        const int c_lo = owner_of(W_, p.P, static_cast<int64_t>(t) * p.spt);
        const int c_hi = owner_of(W_, p.P, static_cast<int64_t>(t) * p.spt + p.spt - 1);
        if (i == 0) {
          const int old = atomicAdd(p.counter + t, 1);
          *last_flag = (old == c_hi - c_lo) ? 1 : 0;
        }
        named_bar_decoders();
        const bool last = *last_flag != 0;
        if (last) {
          __threadfence();
          for (int cc = 0; cc < nchunks; ++cc) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = 0.f;
            for (int c = c_lo; c <= c_hi; ++c) {
              const int ft = static_cast<int>(range_begin(W_, p.P, c) / p.spt);
              const int sl = 2 * c + (t == ft ? 0 : 1);
              const float* src = p.partial + static_cast<int64_t>(sl) * NT * kRows;
#pragma unroll
              for (int q = 0; q < 16; ++q)
                if (cc * 16 + q < ti.m_valid) v[q] += __ldcg(src + (cc * 16 + q) * kRows + i);
            }
            finalize16(p, ti, i, grow, v, cc, xchg);
          }
          if (i == 0) p.counter[t] = 0;
        }
        named_bar_decoders();
      }
      ++seg;
      x = seg_end;
    }
  }

  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace cq
