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
// Warp roles (448 threads):
//   warps 0-7  decoders: weight row i of the tile (TMEM lane i) belongs to
//              thread i%32 of warps i/32 and i/32+4.  Warp q decodes the
//              even slices and warp q+4 the odd ones, each slice whole
//              (128 codes -> 64 BF16x2 words written to TMEM with
//              tcgen05.st, the A operand of the MMA), each from its own BF16
//              pair table per row (two codes -> two levels, one 32-bit word
//              per entry, the entries of all 128 rows interleaved so that
//              every lookup of a warp hits 32 distinct banks), so the two
//              never wait for each other.
//   warp 8     producer, two lanes with two rings of shared-memory stages:
//              lane 0 loads, per 128-code slice, two 2-D TMA boxes of 64
//              weight rows x 16*B bytes of packed codes (32-byte swizzle for
//              W2, 64-byte for W4, none for W3's 48-byte rows, so the
//              decoders' row-per-thread 16-byte reads are bank-conflict
//              free); lane 1 loads the activation tile as 64-column boxes
//              with the 128-byte swizzle.  The code ring is deep and cheap,
//              so the decoders run ahead of the activations.
//   warp 9     TMEM owner and MMA issuer: tcgen05.mma kind::f16 with A from
//              TMEM (decoded weights) and B from shared memory
//              (activations), FP32 accumulators in TMEM, double-buffered so
//              the next tile's MMAs overlap the previous tile's epilogue
//              (the ring of decoded slices shrinks from four to two at
//              NT = 176/192 to make room; NT = 256 would leave room for
//              only one accumulator buffer).
//   warps 10-13 epilogue: tcgen05.ld of the accumulator, output conversion,
//              SwiGLU, stream-K partials and their reduction.
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
constexpr int kThreads = 448;
constexpr int kTmemCols = 512;
constexpr int kTmemRing = 4;          // TMEM slice buffers (64 columns each), at most
constexpr int kDecoders = 256;        // two threads per weight row (even and odd slices)
constexpr int kEpilogue = 128;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kEpiWarp0 = 10;

// NT: token-tile width; TE: entries of a row's pair table (16 when every
// matrix of the launch has B = 2 or 4, 64 when one may have B = 3), or 0 for
// the wide-code decoder (any B in 1..8, levels evaluated per code, no
// tables, slices of up to 128 bytes per row).
template <int NT, int TE>
struct EngineCfg {
  static constexpr int SPS = NT <= 32 ? 4 : (NT == 64 ? 2 : 1);   // slices per stage
  // TMEM: a ring of decoded slices (64 columns each) and the accumulators.
  // Two accumulator buffers (the next tile's MMAs overlap this tile's
  // epilogue) beside a ring of four slices while they fit, else beside a
  // ring of two; at NT = 256 one buffer beside a ring of four.
  static constexpr int FREE2 = (kTmemCols - 2 * NT) / 64;      // ring slots left by 2 buffers
  static constexpr int NBUF = FREE2 >= 2 ? 2 : 1;
  static constexpr int RING = FREE2 >= 4 ? 4 : (FREE2 >= 2 ? FREE2 : kTmemRing);
  static constexpr int DCOL = RING * 64;                        // first accumulator column
  static constexpr int BMIN = TE == 0 ? 1 : 2;                  // code widths of the launch
  static constexpr int BMAX = TE == 0 ? 8 : 4;
  static constexpr int SLICE_W_BYTES = kRows * 16 * BMAX;       // one slice of packed rows
  static constexpr int W_STAGE = SPS * SLICE_W_BYTES;           // codes of SPS slices
  static constexpr int X_STAGE = 256 * SPS * NT;                // 2*SPS boxes of 64 x NT bf16
  static constexpr int XCHG_BYTES = 16 * 64 * 4;
  static constexpr int MISC_BYTES = 1024;
  static constexpr int TBL_BYTES = 2 * TE * kRows * 4;          // two pair tables per row
  static constexpr int BUDGET = 226 * 1024;
  static constexpr int AVAIL = BUDGET - 1024 - TBL_BYTES - XCHG_BYTES - MISC_BYTES;
  // two rings: activations (deep enough to cover the load latency) and codes
  // (small stages, so the decoders can run ahead of the activations).  A
  // finer activation ring (one box per entry) measured much slower: every
  // TMA operation has a fixed issue cost.
  static constexpr int SX_RAW = (AVAIL - 2 * W_STAGE) / X_STAGE;
  static constexpr int SX = SX_RAW > 4 ? 4 : SX_RAW;
  static constexpr int SW_RAW = (AVAIL - SX * X_STAGE) / W_STAGE;
  static constexpr int SW = SW_RAW > 8 ? 8 : SW_RAW;
  static constexpr int SMEM =
      1024 + SX * X_STAGE + SW * W_STAGE + TBL_BYTES + XCHG_BYTES + MISC_BYTES;
  static_assert(SX >= 2 && SW >= 2, "not enough shared memory for two stages per ring");
  static_assert(SMEM <= 227 * 1024, "shared memory budget exceeded");
  static_assert(DCOL + NBUF * NT <= kTmemCols && RING <= kTmemRing, "TMEM budget exceeded");
};

// One quantized matrix operand.
struct MatrixRef {
  const uint8_t* packed;
  const float* scales;
  const uint32_t* ab;     // (a | b << 16), fp16 bits
  int B;
  int reserved;
};

// One expert of a prepared MoE layer table (device memory, 64-byte aligned):
// the TMA descriptors of its packed gate/up and down matrices, then their
// operand descriptions.  Index 0 = gate/up [2I][H], 1 = down [H][I].
struct alignas(64) LayerEntry {
  CUtensorMap map[2];
  MatrixRef mat[2];
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
  // grouped (MoE) mode: tiles enumerate (active expert, row tile, token tile)
  int grouped;
  int which;                   // 0 = gate/up, 1 = down
  const LayerEntry* layer;     // [E]
  const int* g_ttpre;          // [E+1] prefix of token tiles per expert
  const int* g_cnt;            // [E] routes per expert
  const int* g_off;            // [E] first sorted route of each expert
  const int* g_num_tiles;      // device scalar: tiles of this launch
  const int* out_rows;         // optional sorted-position -> output row map
  int E;
  // workspace
  float* partial;        // [2P][NT][128]
  int* counter;          // [num_tiles]
  // extents of the buffers above, checked before every global access
  int64_t y_rows;        // rows of y
  int partial_slots;     // slots of partial
  int counter_len;       // entries of counter
  // control
  uint64_t timeout_ns;
  int debug_skip_first_stage;   // test hook: never issue stage load 0
  uint64_t* trace;              // optional [P][64] profile counters, or null
};

// Optional per-role cycle accounting into p.trace: PROF_MARK starts an
// interval, PROF_ADD(k) adds the cycles since the mark to counter k,
// PROF_FLUSH(base) stores the 8 counters at slots base..base+7 of this CTA.
#define PROF_MARK() (prof_t = p.trace ? clock64() : 0)
#define PROF_ADD(k)                                                         \
  do {                                                                      \
    if (p.trace) {                                                          \
      const long long now_ = clock64();                                     \
      prof[(k)] += now_ - prof_t;                                           \
      prof_t = now_;                                                        \
    }                                                                       \
  } while (0)
#define PROF_COUNT(k)                                                       \
  do {                                                                      \
    if (p.trace) prof[(k)] += 1;                                            \
  } while (0)
#define PROF_FLUSH(base)                                                    \
  do {                                                                      \
    if (p.trace) {                                                          \
      _Pragma("unroll") for (int k_ = 0; k_ < 8; ++k_)                      \
        p.trace[blockIdx.x * 64 + (base) + k_] = prof[k_];                  \
    }                                                                       \
  } while (0)

// Record a failed bounds check (site >= 20) in the device error word.
__device__ __forceinline__ void bad_access(int site) { atomicCAS(&g_device_error, 0, site); }

struct TileInfo {
  MatrixRef mat;
  const CUtensorMap* wmap;   // grouped mode: the expert's TMA descriptor (global memory)
  int rt, tt;
  int x_row0;       // first activation row of the token tile (tensor map row)
  int m_valid;      // valid tokens in this tile (<= NT)
};

// Tile t of the launch.  Plain mode: t = tt * n_rt + rt.  Grouped mode:
// experts in order, each contributing n_rt x ntt(e) tiles (tt fastest), so
// expert e owns tiles [n_rt * ttpre[e], n_rt * ttpre[e+1]).
__device__ __forceinline__ TileInfo resolve_tile(const EngineParams& p, int t, int NT,
                                                 int bmin, int bmax) {
  TileInfo ti;
  if (!p.grouped) {
    ti.mat = p.mat;
    ti.wmap = nullptr;          // plain mode loads through the kernel's own parameter
    // token tiles outermost: CTAs working at the same time share activation
    // tiles, which then stay in L2 (all row tiles' weights fit there anyway)
    ti.tt = t / p.n_rt;
    ti.rt = t - ti.tt * p.n_rt;
    ti.x_row0 = ti.tt * NT;
    const int rem = p.M - ti.x_row0;
    ti.m_valid = rem < NT ? rem : NT;
    return ti;
  }
  // largest e with n_rt * ttpre[e] <= t (experts with no tiles are skipped)
  int lo = 0, hi = p.E;                      // invariant: ttpre[lo]*n_rt <= t < ttpre[hi]*n_rt
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.n_rt * ld_guarded(p.g_ttpre + mid) <= t) lo = mid; else hi = mid;
  }
  const int e = lo;
  if (e < 0 || e >= p.E) bad_access(26);
  const int ntt = ld_guarded(p.g_ttpre + e + 1) - ld_guarded(p.g_ttpre + e);
  const int local = t - p.n_rt * ld_guarded(p.g_ttpre + e);
  ti.rt = local / ntt;
  ti.tt = local - ti.rt * ntt;
  const LayerEntry* le = p.layer + e;
  ti.mat = le->mat[p.which];
  if (ti.mat.B < bmin || ti.mat.B > bmax) {
    // a width this launch's rings and tables were not sized for: flag it and
    // decode a width that stays inside them
    bad_access(28);
    ti.mat.B = 2;
  }
  ti.wmap = &le->map[p.which];
  ti.x_row0 = ld_guarded(p.g_off + e) + ti.tt * NT;
  const int rem = ld_guarded(p.g_cnt + e) - ti.tt * NT;
  ti.m_valid = rem < NT ? rem : NT;
  return ti;
}

// Output row of sorted token position `pos`.
__device__ __forceinline__ int64_t out_row(const EngineParams& p, int pos) {
  if (p.out_rows) return static_cast<int64_t>(ld_guarded(p.out_rows + pos));
  return static_cast<int64_t>(pos);
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

// One segment of a CTA's range: the slices [s0, s1) of tile t.
struct Segment {
  int t, s0, s1;
  int64_t end;
};
__device__ __forceinline__ Segment segment_at(int64_t x, int64_t r1, int spt) {
  Segment g;
  g.t = static_cast<int>(x / spt);
  const int64_t tbeg = static_cast<int64_t>(g.t) * spt;
  g.s0 = static_cast<int>(x - tbeg);
  g.end = tbeg + spt < r1 ? tbeg + spt : r1;
  g.s1 = static_cast<int>(g.end - tbeg);
  return g;
}

// Wait with an inline fast path; the bounded slow path is out of line.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort,
                                           uint64_t timeout_ns, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait(bar, parity, abort, timeout_ns, site);
}

// ---------------------------------------------------------------------------
// decoder helpers
// ---------------------------------------------------------------------------

// The 2^B levels of one row's group (BF16 bits): q(t) in FP64, times s,
// rounded once to FP32 and then to BF16.  Levels are odd in k (q(t) carries
// the sign), so only the positive side is evaluated and the negative codes
// flip the BF16 sign bit.
template <int B>
__device__ __forceinline__ void group_levels(bool valid, float s, uint32_t abw, int mode,
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
    // codes H+j (j = 0..H-1) are the positive side, H-1-j their mirror
#pragma unroll
    for (int j = 0; j < H; ++j) {
      const uint32_t m = bf16_bits(static_cast<float>(level_f64(H + j, B, 0, s, a, b)));
      L[H + j] = m;
      L[H - 1 - j] = m ^ 0x8000u;
    }
  } else {
    // Kc = H-1; code Kc+m has |k| = m (m = 0..H), code Kc-m its mirror
#pragma unroll
    for (int m = 0; m <= H; ++m) {
      const uint32_t v = bf16_bits(static_cast<float>(level_f64(H - 1 + m, B, 1, s, a, b)));
      L[H - 1 + m] = v;
      if (m >= 1 && m <= H - 1) L[H - 1 - m] = v ^ 0x8000u;
    }
  }
}

// Pair-table layout in shared memory: entry e of tile row i is the 32-bit
// word at tbl + e*128 + i (words), so the lookups of a warp always hit 32
// distinct banks.  Entries:
//   B=2: e = u0 | u1<<2 (16 entries)  ->  L[u0] | L[u1] << 16
//   B=3: e = u0 | u1<<3 (64 entries)  ->  L[u0] | L[u1] << 16
//   B=4: e = u        (16 entries)   ->  L[u]  | L[u]  << 16
// with L_u the level of code u.  One thread builds the whole table of its
// row from one evaluation of the levels.
template <int B>
__device__ __forceinline__ void build_table_all(uint32_t* tbl, int i, bool valid, float s,
                                                uint32_t abw, int mode) {
  uint32_t L[1 << B];
  group_levels<B>(valid, s, abw, mode, L);
  if constexpr (B == 2) {
#pragma unroll
    for (int e = 0; e < 16; ++e) tbl[e * kRows + i] = L[e & 3] | (L[e >> 2] << 16);
  } else if constexpr (B == 3) {
#pragma unroll
    for (int e = 0; e < 64; ++e) tbl[e * kRows + i] = L[e & 7] | (L[e >> 3] << 16);
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) tbl[e * kRows + i] = L[e] | (L[e] << 16);
  }
}

// Bits [sh, ...) of word w moved to bit 7 (the table's entry stride in words).
__device__ __forceinline__ uint32_t at_bit7(uint32_t w, int sh) {
  return sh >= 7 ? (w >> (sh - 7)) : (w << (7 - sh));
}

// Decode pairs [P0, P0+32) of one 128-code slice (codes in c[]) into r[].
template <int B, int P0>
__device__ __forceinline__ void decode_half(const uint32_t (&c)[4 * B], const uint32_t* tbl,
                                            uint32_t i, uint32_t (&r)[32]) {
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int p = P0 + q;
    if constexpr (B == 2) {
      const uint32_t v = at_bit7(c[p >> 3], 4 * (p & 7));
      r[q] = tbl[(v & (15u << 7)) | i];
    } else if constexpr (B == 3) {
      const int o = 6 * p;
      const int wi = o >> 5, sh = o & 31;
      uint32_t v;
      if (sh <= 26)
        v = at_bit7(c[wi], sh);
      else
        v = __funnelshift_r(c[wi], c[wi + 1 < 4 * B ? wi + 1 : 4 * B - 1], sh - 7);
      r[q] = tbl[(v & (63u << 7)) | i];
    } else {
      const int sh = 8 * (p & 3);
      const uint32_t w = c[p >> 2];
      const uint32_t lo = tbl[(at_bit7(w, sh) & (15u << 7)) | i];
      const uint32_t hi = tbl[(at_bit7(w, sh + 4) & (15u << 7)) | i];
      r[q] = __byte_perm(lo, hi, 0x7610);
    }
  }
}

// Decode pairs [32*HALF, 32*HALF+32) of one slice into TMEM columns
// taddr .. taddr+31 (taddr already offset by 32*HALF).
template <int B, int HALF>
__device__ __forceinline__ void decode_half_slice_to_tmem(const uint4* codes, uint32_t swz,
                                                          const uint32_t* tbl, uint32_t i,
                                                          uint32_t taddr) {
  uint32_t c[4 * B];
#pragma unroll
  for (int v = 0; v < B; ++v) {
    // only the 16-byte chunks holding this half's bits are needed
    if ((v + 1) * 128 > HALF * 32 * 2 * B && v * 128 < (HALF + 1) * 32 * 2 * B) {
      const uint4 q = codes[v ^ swz];
      c[4 * v + 0] = q.x;
      c[4 * v + 1] = q.y;
      c[4 * v + 2] = q.z;
      c[4 * v + 3] = q.w;
    } else {
      c[4 * v + 0] = c[4 * v + 1] = c[4 * v + 2] = c[4 * v + 3] = 0u;
    }
  }
  uint32_t r[32];
  decode_half<B, 32 * HALF>(c, tbl, i, r);
  tmem_st32(taddr, r);
}

// Wide-code decoder (TE = 0): the level of every code is evaluated on the
// spot, with the same FP64 steps as a table entry (q(t) in FP64, times s,
// rounded once to FP32 and then to BF16).  A 2^B-entry table per row would
// not fit beside the rings for B = 8, and for G = 512 building it costs
// about as much as evaluating each code once.  t = |k| / Kc is taken as
// |k| * (1 / Kc): exact for |k| in {0, Kc}, elsewhere within one FP64 ulp of
// the quotient, 2^-45 of a BF16 step.
struct WideRow {
  double a, b, c, rinv;   // shape parameters, c = 1 - a - b, 1 / Kc'
  float s;                // group scale (0 for rows past N)
  int mult, off;          // k' = mult * u - off: midrise 2u - (2^B - 1), midtread u - Kc
};

__device__ __forceinline__ WideRow wide_row(bool valid, float s, uint32_t abw, int mode, int B) {
  WideRow w;
  w.a = static_cast<double>(__half2float(__ushort_as_half(abw & 0xFFFFu)));
  w.b = static_cast<double>(__half2float(__ushort_as_half(abw >> 16)));
  w.c = 1.0 - w.a - w.b;
  w.s = valid ? s : 0.f;
  w.mult = mode == CQ_GRID_MIDRISE ? 2 : 1;
  w.off = mode == CQ_GRID_MIDRISE ? (1 << B) - 1 : (1 << (B - 1)) - 1;
  w.rinv = 1.0 / static_cast<double>(w.off > 0 ? w.off : 1);
  return w;
}

// FP32 level of code u before the sign (|s q(t)|), and whether k < 0.
__device__ __forceinline__ float wide_level(const WideRow& w, uint32_t u, bool& neg) {
  const int k = w.mult * static_cast<int>(u) - w.off;
  neg = k < 0;
  const int ak = k < 0 ? -k : k;
  // |k| as a double without a conversion instruction: 2^52 + ak, minus 2^52
  double t = (__hiloint2double(0x43300000, ak) - 4503599627370496.0) * w.rinv;
  if (ak == w.off) t = 1.0;
  const double q = t * (w.a + t * (w.b + t * w.c));
  return static_cast<float>(static_cast<double>(w.s) * q);
}

// The B-bit code at bit offset o of the slice words c[] (LSB first).
template <int B>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&c)[4 * B], int o) {
  const int wi = o >> 5, sh = o & 31;
  uint32_t v;
  if (sh + B <= 32)
    v = c[wi] >> sh;
  else
    v = __funnelshift_r(c[wi], c[wi + 1 < 4 * B ? wi + 1 : 4 * B - 1], sh);
  return v & ((1u << B) - 1u);
}

// Decode pairs [32*HALF, 32*HALF+32) of one slice of a B-bit row into TMEM
// columns taddr .. taddr+31: the wide-code counterpart of
// decode_half_slice_to_tmem.
template <int B, int HALF>
__device__ __forceinline__ void decode_wide_half_to_tmem(const uint4* codes, uint32_t swz,
                                                         const WideRow& w, uint32_t taddr) {
  uint32_t c[4 * B];
#pragma unroll
  for (int v = 0; v < B; ++v) {
    if ((v + 1) * 128 > HALF * 32 * 2 * B && v * 128 < (HALF + 1) * 32 * 2 * B) {
      const uint4 q = codes[v ^ swz];
      c[4 * v + 0] = q.x;
      c[4 * v + 1] = q.y;
      c[4 * v + 2] = q.z;
      c[4 * v + 3] = q.w;
    } else {
      c[4 * v + 0] = c[4 * v + 1] = c[4 * v + 2] = c[4 * v + 3] = 0u;
    }
  }
  uint32_t r[32];
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int pr = 32 * HALF + q;                 // pair: codes 2pr (low) and 2pr+1 (high)
    bool n0, n1;
    const float l0 = wide_level(w, code_at<B>(c, 2 * pr * B), n0);
    const float l1 = wide_level(w, code_at<B>(c, (2 * pr + 1) * B), n1);
    const __nv_bfloat162 h = __floats2bfloat162_rn(l0, l1);
    r[q] = *reinterpret_cast<const uint32_t*>(&h) ^ (n0 ? 0x8000u : 0u) ^
           (n1 ? 0x80000000u : 0u);
  }
  tmem_st32(taddr, r);
}

template <int B>
__device__ __forceinline__ void decode_wide_slice_to_tmem(const uint4* codes, uint32_t swz,
                                                          const WideRow& w, uint32_t taddr) {
  decode_wide_half_to_tmem<B, 0>(codes, swz, w, taddr);
  decode_wide_half_to_tmem<B, 1>(codes, swz, w, taddr + 32);
}

// ---------------------------------------------------------------------------
// epilogue helpers (warps 6-9, named barrier 2)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void named_bar_epilogue() {
  asm volatile("bar.sync 2, 128;" ::: "memory");
}

// All-epilogue-threads AND-vote at named barrier 2.  Every epilogue thread
// reaches it once per segment, whether or not one of its waits gave up, so
// the epilogue's named barriers are only entered when all 128 agree.
__device__ __forceinline__ bool vote_all_epilogue(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(ok))
      : "memory");
  return r != 0;
}

// Store 16 accumulator columns (tokens m0..m0+15 of the tile) of tile row i.
__device__ __forceinline__ void finalize16(const EngineParams& p, const TileInfo& ti, int i,
                                           int grow, const float (&v)[16], int cc,
                                           float* xchg) {
  const int m0 = cc * 16;
  if (p.epilogue == CQ_EPI_SWIGLU) {
    // Tile rows i and i + 64 hold the gate and up value of output column
    // rt * 64 + (i & 63).  The gate row finishes tokens 0-7 of the chunk and
    // the up row tokens 8-15: each hands the other half over through xchg.
    const int r = i & 63;
    const bool up = i >= 64;
#pragma unroll
    for (int q = 0; q < 8; ++q) xchg[(up ? q : q + 8) * 64 + r] = up ? v[q] : v[q + 8];
    named_bar_epilogue();
    const int qb = up ? 8 : 0;
    float h[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float other = xchg[(qb + q) * 64 + r];
      const float mine = up ? v[q + 8] : v[q];
      const float g = up ? other : mine;
      const float u = up ? mine : other;
      h[q] = g / (1.0f + __expf(-g)) * u;
    }
    named_bar_epilogue();
    const int col = ti.rt * 64 + r;
    const int mv = min(8, ti.m_valid - (m0 + qb));
    if (col >= p.ldy) {
      if (mv > 0) bad_access(23);
    } else if (!p.out_rows) {
      const int64_t r0 = static_cast<int64_t>(ti.x_row0) + m0 + qb;
      if (mv > 0 && (r0 < 0 || r0 + mv > p.y_rows)) {
        bad_access(23);
      } else if (p.out_bf16) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.y) + r0 * p.ldy + col;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < mv) dst[q * p.ldy] = __float2bfloat16_rn(h[q]);
      } else {
        float* dst = reinterpret_cast<float*>(p.y) + r0 * p.ldy + col;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < mv) dst[q * p.ldy] = h[q];
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q < mv) {
          const int64_t orow = out_row(p, ti.x_row0 + m0 + qb + q);
          const int64_t off = orow * p.ldy + col;
          if (orow < 0 || orow >= p.y_rows) {
            bad_access(23);
          } else if (p.out_bf16)
            reinterpret_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(h[q]);
          else
            reinterpret_cast<float*>(p.y)[off] = h[q];
        }
      }
    }
  } else if (!p.out_rows) {
    // tokens land in consecutive output rows: one bounds check per chunk and
    // a strided store per token (the epilogue warps share their schedulers
    // with the decoders, so few instructions per element matter)
    if (grow < p.N) {
      const int mv = min(16, ti.m_valid - m0);
      const int64_t r0 = static_cast<int64_t>(ti.x_row0) + m0;
      if (r0 < 0 || r0 + mv > p.y_rows || grow >= p.ldy) {
        if (mv > 0) bad_access(23);
      } else if (p.out_bf16) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.y) + r0 * p.ldy + grow;
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (q < mv) dst[q * p.ldy] = __float2bfloat16_rn(v[q]);
      } else {
        float* dst = reinterpret_cast<float*>(p.y) + r0 * p.ldy + grow;
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (q < mv) dst[q * p.ldy] = v[q];
      }
    }
  } else {
    if (grow < p.N) {
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int m = m0 + q;
        if (m < ti.m_valid) {
          const int64_t orow = out_row(p, ti.x_row0 + m);
          const int64_t off = orow * p.ldy + grow;
          if (orow < 0 || orow >= p.y_rows || grow >= p.ldy) {
            bad_access(23);
          } else if (p.out_bf16)
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
template <int NT, int TE>
__global__ void __launch_bounds__(kThreads, 1)
    engine_kernel(const __grid_constant__ EngineParams p,
                  const __grid_constant__ CUtensorMap xmap,
                  const __grid_constant__ CUtensorMap wmap) {
  using C = EngineCfg<NT, TE>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-align the working area (swizzled TMA destinations need it)
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t xring = base;                             // [SX][X_STAGE]
  const uint32_t wring = xring + C::SX * C::X_STAGE;       // [SW][W_STAGE]
  const uint32_t tbl_s = wring + C::SW * C::W_STAGE;       // [2][TE][128] words
  const uint32_t xchg_s = tbl_s + C::TBL_BYTES;
  const uint32_t misc = xchg_s + C::XCHG_BYTES;
  uint8_t* const gbase = smem_raw + (base - raw);
  float* const xchg = reinterpret_cast<float*>(gbase + (xchg_s - base));
  uint32_t* const tbl = reinterpret_cast<uint32_t*>(gbase + (tbl_s - base));
  // barriers and flags
  const uint32_t bar_wfull = misc;                        // [SW] codes landed
  const uint32_t bar_wfree = bar_wfull + 8 * C::SW;       // [SW] decoders done with them
  const uint32_t bar_xfull = bar_wfree + 8 * C::SW;       // [SX] activations landed
  const uint32_t bar_xfree = bar_xfull + 8 * C::SX;       // [SX] MMAs done with them
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
  const long long prof_start = clock64();
  long long prof[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  long long prof_t = 0;

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
      mbar_init(bar_aready + 8 * s, kRows);          // one decoder thread per row and slice
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
    if (!p.grouped) prefetch_tensormap(&wmap);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base =
      *reinterpret_cast<volatile uint32_t*>(gbase + (slot_tmem - base));
  // programmatic dependent launch: the setup above overlapped the preceding
  // grid; nothing written by it is read before this wait returns
  griddep_wait();

  int num_tiles = p.num_tiles;
  if (p.grouped) num_tiles = ld_guarded(p.g_num_tiles);
  const int64_t W = static_cast<int64_t>(num_tiles) * p.spt;
  // CTAs that take part: at most one per slice, so that every CTA of the
  // partition owns at least one slice (the stream-K reduction counts on it)
  const int Pe = W < p.P ? static_cast<int>(W) : p.P;
  const int64_t r0 = cta < Pe ? range_begin(W, Pe, cta) : W;
  const int64_t r1 = cta < Pe ? range_begin(W, Pe, cta + 1) : W;
  const uint64_t tmo = p.timeout_ns;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    // Lane 0 keeps the code ring full, lane 1 the activation ring (both in
    // stages of SPS slices): the decoders run ahead of the activations
    // (bounded by the TMEM ring) and the MMA waits for activations only.
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
        const TileInfo ti = resolve_tile(p, sg.t, NT, C::BMIN, C::BMAX);
        const int Bw = ti.mat.B;
        // first weight row of the two 64-row boxes of this tile
        const int row_a = tile_row(p, ti.rt, 0);
        const int row_b = tile_row(p, ti.rt, 64);
        for (int sb = sg.s0; ok && sb < sg.s1; sb += C::SPS) {
          const int ns = (sg.s1 - sb) < C::SPS ? (sg.s1 - sb) : C::SPS;
          {
            PROF_MARK();
            if (!wait_phase(free0 + 8 * st, (round & 1u) ^ 1u, abort_flag, tmo,
                            SITE_PRODUCER_EMPTY)) {
              ok = false;
              break;
            }
            PROF_ADD(0);
            const bool skip = p.debug_skip_first_stage && load_no == 0;
            if (wl) {
              // the kernel parameter's address is only ever used directly in
              // the TMA instruction; table descriptors must lie inside the table
              const bool map_ok = !p.grouped || (ti.wmap >= &p.layer[0].map[0] &&
                                                 ti.wmap < &p.layer[p.E].map[0]);
              if (!map_ok) bad_access(21);
              if (!skip && map_ok) {
                const uint32_t wbox = 64u * 16u * Bw;               // bytes of one weight box
                const uint32_t wdst = wring + st * C::W_STAGE;
                mbar_arrive_expect_tx(bar_wfull + 8 * st, static_cast<uint32_t>(ns) * 2u * wbox);
                for (int j = 0; j < ns; ++j) {
                  const int cb = (sb + j) * 16 * Bw;               // byte column of the slice
                  const uint32_t sdst = wdst + j * C::SLICE_W_BYTES;
                  if (p.grouped) {
                    tma_load_2d(sdst, ti.wmap, cb, row_a, bar_wfull + 8 * st);
                    tma_load_2d(sdst + wbox, ti.wmap, cb, row_b, bar_wfull + 8 * st);
                  } else {
                    tma_load_2d(sdst, &wmap, cb, row_a, bar_wfull + 8 * st);
                    tma_load_2d(sdst + wbox, &wmap, cb, row_b, bar_wfull + 8 * st);
                  }
                }
              }
            } else if (!skip) {
              const uint32_t xdst = xring + st * C::X_STAGE;
              mbar_arrive_expect_tx(bar_xfull + 8 * st, static_cast<uint32_t>(2 * ns * NT * 128));
              for (int b = 0; b < 2 * ns; ++b)
                tma_load_2d(xdst + b * (NT * 128), &xmap, sb * kSlice + b * 64, ti.x_row0,
                            bar_xfull + 8 * st);
            }
            PROF_ADD(1);
            PROF_COUNT(2);
            ++load_no;
            if (++st == NS) {
              st = 0;
              ++round;
            }
          }
        }
        if (ok) x = sg.end;
      }
      if (wl) PROF_FLUSH(8);
      if (*abort_flag) {
        // make sure no copy is still landing in shared memory before exit:
        // the ring positions armed last are the only ones that may be in flight
        const int armed = load_no < NS ? load_no : NS;
        for (int k = 1; k <= armed; ++k) {
          const int idx = load_no - k;
          if (p.debug_skip_first_stage && idx == 0) continue;
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
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kRows, NT);
      int st = 0, ts = 0;
      uint32_t round = 0, tround = 0, seg = 0;
      bool ok = true;
      for (int64_t x = r0; ok && x < r1;) {
        const Segment sg = segment_at(x, r1, p.spt);
        const uint32_t db = C::NBUF == 2 ? (seg & 1u) : 0u;
        const uint32_t duse = C::NBUF == 2 ? (seg >> 1) : seg;   // earlier uses of buffer db
        PROF_MARK();
        if (!wait_phase(bar_dfree + 8 * db, (duse & 1u) ^ 1u, abort_flag, tmo,
                        SITE_MMA_DFREE)) {
          ok = false;
          break;
        }
        PROF_ADD(0);
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + C::DCOL + db * NT;
        uint32_t acc = 0;
        for (int sb = sg.s0; sb < sg.s1 && ok; sb += C::SPS) {
          const int ns = (sg.s1 - sb) < C::SPS ? (sg.s1 - sb) : C::SPS;
          PROF_MARK();
          if (!wait_phase(bar_xfull + 8 * st, round & 1u, abort_flag, tmo, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          PROF_ADD(1);
          tc_fence_after();
          const uint64_t desc0 = smem_desc_sw128(xring + st * C::X_STAGE);
          for (int j = 0; j < ns; ++j) {
            PROF_MARK();
            if (!wait_phase(bar_aready + 8 * ts, tround & 1u, abort_flag, tmo,
                            SITE_MMA_AREADY)) {
              ok = false;
              break;
            }
            PROF_ADD(2);
            tc_fence_after();
            const uint32_t a0 = tmem_base + ts * 64;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              // activation box 2j + kk/4, 32-byte K step inside its 128-byte rows
              const uint64_t off =
                  static_cast<uint64_t>(((2 * j + (kk >> 2)) * NT * 128 + (kk & 3) * 32) >> 4);
              mma_ts_bf16(d_tmem, a0 + kk * 8, desc0 + off, idesc, acc);
              acc = 1;
            }
            mma_commit(bar_tfree + 8 * ts);
            PROF_ADD(3);
            PROF_COUNT(4);
            if (++ts == C::RING) {
              ts = 0;
              ++tround;
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
        mma_commit(bar_dfull + 8 * db);
        ++seg;
        x = sg.end;
      }
      PROF_FLUSH(16);
      // all issued MMAs have completed before TMEM is released
      mma_commit(bar_fin);
      volatile int dummy = 0;
      mbar_wait(bar_fin, 0, &dummy, tmo, SITE_TEARDOWN);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ decoders
    // Warp q (q < 4) decodes the even slices and warp q + 4 the odd ones,
    // each slice whole, for tile rows 32q .. 32q+31 (TMEM lanes).  Each of
    // the two has its own pair table per row, so neither waits for the other.
    const int q = warp & 3;                              // TMEM lane quarter
    const int h = warp >> 2;                             // parity of the slices decoded
    const int i = q * 32 + lane;                         // tile row / TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t* const mytbl = tbl + h * (TE * kRows);
    int st = 0, ts = 0;
    uint32_t round = 0, tround = 0;
    bool ok = true;
    const int ng = p.K / p.G;
    const int spc = p.G / kSlice;                        // slices per group
    for (int64_t x = r0; ok && x < r1;) {
      const Segment sg = segment_at(x, r1, p.spt);
      const TileInfo ti = resolve_tile(p, sg.t, NT, C::BMIN, C::BMAX);
      const int Bw = ti.mat.B;
      const int grow = tile_row(p, ti.rt, i);
      // 16-byte chunk v of this row sits at chunk (v ^ swz) of the row (TMA swizzle)
      const uint32_t swz =
          Bw == 2 ? ((i >> 2) & 1u) : (Bw == 4 ? ((i >> 1) & 3u) : (Bw == 8 ? (i & 7u) : 0u));
      const bool valid = grow < p.N;
      // group metadata: the current group and a prefetch of the next group
      // this thread meets (its first slice of this segment, then after each
      // switch the group of its first slice past the current group)
      int cur_g = -1;
      WideRow wr = {};
      const int s_first = sg.s0 + ((sg.s0 & 1) != h ? 1 : 0);
      float s_next = 0.f;
      uint32_t ab_next = 0;
      if (valid && s_first < sg.s1) {
        const int g0 = s_first / spc;
        if (g0 < ng) {
          s_next = __ldg(ti.mat.scales + static_cast<int64_t>(grow) * ng + g0);
          ab_next = __ldg(ti.mat.ab + static_cast<int64_t>(grow) * ng + g0);
        } else {
          bad_access(22);
        }
      }
      for (int sb = sg.s0; sb < sg.s1 && ok; sb += C::SPS) {
        const int ns = (sg.s1 - sb) < C::SPS ? (sg.s1 - sb) : C::SPS;
        PROF_MARK();
        if (!wait_phase(bar_wfull + 8 * st, round & 1u, abort_flag, tmo, SITE_DECODER_FULL)) {
          ok = false;
          break;
        }
        PROF_ADD(0);
        const uint32_t wrow = wring + st * C::W_STAGE + i * 16 * Bw;
        for (int j = 0; j < ns; ++j) {
          const int sl = sb + j;
          if ((sl & 1) == h) {
            const int g = sl / spc;
            if (TE == 16 && Bw == 3) {
              // a 64-entry table does not fit this launch's tables (the host
              // never plans it): record it and leave the table alone
              if (g != cur_g && i == 0) bad_access(27);
              cur_g = g;
            }
            if (g != cur_g) {
              // slices of this parity visit groups in order: g is the
              // prefetched one
              const float s_cur = s_next;
              const uint32_t ab_cur = ab_next;
              cur_g = g;
              const int send = (g + 1) * spc;                 // first slice past group g
              const int snext = send + ((send & 1) != h ? 1 : 0);
              const int gn = snext / spc;
              if (valid && snext < sg.s1 && gn < ng) {
                s_next = __ldg(ti.mat.scales + static_cast<int64_t>(grow) * ng + gn);
                ab_next = __ldg(ti.mat.ab + static_cast<int64_t>(grow) * ng + gn);
              }
              if constexpr (TE == 0)
                wr = wide_row(valid, s_cur, ab_cur, p.mode, Bw);
              else if (Bw == 2)
                build_table_all<2>(mytbl, i, valid, s_cur, ab_cur, p.mode);
              else if (Bw == 3)
                build_table_all<3>(mytbl, i, valid, s_cur, ab_cur, p.mode);
              else
                build_table_all<4>(mytbl, i, valid, s_cur, ab_cur, p.mode);
              PROF_COUNT(7);
            }
            PROF_ADD(1);
            if (!wait_phase(bar_tfree + 8 * ts, (tround & 1u) ^ 1u, abort_flag, tmo,
                            SITE_DECODER_TFREE)) {
              ok = false;
              break;
            }
            PROF_ADD(2);
            tc_fence_after();
            const uint32_t taddr = tmem_base + lane_off + ts * 64;
            const uint4* caddr =
                reinterpret_cast<const uint4*>(gbase + (wrow + j * C::SLICE_W_BYTES - base));
            if constexpr (TE == 0) {
              switch (Bw) {
                case 1: decode_wide_slice_to_tmem<1>(caddr, swz, wr, taddr); break;
                case 2: decode_wide_slice_to_tmem<2>(caddr, swz, wr, taddr); break;
                case 3: decode_wide_slice_to_tmem<3>(caddr, swz, wr, taddr); break;
                case 4: decode_wide_slice_to_tmem<4>(caddr, swz, wr, taddr); break;
                case 5: decode_wide_slice_to_tmem<5>(caddr, swz, wr, taddr); break;
                case 6: decode_wide_slice_to_tmem<6>(caddr, swz, wr, taddr); break;
                case 7: decode_wide_slice_to_tmem<7>(caddr, swz, wr, taddr); break;
                default: decode_wide_slice_to_tmem<8>(caddr, swz, wr, taddr); break;
              }
            } else if (Bw == 2) {
              decode_half_slice_to_tmem<2, 0>(caddr, swz, mytbl, i, taddr);
              decode_half_slice_to_tmem<2, 1>(caddr, swz, mytbl, i, taddr + 32);
            } else if (Bw == 3) {
              decode_half_slice_to_tmem<3, 0>(caddr, swz, mytbl, i, taddr);
              decode_half_slice_to_tmem<3, 1>(caddr, swz, mytbl, i, taddr + 32);
            } else {
              decode_half_slice_to_tmem<4, 0>(caddr, swz, mytbl, i, taddr);
              decode_half_slice_to_tmem<4, 1>(caddr, swz, mytbl, i, taddr + 32);
            }
            PROF_ADD(3);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_aready + 8 * ts);
            PROF_ADD(4);
            PROF_COUNT(6);
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
    if (tid == 0) PROF_FLUSH(24);
    if (tid == 255) PROF_FLUSH(32);
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                              // TMEM lane quarter
    const int i = q * 32 + lane;                         // tile row
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t seg = 0;
    bool ok = true;
    for (int64_t x = r0; ok && x < r1;) {
      const Segment sg = segment_at(x, r1, p.spt);
      const TileInfo ti = resolve_tile(p, sg.t, NT, C::BMIN, C::BMAX);
      const int grow = tile_row(p, ti.rt, i);
      const uint32_t db = C::NBUF == 2 ? (seg & 1u) : 0u;
      const uint32_t duse = C::NBUF == 2 ? (seg >> 1) : seg;
      PROF_MARK();
      if (!wait_phase(bar_dfull + 8 * db, duse & 1u, abort_flag, tmo, SITE_DECODER_DFULL))
        ok = false;
      if (!vote_all_epilogue(ok)) {
        ok = false;
        break;
      }
      PROF_ADD(0);
      tc_fence_after();
      const uint32_t daddr = tmem_base + lane_off + C::DCOL + db * NT;
      const int nchunks = (ti.m_valid + 15) >> 4;
      if (sg.s0 == 0 && sg.s1 == p.spt) {
        // whole tile in this CTA: straight to the output
        for (int cc = 0; cc < nchunks; ++cc) {
          uint32_t rr[16];
          tmem_ld16(daddr + cc * 16, rr);
          tmem_wait_ld();
          float v[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(rr[k]);
          finalize16(p, ti, i, grow, v, cc, xchg);
        }
        tc_fence_before();
        mbar_arrive(bar_dfree + 8 * db);
      } else {
        // partial tile: park it in the workspace, the last contributor reduces
        const int first_tile = static_cast<int>(r0 / p.spt);
        const int slot = 2 * cta + (sg.t == first_tile ? 0 : 1);
        const bool slot_ok = slot < p.partial_slots && sg.t < p.counter_len;
        if (!slot_ok && i == 0) bad_access(24);
        float* const mine = p.partial + static_cast<int64_t>(slot_ok ? slot : 0) * NT * kRows;
        for (int cc = 0; cc < nchunks; ++cc) {
          uint32_t rr[16];
          tmem_ld16(daddr + cc * 16, rr);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (slot_ok && cc * 16 + k < ti.m_valid)
              mine[(cc * 16 + k) * kRows + i] = __uint_as_float(rr[k]);
        }
        tc_fence_before();
        mbar_arrive(bar_dfree + 8 * db);
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
      PROF_ADD(1);
      PROF_COUNT(2);
      ++seg;
      x = sg.end;
    }
    if (i == 64) PROF_FLUSH(40);
  }

  __syncthreads();
  if (tid == 0 && p.trace) p.trace[blockIdx.x * 64 + 1] = clock64() - prof_start;
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace cq
