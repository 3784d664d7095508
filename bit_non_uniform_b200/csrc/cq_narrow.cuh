// cq_narrow.cuh -- the narrow-row CubicQuant GEMM: up to 16 activation rows
// (decode-sized batches), sm_100a.
//
// With at most 16 tokens the product streams the packed weights once and its
// cost is turning codes into operands; the multiply-accumulate is cheap.  Each
// pair of codes becomes a BF16x2 operand word through a per-(row, group)
// lookup table in shared memory and goes straight into the register operands
// of the warp-level tensor-core MMA (mma.sync m16n8k16, FP32 accumulation).
//
// Dense fragments.  In an m16n8k16 MMA, lane (g, c) of a warp (g = lane/4,
// c = lane%4) supplies the weights of MMA rows g and g+8 at the K positions
// {2c, 2c+1, 2c+8, 2c+9}, and the activations of token g at the same K
// positions.  The K dimension of the MMA is a free choice as long as both
// operands agree, so "lane column" c is given its own quarter of the row:
// K is cut into four quarters of Q = K/512 slices (128 codes each), lane
// column c walks slices c*Q .. c*Q+Q-1, and at MMA step s of a slice its four
// K positions are the slice's codes 4s .. 4s+3.  All four lane columns then
// add to the same output (row, token): every product of every MMA is useful,
// and one MMA covers 16 weight rows x 8 tokens x 16 codes (two MMAs for 9 to
// 16 tokens).  Quarters are at least a group apart (K/4 >= G), so the four
// lanes of a row read the tables of four different groups: each lane has its
// own tables, interleaved so that a warp's 32 lookups hit 32 distinct banks.
//
// Work split (stream-K).  A row block is 16 weight rows (with the SwiGLU
// epilogue: 8 gate rows and the 8 matching up rows, so MMA rows g and g+8
// hold the gate and up value of the same output).  A unit is (row block rb,
// slice step j): the 16 rows times slice j of each quarter, 8192 weights.
// Units are numbered rb-major and split evenly over the CTAs (one per SM).  A
// CTA builds the level tables of every (row, group) its units touch; its
// warps then take the units round robin and leave each unit's partial sums
// in a shared-memory slot.  After one barrier, warp r sums the slots of the
// CTA's row block r (slice steps in order) and writes it out.  A row block
// shared by consecutive CTAs: the later CTAs park their parts in the
// workspace and count them; the first CTA (the owner) waits for the count
// and adds the parts in CTA order.  A CTA publishes its own part before it
// waits for any, so the waits form a chain that ends at the last CTA.
// Results are run-to-run deterministic.
//
// Loads.  Each warp loads the codes of its own units straight into registers
// with 16-byte global loads (the lane's two rows of one slice of its
// quarter), NB units ahead of its decoding, and the CTA stages its
// activations once, with 16-byte asynchronous copies, as [slice step][k pair]
// [token][quarter][8 values], so that a warp's 16-byte activation loads are
// conflict free.  No fence or barrier lies between a warp's first code load
// and its last unit: a fence (and a barrier, which orders memory like one)
// waits until the loads in flight have landed, which would stop the warp
// until the codes of its later units arrive.  The CTA's rows are also
// prefetched into L2 in a few bulk requests at the start.  (Box copies of 16
// rows x 4 quarters x one 48-byte slice came in too slowly: the copy engine
// handles such short rows at a few bytes per cycle.)  No shared-memory ring,
// no producer warp: eight warps build the tables, decode, multiply and
// finish row blocks.
//
// This is the narrow-row GEMV of the article's A16 path ("压缩权重必须“边解码、
// 边计算”"): codes and group parameters -> levels generated in the tile ->
// model-dtype operands -> dot product with FP32 accumulation -> output dtype,
// the weights never materialised; the group scale is folded into the BF16
// level (BF16(s q) has the relative rounding of BF16(q)).
#pragma once

#include "cq.h"
#include "cq_device.cuh"
#include "cq_gemv.cuh"

namespace cq {

constexpr int kNrCompute = 8;                   // warps
constexpr int kNrThreads = kNrCompute * 32;
constexpr int kNrMaxRbl = 8;                    // row blocks one CTA may touch
static_assert(kNrMaxRbl <= kNrCompute, "one warp sums each row block");
constexpr int kNrMaxUnits = 96;                 // units one CTA may own
constexpr int kNrMaxJ = 64;                     // slice steps per quarter (K <= 32768)
constexpr int kNrPreItems = 4;                  // table items per thread loaded up front
// flags
constexpr int kNrBarBytes = 64;
// the processing order of a CTA's units and its inverse (unit of (rbl, j))
constexpr int kNrOrderBytes = 4 * (kNrMaxUnits + kNrMaxRbl * kNrMaxJ);

struct NarrowParams {
  int N, K, G, mode, epilogue, out_bf16;
  int M;               // tokens (1..MT)
  int n_rb;            // row blocks
  int Q;               // slices per quarter, K / 512
  int spc;             // slices per group, G / 128
  int ng;              // groups per row
  int L;               // groups one quarter may touch (table blocks per row block and item)
  int U;               // units, n_rb * Q
  int P;               // CTAs
  int max_rbl;         // row blocks of the largest CTA share (table layout)
  int max_units;       // units of the largest CTA share (slot layout)
  int tbl_off, x_off, slot_off;   // shared-memory layout (bytes from the base)
  int smem_bytes;
  const uint8_t* packed;          // [N][K*B/8]
  int64_t row_bytes;              // K*B/8
  const float* scales;
  const uint32_t* ab;  // (a | b << 16), fp16 bits
  const uint16_t* x;   // [M][K] bf16
  void* y;
  int64_t ldy;
  int* counter;        // [n_rb] row blocks shared by CTAs (zero between calls)
  float* partial;      // [P][32 lanes][4 * MT/8]: a CTA's part of its first row block
  int counter_len, partial_slots;
  uint64_t timeout_ns;
  unsigned long long* trace;   // optional [P][64] clock64 stamps
};

template <int B>
struct NrCfg {
  static constexpr int E = (B == 3) ? 64 : 16;     // table entries per (row, group)
  static constexpr int SLICE = 16 * B;             // bytes of one row's slice
};

#define NR_STAMP(k)                                                                 \
  do {                                                                              \
    if (p.trace) p.trace[blockIdx.x * 64 + (k)] = clock64();                        \
  } while (0)

// Stream-K partition of the units: CTA c owns [begin(c), begin(c+1)).
__device__ __forceinline__ int nr_begin(int U, int P, int c) {
  return static_cast<int>((static_cast<int64_t>(c) * U) / P);
}
__device__ __forceinline__ int nr_owner(int U, int P, int u) {
  return static_cast<int>((static_cast<int64_t>(u + 1) * P - 1) / U);
}

// Table item id of a CTA (block = id / 32, lane = id % 32): the weight row and
// group its table holds; false when there is none (rows past N, groups past
// the lane column's quarter), whose table is zero.
__device__ __forceinline__ bool nr_item(const NarrowParams& p, int rb_lo, int id, int& row,
                                        int& grp) {
  const int ln = id & 31;
  const int blk = id >> 5;
  const int lgi = blk % p.L;
  const int it = (blk / p.L) & 1;
  const int rb = rb_lo + blk / (2 * p.L);
  const int g = ln >> 2, c = ln & 3;
  row = gv_row(p.N, p.epilogue, rb, it, g);
  grp = (c * p.Q) / p.spc + lgi;
  const int grp_last = ((c + 1) * p.Q - 1) / p.spc;
  return row < p.N && grp <= grp_last && grp < p.ng && rb < p.n_rb;
}

// First group of quarter c and the table block (0..L-1) of slice step j in it.
__device__ __forceinline__ int nr_lgi(int Q, int spc, int c, int j) {
  return (c * Q + j) / spc - (c * Q) / spc;
}

// Output of one lane's D fragment values v (rows g, g+8 x tokens 2c, 2c+1,
// and 8 + those for the second MMA) of row block rb: plain y[m][row], or with
// the SwiGLU epilogue (gate row g, up row g+8) h[m][rb*8 + g].
template <int MT>
__device__ __forceinline__ void nr_store_lane(const NarrowParams& p, int rb, int lane,
                                              const float (&v)[4 * (MT / 8)]) {
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int h = 0; h < MT / 8; ++h) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = 8 * h + 2 * c + e;
      if (m >= p.M) continue;
      const float top = v[h * 4 + e], bot = v[h * 4 + 2 + e];
      if (p.epilogue == CQ_EPI_SWIGLU) {
        const float hv = gv_silu(top) * bot;
        const int64_t off = static_cast<int64_t>(m) * p.ldy + rb * 8 + g;
        if (p.out_bf16)
          reinterpret_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(hv);
        else
          reinterpret_cast<float*>(p.y)[off] = hv;
      } else {
#pragma unroll
        for (int it = 0; it < 2; ++it) {
          const int row = rb * 16 + 8 * it + g;
          if (row >= p.N) continue;
          const int64_t off = static_cast<int64_t>(m) * p.ldy + row;
          const float val = it ? bot : top;
          if (p.out_bf16)
            reinterpret_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(val);
          else
            reinterpret_cast<float*>(p.y)[off] = val;
        }
      }
    }
  }
}

// Sum of row block rb over this CTA's units (slice steps in order), then: a
// row block the CTA holds whole is written out; one shared with the
// following CTAs (this CTA holds its first units and finishes it last: the
// owner) waits for their parts and adds them in CTA order; one shared with
// the preceding CTA (it holds the row block's last units, which it does
// first) parks its part in the workspace and counts it.  One warp; returns
// false when a bounded wait gave up.
template <int MT>
__device__ __noinline__ bool nr_finish_row_block(const NarrowParams& p, int cta, int rb, int u0,
                                                 int u1, int rbl, const int* inv,
                                                 const float* slot_f, int lane,
                                                 volatile int* abort) {
  constexpr int NV = 4 * (MT / 8);
  const int ja = max(u0, rb * p.Q) - rb * p.Q;
  const int jb = min(u1, (rb + 1) * p.Q) - rb * p.Q;
  float v[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) v[k] = 0.f;
  for (int jj = ja; jj < jb; ++jj) {
    const float* src = slot_f + (inv[rbl * kNrMaxJ + jj] * 32 + lane) * NV;
#pragma unroll
    for (int k = 0; k < NV; ++k) v[k] += src[k];
  }
  if (ja == 0 && jb == p.Q) {
    nr_store_lane<MT>(p, rb, lane, v);
    return true;
  }
  const int c_lo = nr_owner(p.U, p.P, rb * p.Q);
  const int c_hi = nr_owner(p.U, p.P, (rb + 1) * p.Q - 1);
  if (rb >= p.counter_len || c_hi >= p.partial_slots) {
    if (lane == 0) atomicCAS(&g_device_error, 0, 42);
    return false;
  }
  if (cta != c_lo) {
    float* dst = p.partial + (static_cast<int64_t>(cta) * 32 + lane) * NV;
#pragma unroll
    for (int k = 0; k < NV; ++k) __stcg(dst + k, v[k]);
    const long long t_f = p.trace ? clock64() : 0;
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(p.counter + rb, 1);
    if (lane == 0 && p.trace) {
      p.trace[blockIdx.x * 64 + 40] = clock64();
      p.trace[blockIdx.x * 64 + 43] = clock64() - t_f;
    }
    return true;
  }
  if (lane == 0 && p.trace) p.trace[blockIdx.x * 64 + 41] = clock64();
  // the owner: the other CTAs did their part of rb first
  bool ok = true;
  if (lane == 0) {
    const volatile int* ctr = p.counter + rb;
    const uint64_t t0 = globaltimer();
    while (*ctr != c_hi - c_lo) {
      if (*abort) {
        ok = false;
        break;
      }
      if (globaltimer() - t0 > p.timeout_ns) {
        *abort = SITE_NR_PARTIAL;
        atomicCAS(&g_device_error, 0, SITE_NR_PARTIAL);
        ok = false;
        break;
      }
      __nanosleep(100);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (lane == 0 && p.trace) p.trace[blockIdx.x * 64 + 42] = clock64();
  if (!ok) return false;
  __threadfence();
  for (int cc = c_lo + 1; cc <= c_hi; ++cc) {
    const float* src = p.partial + (static_cast<int64_t>(cc) * 32 + lane) * NV;
#pragma unroll
    for (int k = 0; k < NV; ++k) v[k] += __ldcg(src + k);
  }
  nr_store_lane<MT>(p, rb, lane, v);
  __syncwarp();
  if (lane == 0) p.counter[rb] = 0;
  return true;
}

// The lane's codes of one unit: rows g (c0) and g+8 (c1) of the row block,
// slice j of quarter c, B 16-byte vectors each, straight from global memory
// (not kept in L1: every byte is read once).  Rows past N read as zero.
template <int B>
__device__ __forceinline__ void nr_load_codes(const NarrowParams& p, int rb, int j, int g, int c,
                                              uint32_t (&c0)[4 * B], uint32_t (&c1)[4 * B]) {
  const int r0 = gv_row(p.N, p.epilogue, rb, 0, g);
  const int r1 = gv_row(p.N, p.epilogue, rb, 1, g);
  const int64_t off = static_cast<int64_t>(c) * (p.row_bytes / 4) + j * (16 * B);
#pragma unroll
  for (int v = 0; v < B; ++v) {
    uint4 q0 = make_uint4(0u, 0u, 0u, 0u), q1 = make_uint4(0u, 0u, 0u, 0u);
    if (r0 < p.N)
      q0 = ldg_stream16(p.packed + static_cast<int64_t>(r0) * p.row_bytes + off + 16 * v);
    if (r1 < p.N)
      q1 = ldg_stream16(p.packed + static_cast<int64_t>(r1) * p.row_bytes + off + 16 * v);
    c0[4 * v + 0] = q0.x;
    c0[4 * v + 1] = q0.y;
    c0[4 * v + 2] = q0.z;
    c0[4 * v + 3] = q0.w;
    c1[4 * v + 0] = q1.x;
    c1[4 * v + 1] = q1.y;
    c1[4 * v + 2] = q1.z;
    c1[4 * v + 3] = q1.w;
  }
}

template <int B, int MT>
__global__ void __launch_bounds__(kNrThreads, 1)
    narrow_kernel(const __grid_constant__ NarrowParams p) {
  using C = NrCfg<B>;
  constexpr int E = C::E;
  constexpr int NV = 4 * (MT / 8);                  // partial floats per lane and unit
  constexpr int NB = B == 4 ? 1 : 2;                // units of codes loaded ahead
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  // the tables are addressed by OR: their base is aligned to a table block
  const uint32_t base = (raw + (E * 128u - 1u)) & ~(E * 128u - 1u);
  uint8_t* const gbase = smem_raw + (base - raw);
  const uint32_t tbl0 = base + p.tbl_off;
  const uint32_t xs0 = base + p.x_off;
  const uint32_t fl = raw + static_cast<uint32_t>(p.smem_bytes - kNrBarBytes - kNrOrderBytes);
  volatile int* const flags = reinterpret_cast<volatile int*>(smem_raw + (fl - raw));
  // order[i] of the CTA's units in processing order: rbl | j << 8;
  // inv[rbl * kNrMaxJ + j] = i
  int* const order = reinterpret_cast<int*>(smem_raw + (fl + kNrBarBytes - raw));
  int* const inv = order + kNrMaxUnits;
  uint32_t* const tblw = reinterpret_cast<uint32_t*>(gbase + p.tbl_off);
  float* const slot_f = reinterpret_cast<float*>(gbase + p.slot_off);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int cta = blockIdx.x;
  const int u0 = nr_begin(p.U, p.P, cta), u1 = nr_begin(p.U, p.P, cta + 1);
  const int n_units = u1 - u0;
  const int rb_lo = u0 / p.Q;
  const int n_rbl = (u1 - 1) / p.Q - rb_lo + 1;

  // ------------------------------------------------------------------ setup
  if (tid == 0) {
    NR_STAMP(0);
    griddep_launch_dependents();
    int bad = 0;
    if (n_units < 1 || n_units > p.max_units || n_units > kNrMaxUnits || n_rbl > p.max_rbl ||
        n_rbl > kNrMaxRbl || p.Q > kNrMaxJ || p.M < 1 || p.M > MT)
      bad = 40;
    // processing order: row block by row block
    int i = 0;
    for (int rbl = 0; rbl < n_rbl && !bad; ++rbl) {
      for (int j = 0; j < p.Q; ++j) {
        const int u = (rb_lo + rbl) * p.Q + j;
        if (u >= u0 && u < u1) {
          inv[rbl * kNrMaxJ + j] = i;
          order[i++] = rbl | (j << 8);
        }
      }
    }
    if (!bad && i != n_units) bad = 41;
    flags[0] = bad;
    flags[2] = 0;          // abort: a bounded wait gave up
    if (bad) atomicCAS(&g_device_error, 0, bad);
  }
  __syncthreads();
  // programmatic dependent launch: nothing written by the preceding grid is
  // read (and nothing is written) before this returns
  griddep_wait();
  if (tid == 0) NR_STAMP(4);
  if (flags[0]) return;
  // the rows of this CTA's row blocks, brought into L2 in a few bulk
  // prefetches: the lanes' 16-byte code loads then hit L2
  if (warp == 0 && lane < n_rbl * 2) {
    const int rb = rb_lo + (lane >> 1), half = lane & 1;
    if (rb < p.n_rb) {
      int r0, nrows;
      if (p.epilogue == CQ_EPI_SWIGLU) {
        r0 = (half ? (p.N >> 1) : 0) + rb * 8;
        nrows = 8;
      } else {
        r0 = rb * 16 + half * 8;
        nrows = min(8, p.N - r0);
      }
      if (nrows > 0) {
        const int64_t bytes = static_cast<int64_t>(nrows) * p.row_bytes;
        const uint8_t* src = p.packed + static_cast<int64_t>(r0) * p.row_bytes;
        for (int64_t o = 0; o < bytes; o += (1 << 20)) {
          const int64_t n = bytes - o < (1 << 20) ? bytes - o : (1 << 20);
          prefetch_l2_bulk(src + o, static_cast<uint32_t>(n));
        }
      }
    }
  }

  // -------------------------------------------------------- level tables
  // block (rbl, it, lgi) holds the tables of lanes (g, c) = rows (rb, it, g)
  // x groups (first group of quarter c) + lgi, entry e of lane l at word
  // (block * E + e) * 32 + l.  The group parameters go out first, before
  // the bulk of the loads, so that the tables are not held up behind them.
    const int n_items = n_rbl * 2 * p.L * 32;
    float s_pre[kNrPreItems];
    uint32_t ab_pre[kNrPreItems];
#pragma unroll
    for (int k = 0; k < kNrPreItems; ++k) {
      s_pre[k] = 0.f;
      ab_pre[k] = 0u;
      const int id = tid + k * kNrThreads;
      int row, grp;
      if (id < n_items && nr_item(p, rb_lo, id, row, grp)) {
        const int64_t mi = static_cast<int64_t>(row) * p.ng + grp;
        s_pre[k] = __uint_as_float(ldg_u32_ordered(p.scales + mi));
        ab_pre[k] = ldg_u32_ordered(p.ab + mi);
      }
    }

  // ------------------------------------------------------- activations
  // every slice step's activations, as 16-byte chunks (j, s'', m, c)
  {
    const int n_chunks = p.Q * 16 * p.M * 4;
    for (int ch = tid; ch < n_chunks; ch += kNrThreads) {
      const int cq = ch & 3;
      const int m = (ch >> 2) % p.M;
      const int js = (ch >> 2) / p.M;                   // j * 16 + s''
      const int j = js >> 4, s2 = js & 15;
      const uint16_t* src =
          p.x + static_cast<int64_t>(m) * p.K + cq * (p.K / 4) + j * 128 + s2 * 8;
      cp_async16(xs0 + ch * 16, src);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  {
    for (int k = 0, id = tid; id < n_items; ++k, id += kNrThreads) {
      const int ln = id & 31;
      const int blk = id >> 5;
      int row, grp;
      const bool valid = nr_item(p, rb_lo, id, row, grp);
      float s = 0.f;
      uint32_t abw = 0u;
      if (k < kNrPreItems) {
#pragma unroll
        for (int kk = 0; kk < kNrPreItems; ++kk)
          if (kk == k) {
            s = s_pre[kk];
            abw = ab_pre[kk];
          }
      } else if (valid) {
        const int64_t mi = static_cast<int64_t>(row) * p.ng + grp;
        s = __ldg(p.scales + mi);
        abw = __ldg(p.ab + mi);
      }
      uint32_t Lv[1 << B];
      gv_levels<B>(valid, s, abw, p.mode, Lv);
      uint32_t* const tb = tblw + blk * (E * 32) + ln;
      if constexpr (B == 4) {
#pragma unroll
        for (int e = 0; e < 16; ++e) tb[e * 32] = Lv[e] | (Lv[e] << 16);
      } else {
        constexpr int NL = 1 << B;
#pragma unroll
        for (int e = 0; e < E; ++e) tb[e * 32] = Lv[e & (NL - 1)] | (Lv[e / NL] << 16);
      }
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (tid == 0) NR_STAMP(2);
  // codes of this warp's first units (registers).  From here to the end of
  // the units no fence or barrier is passed: either would wait for these
  // loads, and for the ones issued NB units ahead inside the loop.
  uint32_t cn0[NB][4 * B], cn1[NB][4 * B];
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    const int i = warp + k * kNrCompute;
#pragma unroll
    for (int w = 0; w < 4 * B; ++w) cn0[k][w] = cn1[k][w] = 0u;
    if (i < n_units) {
      const int ord = order[i];
      nr_load_codes<B>(p, rb_lo + (ord & 255), ord >> 8, g, c, cn0[k], cn1[k]);
    }
  }


  // ------------------------------------------------------------ the units
  long long cyc_work = 0;
  if (p.trace && lane == 0) p.trace[blockIdx.x * 64 + 44 + warp] = clock64();
  for (int i = warp; i < n_units; i += kNrCompute) {
    const long long t_a = p.trace ? clock64() : 0;
    const int ord = order[i];
    const int rbl = ord & 255, j = ord >> 8;
    // this unit's codes; the warp's unit NB ahead goes into the freed buffer
    uint32_t c0[4 * B], c1[4 * B];
#pragma unroll
    for (int w = 0; w < 4 * B; ++w) {
      c0[w] = cn0[0][w];
      c1[w] = cn1[0][w];
    }
#pragma unroll
    for (int kb = 0; kb + 1 < NB; ++kb)
#pragma unroll
      for (int w = 0; w < 4 * B; ++w) {
        cn0[kb][w] = cn0[kb + 1][w];
        cn1[kb][w] = cn1[kb + 1][w];
      }
    {
      const int ia = i + NB * kNrCompute;
      if (ia < n_units) {
        const int oa = order[ia];
        nr_load_codes<B>(p, rb_lo + (oa & 255), oa >> 8, g, c, cn0[NB - 1], cn1[NB - 1]);
      }
    }
    const int lgi = nr_lgi(p.Q, p.spc, c, j);
    const uint32_t blk0 = static_cast<uint32_t>(((rbl * 2 + 0) * p.L + lgi) * E * 128);
    const uint32_t blk1 = static_cast<uint32_t>(((rbl * 2 + 1) * p.L + lgi) * E * 128);
    const uint32_t tl0 = tbl0 + blk0 + lane * 4;
    const uint32_t tl1 = tbl0 + blk1 + lane * 4;
    // activations: [j][k pair s''][token][quarter][8 values]
    const uint32_t xa = xs0 + j * p.M * 1024 + (g * 4 + c) * 16;
    const uint32_t xstride = static_cast<uint32_t>(p.M) * 64u;
    const bool xl0 = g < p.M;
    const bool xl1 = MT == 16 && g + 8 < p.M;
    float acc[2][MT / 8][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int h = 0; h < MT / 8; ++h)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][h][b] = 0.f;
    // software-pipelined: the lookups of MMA step s+2 and the activations of
    // the next k pair are issued before the MMA of step s
    uint4 xv0 = make_uint4(0u, 0u, 0u, 0u), xv1 = make_uint4(0u, 0u, 0u, 0u);
    uint4 xn0 = xv0, xn1 = xv1;
    if (xl0) xv0 = lds128(xa);
    if (MT == 16 && xl1) xv1 = lds128(xa + 8 * 64);
    uint32_t a[3][4];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      a[s][0] = gv_pair<B>(c0, 2 * s, tl0);
      a[s][1] = gv_pair<B>(c1, 2 * s, tl1);
      a[s][2] = gv_pair<B>(c0, 2 * s + 1, tl0);
      a[s][3] = gv_pair<B>(c1, 2 * s + 1, tl1);
    }
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2) {
      if (s2 + 1 < 16) {
        if (xl0) xn0 = lds128(xa + (s2 + 1) * xstride);
        if (MT == 16 && xl1) xn1 = lds128(xa + (s2 + 1) * xstride + 8 * 64);
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int s = 2 * s2 + h2;          // MMA step: codes 4s .. 4s+3
        if (s + 2 < 32) {
          const int sn = s + 2;
          a[sn % 3][0] = gv_pair<B>(c0, 2 * sn, tl0);
          a[sn % 3][1] = gv_pair<B>(c1, 2 * sn, tl1);
          a[sn % 3][2] = gv_pair<B>(c0, 2 * sn + 1, tl0);
          a[sn % 3][3] = gv_pair<B>(c1, 2 * sn + 1, tl1);
        }
        const uint32_t* as = a[s % 3];
        const uint32_t b0 = h2 ? xv0.z : xv0.x, b1 = h2 ? xv0.w : xv0.y;
        mma_16816_bf16(acc[h2][0], as[0], as[1], as[2], as[3], b0, b1);
        if constexpr (MT == 16) {
          const uint32_t e0 = h2 ? xv1.z : xv1.x, e1 = h2 ? xv1.w : xv1.y;
          mma_16816_bf16(acc[h2][1], as[0], as[1], as[2], as[3], e0, e1);
        }
      }
      xv0 = xn0;
      xv1 = xn1;
    }
    // the unit's partial sums: [unit][lane][NV]
    float* const sl = slot_f + (i * 32 + lane) * NV;
#pragma unroll
    for (int h = 0; h < MT / 8; ++h)
#pragma unroll
      for (int b = 0; b < 4; ++b) sl[h * 4 + b] = acc[0][h][b] + acc[1][h][b];
    if (p.trace) cyc_work += clock64() - t_a;
  }
  // ------------------------------------------------------- the row blocks
  // every unit is in its slot; warp rbl sums row block rbl (a row block
  // shared with the next CTA waits for that CTA's part, which it publishes
  // here too, after its own units: no CTA waits before publishing)
  __syncthreads();
  const long long t_c = p.trace ? clock64() : 0;
  if (warp < n_rbl)   // a wait that gives up sets the error flag itself
    nr_finish_row_block<MT>(p, cta, rb_lo + warp, u0, u1, warp, inv, slot_f, lane, flags + 2);
  if (p.trace && lane == 0) {
    p.trace[blockIdx.x * 64 + 52 + warp] = t_c;
    p.trace[blockIdx.x * 64 + 8 + 3 * warp] = 0;
    p.trace[blockIdx.x * 64 + 9 + 3 * warp] = cyc_work;
    p.trace[blockIdx.x * 64 + 10 + 3 * warp] = clock64() - t_c;
  }
  __syncthreads();
  if (tid == 0) NR_STAMP(1);
}

}  // namespace cq
