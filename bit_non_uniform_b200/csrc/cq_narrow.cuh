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
// CTA builds the level tables of every (row, group) its units touch while its
// first loads are in flight; its warps then take the units round robin, row
// block by row block when every slice step's activations fit in shared
// memory (else slice step by slice step, through a ring of activation
// stages).  A unit's partial sums go to a shared-memory slot; the warp that
// finishes a row block's last unit sums the row block's slots (slice steps
// in order) and writes it out.  A row block shared by consecutive CTAs is
// finished early by the later ones (it is the first row block they do),
// which park their parts in the workspace; the first CTA (the owner, which
// does it last) adds them in CTA order.  Results are run-to-run
// deterministic.
//
// Roles: eight compute warps (tables, decode + MMA, sums, epilogue) and one
// producer warp whose first lane keeps two TMA rings full: code stages (one
// unit each, a 3-D/4-D box of 16 rows x 4 quarters x one slice) and
// activation stages (one slice step of every token, a 4-D box that lands
// interleaved as [k pair][token][quarter][8 values], so a warp's 16-byte
// activation loads are conflict free).
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

constexpr int kNrCompute = 8;                   // compute warps
constexpr int kNrProducerWarp = 8;
constexpr int kNrThreads = (kNrCompute + 1) * 32;
constexpr int kNrMaxRbl = 8;                    // row blocks one CTA may touch
constexpr int kNrMaxUnits = 96;                 // units one CTA may own
constexpr int kNrMaxJ = 64;                     // slice steps per quarter (K <= 32768)
constexpr int kNrMaxCS = 96;                    // code stages
constexpr int kNrMaxXS = 64;                    // activation stages
// barriers, flags, the issue tags of the two rings, and per row block the
// units of the CTA and how many of them are done
constexpr int kNrBarBytes =
    8 * (2 * kNrMaxCS + 2 * kNrMaxXS) + 64 + 4 * (kNrMaxCS + kNrMaxXS) + 8 * kNrMaxRbl;
// the processing order of a CTA's units, its inverse (unit of (rbl, j)) and
// the slice step of each activation stage
constexpr int kNrOrderBytes = 4 * (kNrMaxUnits + kNrMaxRbl * kNrMaxJ + kNrMaxXS);

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
  int CS, XS;          // code / activation stages
  int resident_x;      // 1: every slice step's activations stay loaded (XS = Q)
  int tbl_off, code_off, x_off, slot_off;   // shared-memory layout (bytes from the base)
  int smem_bytes;
  const float* scales;
  const uint32_t* ab;  // (a | b << 16), fp16 bits
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
  static constexpr int STAGE = 16 * 4 * SLICE;     // one unit's codes
};

// Wait (bounded) until a ring stage's issue tag shows `use`: the producer
// writes the tag when it issues that use into the stage, after the stage's
// previous use has landed and been released.  A consumer then waits on the
// stage's full barrier with the parity of `use` knowing that the barrier's
// pending phase is exactly that use (a parity wait alone cannot tell phases
// two apart, and a consumer may reach its unit before the stage's previous
// use has even landed).
__device__ __forceinline__ bool nr_wait_tag(const volatile int* tag, int use, volatile int* abort,
                                            uint64_t timeout_ns, int site) {
  if (*tag == use) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    __nanosleep(64);
    if (*tag == use) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > timeout_ns) {
      *abort = site;
      atomicCAS(&g_device_error, 0, site);
      return false;
    }
  }
}

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
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(p.counter + rb, 1);
    return true;
  }
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

template <int B, int MT>
__global__ void __launch_bounds__(kNrThreads, 1)
    narrow_kernel(const __grid_constant__ NarrowParams p,
                  const __grid_constant__ CUtensorMap wmap,
                  const __grid_constant__ CUtensorMap xmap) {
  using C = NrCfg<B>;
  constexpr int E = C::E;
  constexpr int NV = 4 * (MT / 8);                  // partial floats per lane and unit
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  // the tables are addressed by OR: their base is aligned to a table block
  const uint32_t base = (raw + (E * 128u - 1u)) & ~(E * 128u - 1u);
  uint8_t* const gbase = smem_raw + (base - raw);
  const uint32_t tbl0 = base + p.tbl_off;
  const uint32_t codes0 = base + p.code_off;
  const uint32_t xs0 = base + p.x_off;
  const uint32_t bars = raw + static_cast<uint32_t>(p.smem_bytes - kNrBarBytes - kNrOrderBytes);
  const uint32_t bar_cfull = bars;                           // [CS]
  const uint32_t bar_cempty = bar_cfull + 8 * kNrMaxCS;      // [CS]
  const uint32_t bar_xfull = bar_cempty + 8 * kNrMaxCS;      // [XS]
  const uint32_t bar_xempty = bar_xfull + 8 * kNrMaxXS;      // [XS]
  volatile int* const flags =
      reinterpret_cast<volatile int*>(smem_raw + (bar_xempty + 8 * kNrMaxXS - raw));
  volatile int* const ctag = flags + 16;                    // [CS] unit issued into a code stage
  volatile int* const xtag = ctag + kNrMaxCS;               // [XS] use issued into an x stage
  int* const cnt_rb = const_cast<int*>(xtag + kNrMaxXS);    // [rbl] the CTA's units of it
  int* const done_rb = cnt_rb + kNrMaxRbl;                  // [rbl] of those, finished
  // order[i] of the CTA's units in processing order: rbl | j << 8 | t << 16
  // (t = rank of j among the CTA's slice steps, the activation stage use);
  // inv[rbl * kNrMaxJ + j] = i; jsel[t] = j
  int* const order = reinterpret_cast<int*>(smem_raw + (bars + kNrBarBytes - raw));
  int* const inv = order + kNrMaxUnits;
  int* const jsel = inv + kNrMaxRbl * kNrMaxJ;
  uint32_t* const tblw = reinterpret_cast<uint32_t*>(gbase + p.tbl_off);
  float* const slot_f = reinterpret_cast<float*>(gbase + p.slot_off);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint64_t tmo = p.timeout_ns;
  const int cta = blockIdx.x;
  const int u0 = nr_begin(p.U, p.P, cta), u1 = nr_begin(p.U, p.P, cta + 1);
  const int n_units = u1 - u0;
  const int rb_lo = u0 / p.Q;
  const int n_rbl = (u1 - 1) / p.Q - rb_lo + 1;

  // ------------------------------------------------------------------ setup
  if (tid == 0) {
    NR_STAMP(0);
    griddep_launch_dependents();
    for (int s = 0; s < p.CS; ++s) {
      mbar_init(bar_cfull + 8 * s, 1);
      mbar_init(bar_cempty + 8 * s, 1);
      ctag[s] = -1;
    }
    for (int s = 0; s < p.XS; ++s) {
      mbar_init(bar_xfull + 8 * s, 1);
      mbar_init(bar_xempty + 8 * s, kNrMaxRbl);
      xtag[s] = -1;
    }
    int bad = 0;
    if (n_units < 1 || n_units > p.max_units || n_units > kNrMaxUnits || n_rbl > p.max_rbl ||
        n_rbl > kNrMaxRbl || p.Q > kNrMaxJ || p.CS > kNrMaxCS || p.XS > kNrMaxXS || p.CS < 1 ||
        p.XS < 1 || p.M < 1 || p.M > MT)
      bad = 40;
    // slice steps present in this CTA, in order: their rank is the
    // activation stage use
    int t = 0;
    int jrank[kNrMaxJ];
    for (int j = 0; j < p.Q && !bad; ++j) {
      bool any = false;
      for (int rbl = 0; rbl < n_rbl; ++rbl) {
        const int u = (rb_lo + rbl) * p.Q + j;
        any = any || (u >= u0 && u < u1);
      }
      jrank[j] = any ? t : -1;
      if (any) jsel[t++] = j;
    }
    if (p.resident_x && t > p.XS) bad = 44;
    for (int rbl = 0; rbl < n_rbl && !bad; ++rbl) {
      cnt_rb[rbl] = 0;
      done_rb[rbl] = 0;
    }
    // processing order: with every activation stage resident, row block by
    // row block (a row block shared with the previous CTA comes first and
    // is finished early); else slice step by slice step
    int i = 0;
    for (int a = 0; a < (p.resident_x ? n_rbl : p.Q) && !bad; ++a) {
      for (int b = 0; b < (p.resident_x ? p.Q : n_rbl); ++b) {
        const int rbl = p.resident_x ? a : b, j = p.resident_x ? b : a;
        const int u = (rb_lo + rbl) * p.Q + j;
        if (u >= u0 && u < u1) {
          inv[rbl * kNrMaxJ + j] = i;
          order[i++] = rbl | (j << 8) | (jrank[j] << 16);
          ++cnt_rb[rbl];
        }
      }
    }
    if (!bad && i != n_units) bad = 41;
    flags[0] = bad;
    flags[1] = t;          // slice steps of this CTA
    flags[2] = 0;          // abort: a bounded wait gave up
    if (bad) atomicCAS(&g_device_error, 0, bad);
    fence_mbar_init();
  }
  __syncthreads();
  // programmatic dependent launch: nothing written by the preceding grid is
  // read (and nothing is written) before this returns
  griddep_wait();
  if (tid == 0) NR_STAMP(4);
  if (flags[0]) return;
  const int n_j = flags[1];

  int issued_c = 0, issued_x = 0;           // producer: copies issued so far
  if (warp == kNrProducerWarp) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&wmap);
      prefetch_tensormap(&xmap);
      bool ok = true;
      if (p.resident_x) {
        // every slice step's activations, once
        for (int t = 0; t < n_j; ++t) {
          xtag[t] = t;
          mbar_arrive_expect_tx(bar_xfull + 8 * t, static_cast<uint32_t>(p.M) * 1024u);
          tma_load_4d(xs0 + t * p.M * 1024, &xmap, 0, 0, 0, jsel[t] * 16, bar_xfull + 8 * t);
          ++issued_x;
        }
      }
      int t_next = 0;                       // ring mode: next activation use to load
      for (int i = 0; i < n_units && ok; ++i) {
        const int ord = order[i];
        const int rbl = ord & 255, j = (ord >> 8) & 255, t = ord >> 16;
        if (!p.resident_x && t == t_next) {
          // the activation stage of slice step j: the units of this step release it
          const int xs = t % p.XS;
          if (!gv_wait(bar_xempty + 8 * xs, ((t / p.XS) & 1) ^ 1, flags + 2, tmo,
                       SITE_NR_XEMPTY)) {
            ok = false;
            break;
          }
          int cnt = 0;
          for (int r = 0; r < n_rbl; ++r) {
            const int u = (rb_lo + r) * p.Q + j;
            cnt += (u >= u0 && u < u1) ? 1 : 0;
          }
          // arrivals of the units that will not use this stage
          if (kNrMaxRbl - cnt > 0) mbar_arrive_cnt(bar_xempty + 8 * xs, kNrMaxRbl - cnt);
          xtag[xs] = t;
          mbar_arrive_expect_tx(bar_xfull + 8 * xs, static_cast<uint32_t>(p.M) * 1024u);
          tma_load_4d(xs0 + xs * p.M * 1024, &xmap, 0, 0, 0, j * 16, bar_xfull + 8 * xs);
          ++t_next;
          ++issued_x;
        }
        const int cs = i % p.CS;
        if (!gv_wait(bar_cempty + 8 * cs, ((i / p.CS) & 1) ^ 1, flags + 2, tmo,
                     SITE_NR_CEMPTY)) {
          ok = false;
          break;
        }
        ctag[cs] = i;
        mbar_arrive_expect_tx(bar_cfull + 8 * cs, static_cast<uint32_t>(C::STAGE));
        const int rb = rb_lo + rbl;
        if (p.epilogue == CQ_EPI_SWIGLU)
          tma_load_4d(codes0 + cs * C::STAGE, &wmap, j * C::SLICE, 0, rb * 8, 0,
                      bar_cfull + 8 * cs);
        else
          tma_load_3d(codes0 + cs * C::STAGE, &wmap, j * C::SLICE, 0, rb * 16,
                      bar_cfull + 8 * cs);
        ++issued_c;
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- compute warps
    // level tables: block (rbl, it, lgi) holds the tables of lanes (g, c) =
    // rows (rb, it, g) x groups (first group of quarter c) + lgi, entry e of
    // lane l at word (block * E + e) * 32 + l
    const int n_items = n_rbl * 2 * p.L * 32;
    for (int id = tid; id < n_items; id += kNrCompute * 32) {
      const int ln = id & 31;
      const int blk = id >> 5;
      const int lgi = blk % p.L;
      const int it = (blk / p.L) & 1;
      const int rbl = blk / (2 * p.L);
      const int g = ln >> 2, c = ln & 3;
      const int rb = rb_lo + rbl;
      const int row = gv_row(p.N, p.epilogue, rb, it, g);
      const int grp = (c * p.Q) / p.spc + lgi;
      const int grp_last = ((c + 1) * p.Q - 1) / p.spc;
      const bool valid = row < p.N && grp <= grp_last && grp < p.ng && rb < p.n_rb;
      float s = 0.f;
      uint32_t abw = 0u;
      if (valid) {
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
    asm volatile("bar.sync 1, %0;" ::"n"(kNrCompute * 32) : "memory");
    if (tid == 0) NR_STAMP(2);

    const int g = lane >> 2, c = lane & 3;
    // 16-byte chunk order of the code reads (keeps them conflict free)
    const int rot = B == 2 ? (g & 1) : (B == 4 ? (g & 1) + 2 * (c >> 1) : 0);
    long long cyc_wait = 0, cyc_work = 0, cyc_fin = 0;
    bool ok = true;
    for (int i = warp; i < n_units && ok; i += kNrCompute) {
      const long long t_a = p.trace ? clock64() : 0;
      const int ord = order[i];
      const int rbl = ord & 255, j = (ord >> 8) & 255, t = ord >> 16;
      const int cs = i % p.CS, xs = t % p.XS;
      const bool tag_ok = nr_wait_tag(ctag + cs, i, flags + 2, tmo, SITE_NR_CFULL);
      if (!__all_sync(0xffffffffu, tag_ok) ||
          !gv_wait_warp(bar_cfull + 8 * cs, (i / p.CS) & 1, flags + 2, tmo, SITE_NR_CFULL)) {
        ok = false;
        break;
      }
      // the lane's two rows (g, g+8) of slice j of quarter c
      const uint32_t cb = codes0 + cs * C::STAGE + (g * 4 + c) * C::SLICE;
      uint32_t c0[4 * B], c1[4 * B];
#pragma unroll
      for (int v = 0; v < B; ++v) {
        int vv = v + rot;
        while (vv >= B) vv -= B;
        const uint4 q0 = lds128(cb + 16 * vv);
        const uint4 q1 = lds128(cb + 32 * C::SLICE + 16 * vv);
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
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_cempty + 8 * cs);
      const bool xtag_ok = nr_wait_tag(xtag + xs, t, flags + 2, tmo, SITE_NR_XFULL);
      if (!__all_sync(0xffffffffu, xtag_ok) ||
          !gv_wait_warp(bar_xfull + 8 * xs, (t / p.XS) & 1, flags + 2, tmo, SITE_NR_XFULL)) {
        ok = false;
        break;
      }
      const long long t_b = p.trace ? clock64() : 0;
      const int lgi = nr_lgi(p.Q, p.spc, c, j);
      const uint32_t blk0 = static_cast<uint32_t>(((rbl * 2 + 0) * p.L + lgi) * E * 128);
      const uint32_t blk1 = static_cast<uint32_t>(((rbl * 2 + 1) * p.L + lgi) * E * 128);
      const uint32_t tl0 = tbl0 + blk0 + lane * 4;
      const uint32_t tl1 = tbl0 + blk1 + lane * 4;
      // activations: [k pair s''][token][quarter][8 values]
      const uint32_t xa = xs0 + xs * p.M * 1024 + (g * 4 + c) * 16;
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
      uint4 xv0 = make_uint4(0u, 0u, 0u, 0u), xv1 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int s2 = 0; s2 < 16; ++s2) {
        if (xl0) xv0 = lds128(xa + s2 * xstride);
        if (MT == 16 && xl1) xv1 = lds128(xa + s2 * xstride + 8 * 64);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int s = 2 * s2 + h2;          // MMA step: codes 4s .. 4s+3
          const uint32_t a0 = gv_pair<B>(c0, 2 * s, tl0);
          const uint32_t a1 = gv_pair<B>(c1, 2 * s, tl1);
          const uint32_t a2 = gv_pair<B>(c0, 2 * s + 1, tl0);
          const uint32_t a3 = gv_pair<B>(c1, 2 * s + 1, tl1);
          const uint32_t b0 = h2 ? xv0.z : xv0.x, b1 = h2 ? xv0.w : xv0.y;
          mma_16816_bf16(acc[h2][0], a0, a1, a2, a3, b0, b1);
          if constexpr (MT == 16) {
            const uint32_t e0 = h2 ? xv1.z : xv1.x, e1 = h2 ? xv1.w : xv1.y;
            mma_16816_bf16(acc[h2][1], a0, a1, a2, a3, e0, e1);
          }
        }
      }
      __syncwarp();
      if (!p.resident_x && lane == 0) mbar_arrive(bar_xempty + 8 * xs);
      // the unit's partial sums: [unit][lane][NV]
      float* const sl = slot_f + (i * 32 + lane) * NV;
#pragma unroll
      for (int h = 0; h < MT / 8; ++h)
#pragma unroll
        for (int b = 0; b < 4; ++b) sl[h * 4 + b] = acc[0][h][b] + acc[1][h][b];
      // the warp that finishes a row block's last unit in this CTA sums it
      __threadfence_block();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = atomicAdd(done_rb + rbl, 1) + 1 == cnt_rb[rbl];
      last = __shfl_sync(0xffffffffu, last, 0);
      const long long t_c = p.trace ? clock64() : 0;
      if (last) {
        __threadfence_block();
        if (!nr_finish_row_block<MT>(p, cta, rb_lo + rbl, u0, u1, rbl, inv, slot_f, lane,
                                     flags + 2))
          ok = false;
      }
      if (p.trace) {
        const long long t_d = clock64();
        cyc_wait += t_b - t_a;
        cyc_work += t_c - t_b;
        cyc_fin += t_d - t_c;
      }
    }
    if (p.trace && lane == 0) {
      p.trace[blockIdx.x * 64 + 8 + 3 * warp] = cyc_wait;
      p.trace[blockIdx.x * 64 + 9 + 3 * warp] = cyc_work;
      p.trace[blockIdx.x * 64 + 10 + 3 * warp] = cyc_fin;
    }
  }
  __syncthreads();
  if (tid == 0) NR_STAMP(1);
  if (flags[2]) {
    // a wait gave up: no copy may still be landing in shared memory at exit
    if (warp == kNrProducerWarp && lane == 0) {
      volatile int dummy = 0;
      for (int k = 1; k <= issued_c && k <= p.CS; ++k) {
        const int i = issued_c - k;
        mbar_wait(bar_cfull + 8 * (i % p.CS), (i / p.CS) & 1, &dummy, tmo, SITE_TEARDOWN);
      }
      const int xk = p.resident_x ? issued_x : (issued_x < p.XS ? issued_x : p.XS);
      for (int k = 1; k <= xk; ++k) {
        const int t = issued_x - k;
        mbar_wait(bar_xfull + 8 * (t % p.XS), (t / p.XS) & 1, &dummy, tmo, SITE_TEARDOWN);
      }
    }
    __syncthreads();
  }
}

}  // namespace cq
