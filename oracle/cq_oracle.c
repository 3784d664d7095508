/*
 * cq_oracle.c -- CPU reference ("oracle") for CubicQuant weight-only GEMM.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It is deliberately plain and slow: FP64
 * arithmetic, naive loops, no blocking, no reordering of any sum beyond the
 * definitions below.  It shares no code with the CUDA library.
 *
 * Source of the method: the ModelScope article "CubicQuant：用三次曲线重塑低
 * 比特量化，Kimi K3 2.5Bit 模型首发实践" (cited below as [CQ]), sections
 *   [CQ core]    "CubicQuant 核心：把直线网格“掰弯”"   (format and decode)
 *   [CQ two]     "为什么只用两个形状参数？"              (dense code stream)
 *   [CQ bits]    "存储开销是透明的：B+64/G bit"          (storage identity)
 *   [CQ fit]     "从曲线到量化器：数据无关的组内拟合"     (group fitter)
 *   [CQ fused]   "压缩权重必须“边解码、边计算”"          (A16 execution)
 *   [CQ a8]      "一份 checkpoint，同时服务 A16 与 Dynamic A8" (A8 mode)
 *
 * The article's displayed formulas were lost when the page was extracted;
 * the readings used here are:
 *   - code u in [0, 2^B-1], MIDRISE grid (the build contract):
 *       Kc = (2^B-1)/2, k = u - Kc, t = |k|/Kc, sign(k) never 0;
 *   - MIDTREAD grid (sign-magnitude alternative, also supported):
 *       Kc = 2^(B-1)-1, k = u - Kc, t = |k|/Kc, sign(0) = 0; the formula is
 *       applied as written to every code, including the unused 2^B-1;
 *   - q(t) = a t + b t^2 + c t^3 with c = 1 - a - b  [CQ core];
 *   - w = s * sign(k) * q(t), s FP32, a and b FP16  [CQ core];
 *   - codes are packed LSB-first: code k of a row occupies bits
 *     [k*B, k*B+B) of the row's byte stream, bit j in byte j/8 at bit j%8
 *     (the article only says "dense, contiguous"  [CQ two]);
 *   - groups are G consecutive elements along K inside one row; scales are
 *     float32 [N][K/G]; ab is fp16 [N][K/G][2] holding (a, b);
 *   - Dynamic A8 (its formulas were lost as well): the weight carrier of
 *     code u is RNE(127 * sign(k) * q(t)) on the symmetric INT8 grid; each
 *     activation row is quantized by its own absmax (x -> RNE(127 x /
 *     absmax)); the integer dot product of a group is scaled by
 *     (absmax / 127) * (s / 127); the joint fit minimises L_C + lambda *
 *     L_A8 with the codes of the nearest continuous level.
 *
 * The end of the file evaluates [CQ two]'s error bound (Lloyd-Max <= Cubic
 * <= best clipped INT) on the Gaussian and Laplace densities themselves.
 *
 * Parity pins for every function are in tests/test_oracle_*.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define CQO_MIDRISE 0
#define CQO_MIDTREAD 1

/* ------------------------------------------------------------------------ */
/* IEEE number helpers (written from the binary16 / bfloat16 definitions)    */
/* ------------------------------------------------------------------------ */

/* binary16 bit pattern -> exact double. */
double cqo_half_to_double(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);              /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);  /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* double -> binary16 bit pattern, round to nearest, ties to even. */
uint16_t cqo_double_to_half(double x)
{
    uint16_t sign = (uint16_t)(signbit(x) ? 0x8000 : 0);
    double ax = fabs(x);
    if (isnan(x))
        return 0x7e00;
    if (ax >= 65520.0)                           /* rounds to infinity */
        return sign | 0x7c00;
    if (ax < ldexp(1.0, -14)) {                  /* subnormal range, unit 2^-24 */
        double q = ax * 16777216.0;              /* exact scaling by 2^24 */
        double r = nearbyint(q);                 /* default mode: ties to even */
        return sign | (uint16_t)r;               /* r == 1024 gives min normal */
    }
    int e;
    double f = frexp(ax, &e);                    /* ax = f * 2^e, f in [0.5,1) */
    /* significand with 11 bits: ax = M * 2^(e-11), M in [1024, 2048) */
    double M = nearbyint(ldexp(f, 11));
    if (M == 2048.0) { M = 1024.0; e += 1; }
    int E = e - 1 + 15;                          /* biased exponent */
    if (E >= 31)
        return sign | 0x7c00;
    return sign | (uint16_t)(E << 10) | (uint16_t)((int)M - 1024);
}

/* float -> bfloat16 bit pattern, round to nearest, ties to even. */
uint16_t cqo_float_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return 0x7fc0;                           /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

double cqo_bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Bit stream  [CQ two]: dense B-bit codes, LSB-first inside each row         */
/* ------------------------------------------------------------------------ */

/* codes[N][K] (one code per byte, each < 2^B) -> packed[N][K*B/8]. */
void cqo_pack(const uint8_t *codes, int64_t N, int64_t K, int B, uint8_t *packed)
{
    int64_t row_bytes = K * B / 8;
    memset(packed, 0, (size_t)(N * row_bytes));
    for (int64_t n = 0; n < N; n++) {
        uint8_t *dst = packed + n * row_bytes;
        for (int64_t k = 0; k < K; k++) {
            unsigned u = codes[n * K + k];
            for (int j = 0; j < B; j++) {
                int64_t bit = k * B + j;
                if ((u >> j) & 1u)
                    dst[bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
        }
    }
}

/* packed[N][K*B/8] -> codes[N][K]. */
void cqo_unpack(const uint8_t *packed, int64_t N, int64_t K, int B, uint8_t *codes)
{
    int64_t row_bytes = K * B / 8;
    for (int64_t n = 0; n < N; n++) {
        const uint8_t *src = packed + n * row_bytes;
        for (int64_t k = 0; k < K; k++) {
            unsigned u = 0;
            for (int j = 0; j < B; j++) {
                int64_t bit = k * B + j;
                u |= (unsigned)((src[bit / 8] >> (bit % 8)) & 1u) << j;
            }
            codes[n * K + k] = (uint8_t)u;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Level math  [CQ core]                                                     */
/* ------------------------------------------------------------------------ */

/* Signed coordinate of code u: returns sign(k) in {-1,0,+1} and t = |k|/Kc. */
void cqo_coord(int u, int B, int mode, int *sign, double *t)
{
    if (mode == CQO_MIDRISE) {
        double Kc = ((1 << B) - 1) / 2.0;        /* half-integer half-range */
        double k = (double)u - Kc;               /* never zero */
        *sign = k > 0 ? 1 : -1;
        *t = fabs(k) / Kc;
    } else {
        int Kc = (1 << (B - 1)) - 1;
        int k = u - Kc;
        *sign = (k > 0) - (k < 0);
        *t = (double)abs(k) / (double)Kc;
    }
}

/* q(t) = a t + b t^2 + c t^3, c = 1 - a - b, evaluated term by term in FP64. */
double cqo_q(double t, double a, double b)
{
    double c = 1.0 - a - b;
    return a * t + b * t * t + c * t * t * t;
}

/* Reconstructed weight w = s * sign(k) * q(t) in FP64 for code u. */
double cqo_level(int u, int B, int mode, float s, uint16_t a_h, uint16_t b_h)
{
    int sg;
    double t;
    cqo_coord(u, B, mode, &sg, &t);
    double a = cqo_half_to_double(a_h);
    double b = cqo_half_to_double(b_h);
    return (double)s * (double)sg * cqo_q(t, a, b);
}

/* All 2^B levels of one group, in code order. */
void cqo_levels(int B, int mode, float s, uint16_t a_h, uint16_t b_h, double *out)
{
    for (int u = 0; u < (1 << B); u++)
        out[u] = cqo_level(u, B, mode, s, a_h, b_h);
}

/*
 * Exact monotonicity test of q on [0,1] for stored FP16 (a, b): q'(t) =
 * a + 2 b t + 3 c t^2 > 0 for every t in [0,1] ([CQ core]: "candidates must
 * satisfy q'(t) > 0 so that levels never cross").  Every FP16 value is an
 * integer multiple of 2^-24, so A = a*2^24, Bv = b*2^24, C = 2^24 - A - Bv
 * are integers and the test is done in exact integer arithmetic:
 *   q'(0) = a > 0,  q'(1) = 3 - 2a - b > 0, and when the parabola 3c t^2 +
 *   2b t + a has its minimum inside (0,1) (c > 0 and 0 < -b < 3c), the
 *   minimum a - b^2/(3c) must be > 0, i.e. Bv^2 < 3 A C.
 * Returns 1 when q is strictly increasing on [0,1].
 */
int cqo_is_monotone(uint16_t a_h, uint16_t b_h)
{
    double a = cqo_half_to_double(a_h), b = cqo_half_to_double(b_h);
    if (!isfinite(a) || !isfinite(b))
        return 0;
    __int128 A = (__int128)llround(ldexp(a, 24));
    __int128 Bv = (__int128)llround(ldexp(b, 24));
    __int128 one = (__int128)1 << 24;
    __int128 C = one - A - Bv;
    if (A <= 0)
        return 0;
    if (3 * one - 2 * A - Bv <= 0)
        return 0;
    if (C > 0 && -Bv > 0 && -Bv < 3 * C) {
        if (Bv * Bv >= 3 * A * C)
            return 0;
    }
    return 1;
}

/* ------------------------------------------------------------------------ */
/* Dynamic A8  [CQ a8]                                                       */
/* ------------------------------------------------------------------------ */

/*
 * INT8 carrier of code u: the normalised level sign(k) q(t) placed on the
 * symmetric INT8 grid, RNE(127 sign(k) q(t)) with q in FP64, saturated to
 * [-127, 127] (only the midtread grid's unused code can leave that range).
 * The carrier reconstruction of a weight is s * carrier / 127.
 */
int cqo_carrier(int u, int B, int mode, uint16_t a_h, uint16_t b_h)
{
    int sg;
    double t;
    cqo_coord(u, B, mode, &sg, &t);
    double a = cqo_half_to_double(a_h);
    double b = cqo_half_to_double(b_h);
    double r = nearbyint(127.0 * (double)sg * cqo_q(t, a, b));  /* ties to even */
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return (int)r;
}

/* All 2^B carriers of one group, in code order. */
void cqo_carriers(int B, int mode, uint16_t a_h, uint16_t b_h, int8_t *out)
{
    for (int u = 0; u < (1 << B); u++)
        out[u] = (int8_t)cqo_carrier(u, B, mode, a_h, b_h);
}

/*
 * Dynamic per-row INT8 quantization of bf16 activations x [M][K]: absmax =
 * max |x| of the row; inv = 127 / absmax and every product x * inv rounded
 * to FP32, then to the nearest integer (ties to even), saturated to
 * [-127, 127].  These decisions are taken in FP32, the precision of a GPU
 * kernel taking them.  A zero row gives absmax 0 and all-zero codes.
 */
void cqo_quant_rows(const uint16_t *x, int64_t M, int64_t K, int8_t *xq, float *absmax)
{
    for (int64_t m = 0; m < M; m++) {
        float mx = 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float v = (float)cqo_bf16_to_double(x[m * K + k]);
            if (fabsf(v) > mx) mx = fabsf(v);
        }
        absmax[m] = mx;
        float inv = mx > 0.0f ? 127.0f / mx : 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float v = (float)cqo_bf16_to_double(x[m * K + k]);
            float p = v * inv;
            float r = nearbyintf(p);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            xq[m * K + k] = (int8_t)r;
        }
    }
}

/*
 * Dynamic-A8 GEMM: for every (m, n) and group g the exact integer dot
 * product acc = sum over the group of xq[m][k] * carrier(u[n][k]), then
 * the group scaling y[m][n] = sum_g (absmax[m] / 127) (s[n][g] / 127) acc,
 * here in FP64 with the groups in order.  bound[m][n] (may be NULL) is the
 * same sum over |xq * carrier|: the scale of the tolerance.
 */
void cqo_gemm_a8(const int8_t *xq, const float *absmax, int64_t M, const uint8_t *packed,
                 const float *scales, const uint16_t *ab, int64_t N, int64_t K, int B, int G,
                 int mode, double *y, double *bound)
{
    int64_t ng = K / G, rb = K * B / 8;
    uint8_t *codes = (uint8_t *)malloc((size_t)K);
    int8_t *car = (int8_t *)malloc((size_t)K);
    int8_t tab[256];
    for (int64_t n = 0; n < N; n++) {
        cqo_unpack(packed + n * rb, 1, K, B, codes);
        for (int64_t g = 0; g < ng; g++) {
            cqo_carriers(B, mode, ab[(n * ng + g) * 2 + 0], ab[(n * ng + g) * 2 + 1], tab);
            for (int64_t k = g * G; k < (g + 1) * G; k++)
                car[k] = tab[codes[k]];
        }
        for (int64_t m = 0; m < M; m++) {
            double acc_y = 0.0, acc_b = 0.0;
            double sx = (double)absmax[m] / 127.0;
            for (int64_t g = 0; g < ng; g++) {
                int64_t acc = 0, aabs = 0;
                for (int64_t k = g * G; k < (g + 1) * G; k++) {
                    int64_t p = (int64_t)xq[m * K + k] * (int64_t)car[k];
                    acc += p;
                    aabs += p < 0 ? -p : p;
                }
                double f = sx * ((double)scales[n * ng + g] / 127.0);
                acc_y += f * (double)acc;
                acc_b += fabs(f) * (double)aabs;
            }
            y[m * N + n] = acc_y;
            if (bound) bound[m * N + n] = acc_b;
        }
    }
    free(codes);
    free(car);
}

/* ------------------------------------------------------------------------ */
/* Decode  [CQ core] + [CQ fused]                                            */
/* ------------------------------------------------------------------------ */

/*
 * packed + scales + ab -> W in three forms: exact FP64 levels (may be NULL),
 * the FP64 level rounded once to FP32, and that FP32 rounded to BF16.
 */
void cqo_decode(const uint8_t *packed, const float *scales, const uint16_t *ab,
                int64_t N, int64_t K, int B, int G, int mode,
                double *w64, float *w32, uint16_t *w16)
{
    int64_t ng = K / G;
    uint8_t *codes = (uint8_t *)malloc((size_t)K);
    for (int64_t n = 0; n < N; n++) {
        cqo_unpack(packed + n * (K * B / 8), 1, K, B, codes);
        for (int64_t k = 0; k < K; k++) {
            int64_t g = k / G;
            float s = scales[n * ng + g];
            uint16_t a_h = ab[(n * ng + g) * 2 + 0];
            uint16_t b_h = ab[(n * ng + g) * 2 + 1];
            double L = cqo_level(codes[k], B, mode, s, a_h, b_h);
            float L32 = (float)L;                /* one RNE rounding to FP32 */
            if (w64) w64[n * K + k] = L;
            if (w32) w32[n * K + k] = L32;
            if (w16) w16[n * K + k] = cqo_float_to_bf16(L32);
        }
    }
    free(codes);
}

/* ------------------------------------------------------------------------ */
/* GEMM  [CQ fused]: y[m][n] = sum_k x[m][k] * w[n][k], FP64                 */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *x; int64_t M;
    const uint8_t *packed; const float *scales; const uint16_t *ab;
    int64_t N, K; int B, G, mode;
    int operand_bf16;
    double *y, *bound;
    int64_t n0, n1;
} gemm_job;

static void *gemm_worker(void *p)
{
    gemm_job *j = (gemm_job *)p;
    double *wrow = (double *)malloc((size_t)j->K * sizeof(double));
    int64_t rb = j->K * j->B / 8, ng = j->K / j->G;
    for (int64_t n = j->n0; n < j->n1; n++) {
        /* this row's exact levels */
        cqo_decode(j->packed + n * rb, j->scales + n * ng, j->ab + n * ng * 2,
                   1, j->K, j->B, j->G, j->mode, wrow, NULL, NULL);
        /* the model-dtype operand: each level rounded once to FP32, then to
         * BF16 ([CQ fused]: levels are converted to the model dtype before
         * the dot product) */
        if (j->operand_bf16)
            for (int64_t k = 0; k < j->K; k++)
                wrow[k] = cqo_bf16_to_double(cqo_float_to_bf16((float)wrow[k]));
        for (int64_t m = 0; m < j->M; m++) {
            double acc = 0.0, bnd = 0.0;
            for (int64_t k = 0; k < j->K; k++) {
                double xv = cqo_bf16_to_double(j->x[m * j->K + k]);
                acc += xv * wrow[k];
                bnd += fabs(xv * wrow[k]);
            }
            j->y[m * j->N + n] = acc;
            if (j->bound)
                j->bound[m * j->N + n] = bnd;
        }
    }
    free(wrow);
    return NULL;
}

int cqo_num_threads(int requested)
{
    if (requested > 0)
        return requested;
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    return c > 0 ? (int)c : 1;
}

/*
 * x: bf16 [M][K]; W given packed.  y and bound: double [M][N], where
 * bound[m][n] = sum_k |x[m][k] * w[n][k]| (the scale of the tolerance).
 * w is the exact FP64 level, or, with operand_bf16, that level rounded to
 * FP32 and then to BF16 (the operand the tensor cores multiply).
 * Rows of W are split across threads; each output is one plain sequential
 * sum over k.
 */
void cqo_gemm_ex(const uint16_t *x, int64_t M, const uint8_t *packed, const float *scales,
                 const uint16_t *ab, int64_t N, int64_t K, int B, int G, int mode,
                 int operand_bf16, double *y, double *bound, int nthreads)
{
    int T = cqo_num_threads(nthreads);
    if (T > N) T = (int)(N > 0 ? N : 1);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * T);
    gemm_job *jobs = (gemm_job *)malloc(sizeof(gemm_job) * T);
    for (int i = 0; i < T; i++) {
        gemm_job j = {x, M, packed, scales, ab, N, K, B, G, mode, operand_bf16, y, bound,
                      N * i / T, N * (i + 1) / T};
        jobs[i] = j;
        pthread_create(&th[i], NULL, gemm_worker, &jobs[i]);
    }
    for (int i = 0; i < T; i++)
        pthread_join(th[i], NULL);
    free(th);
    free(jobs);
}

/* The FP64-level product (operand_bf16 = 0). */
void cqo_gemm(const uint16_t *x, int64_t M, const uint8_t *packed, const float *scales,
              const uint16_t *ab, int64_t N, int64_t K, int B, int G, int mode,
              double *y, double *bound, int nthreads)
{
    cqo_gemm_ex(x, M, packed, scales, ab, N, K, B, G, mode, 0, y, bound, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Data-free group fitter  [CQ fit]                                          */
/* ------------------------------------------------------------------------ */

/*
 * Nearest level: the index u of the level closest to v, ties to the lower
 * code.  Levels are sorted ascending (q is increasing and the grid is
 * sign-symmetric), so a binary search finds the bracketing pair.
 */
int cqo_nearest(const double *lv, int nlev, double v)
{
    int lo = 0, hi = nlev - 1;
    if (v <= lv[0]) return 0;
    if (v >= lv[hi]) return hi;
    while (hi - lo > 1) {                       /* invariant lv[lo] < v < lv[hi] */
        int mid = (lo + hi) / 2;
        if (lv[mid] <= v) lo = mid; else hi = mid;
    }
    if (lv[lo] == v) return lo;
    return (v - lv[lo] <= lv[hi] - v) ? lo : hi;
}

/* Linear-scan nearest level (brute force, used by the tests as a pin). */
int cqo_nearest_bruteforce(const double *lv, int nlev, double v)
{
    int best = 0;
    double bd = fabs(v - lv[0]);
    for (int u = 1; u < nlev; u++) {
        double d = fabs(v - lv[u]);
        if (d < bd) { bd = d; best = u; }
    }
    return best;
}

typedef struct {
    /* candidate grid */
    int na, nb, nalpha;
    const double *a_grid, *b_grid, *alpha_grid;
    int uniform_only;          /* 1: only (a,b) = (1,0)  -> optimal clipped INT */
    double lambda;             /* weight of the carrier error in the objective */
} fit_cfg;

/* Number of codes a grid mode uses: 2^B (midrise) or 2^B - 1 (midtread). */
static int used_levels(int B, int mode)
{
    return mode == CQO_MIDRISE ? (1 << B) : (1 << B) - 1;
}

/*
 * SSE of group w[G] under (s, a_h, b_h) with every weight on its nearest
 * continuous level; codes written when codes_out != NULL.  When sse_a8 is
 * not NULL it receives the carrier error of the same codes, the sum of
 * (w - s * carrier(u) / 127)^2  [CQ a8].
 */
static double group_sse(const double *w, int G, int B, int mode, float s,
                        uint16_t a_h, uint16_t b_h, uint8_t *codes_out, int *clipped,
                        double *sse_a8)
{
    double lv[256];
    int8_t car[256];
    int nl = used_levels(B, mode);
    cqo_levels(B, mode, s, a_h, b_h, lv);
    if (sse_a8) cqo_carriers(B, mode, a_h, b_h, car);
    double sse = 0.0, sse8 = 0.0;
    int clip = 0;
    for (int i = 0; i < G; i++) {
        int u = cqo_nearest(lv, nl, w[i]);
        double e = w[i] - lv[u];
        sse += e * e;
        if (sse_a8) {
            double e8 = w[i] - (double)s * (double)car[u] / 127.0;
            sse8 += e8 * e8;
        }
        if (fabs(w[i]) > (double)s) clip++;
        if (codes_out) codes_out[i] = (uint8_t)u;
    }
    if (clipped) *clipped = clip;
    if (sse_a8) *sse_a8 = sse8;
    return sse;
}

/*
 * Fit one group, following the article's steps [CQ fit]:
 *   (1) the group is given;
 *   (2) search monotone (a, b) candidates -- the uniform point (1, 0) is
 *       always a candidate;
 *   (3) jointly search the scale / clipping threshold s = alpha * max|w|;
 *   (4) assign every weight to its nearest reconstruction level;
 *   (5) cast a, b to FP16 and keep s in FP32, then recompute the codes and
 *       the error with the stored values.
 * The objective is the group's squared error L_C, plus lambda times the
 * carrier error L_A8 of the same codes when lambda > 0 (the A8 carrier
 * correction of [CQ a8]).  Ties keep the earliest candidate in enumeration
 * order: (1,0) first, then the (a,b) grid in order, and for each (a,b)
 * alpha ascending.
 * Outputs: codes[G], s, a_h, b_h, the carrier error (sse_a8, may be NULL);
 * return value = L_C with the stored values.
 */
static double fit_group(const double *w, int G, int B, int mode, const fit_cfg *cfg,
                        uint8_t *codes, float *s_out, uint16_t *a_out, uint16_t *b_out,
                        int *clipped, double *sse_a8)
{
    double mx = 0.0;
    for (int i = 0; i < G; i++)
        if (fabs(w[i]) > mx) mx = fabs(w[i]);
    if (mx == 0.0) {                             /* all-zero group */
        *s_out = 0.0f;
        *a_out = cqo_double_to_half(1.0);
        *b_out = cqo_double_to_half(0.0);
        return group_sse(w, G, B, mode, 0.0f, *a_out, *b_out, codes, clipped, sse_a8);
    }
    const int joint = cfg->lambda > 0.0;
    double best = INFINITY;
    double best_a = 1.0, best_b = 0.0;
    float best_s = (float)mx;
    int ncand = cfg->uniform_only ? 1 : 1 + cfg->na * cfg->nb;
    for (int c = 0; c < ncand; c++) {
        double a, b;
        if (c == 0) { a = 1.0; b = 0.0; }
        else {
            a = cfg->a_grid[(c - 1) / cfg->nb];
            b = cfg->b_grid[(c - 1) % cfg->nb];
            if (a == 1.0 && b == 0.0) continue;
        }
        uint16_t a_h = cqo_double_to_half(a), b_h = cqo_double_to_half(b);
        if (!cqo_is_monotone(a_h, b_h)) continue;
        for (int ia = 0; ia < cfg->nalpha; ia++) {
            float s = (float)(cfg->alpha_grid[ia] * mx);
            double e8 = 0.0;
            double e = group_sse(w, G, B, mode, s, a_h, b_h, NULL, NULL, joint ? &e8 : NULL);
            if (joint) e += cfg->lambda * e8;
            if (e < best) { best = e; best_a = a; best_b = b; best_s = s; }
        }
    }
    /* step (5): FP16 a, b and FP32 s, then codes and error recomputed */
    *a_out = cqo_double_to_half(best_a);
    *b_out = cqo_double_to_half(best_b);
    *s_out = best_s;
    return group_sse(w, G, B, mode, best_s, *a_out, *b_out, codes, clipped, sse_a8);
}

typedef struct {
    const double *w; int64_t ngroups; int G, B, mode;
    const fit_cfg *cfg;
    uint8_t *codes; float *s; uint16_t *ab; double *sse; int32_t *clipped; double *sse_a8;
    int64_t g0, g1;
} fit_job;

static void *fit_worker(void *p)
{
    fit_job *j = (fit_job *)p;
    for (int64_t g = j->g0; g < j->g1; g++) {
        int clip = 0;
        double e = fit_group(j->w + g * j->G, j->G, j->B, j->mode, j->cfg,
                             j->codes + g * j->G, &j->s[g], &j->ab[2 * g],
                             &j->ab[2 * g + 1], &clip, j->sse_a8 ? &j->sse_a8[g] : NULL);
        j->sse[g] = e;
        j->clipped[g] = clip;
    }
    return NULL;
}

/*
 * Fit ngroups independent groups of G weights (w is [ngroups][G]) with the
 * objective L_C + lambda * L_A8 (lambda = 0: the A16 fit).
 * Outputs per group: codes [ngroups][G], s [ngroups], ab [ngroups][2] (fp16
 * bits), sse [ngroups] (L_C), clipped [ngroups] (count of |w| > s), and
 * sse_a8 [ngroups] (L_A8, may be NULL).
 */
void cqo_fit_joint(const double *w, int64_t ngroups, int G, int B, int mode,
                   const double *a_grid, int na, const double *b_grid, int nb,
                   const double *alpha_grid, int nalpha, int uniform_only, double lambda,
                   uint8_t *codes, float *s, uint16_t *ab, double *sse, int32_t *clipped,
                   double *sse_a8, int nthreads)
{
    fit_cfg cfg = {na, nb, nalpha, a_grid, b_grid, alpha_grid, uniform_only, lambda};
    int T = cqo_num_threads(nthreads);
    if (T > ngroups) T = (int)(ngroups > 0 ? ngroups : 1);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * T);
    fit_job *jobs = (fit_job *)malloc(sizeof(fit_job) * T);
    for (int i = 0; i < T; i++) {
        fit_job j = {w, ngroups, G, B, mode, &cfg, codes, s, ab, sse, clipped, sse_a8,
                     ngroups * i / T, ngroups * (i + 1) / T};
        jobs[i] = j;
        pthread_create(&th[i], NULL, fit_worker, &jobs[i]);
    }
    for (int i = 0; i < T; i++)
        pthread_join(th[i], NULL);
    free(th);
    free(jobs);
}

/* The A16 fit: cqo_fit_joint with lambda = 0. */
void cqo_fit(const double *w, int64_t ngroups, int G, int B, int mode,
             const double *a_grid, int na, const double *b_grid, int nb,
             const double *alpha_grid, int nalpha, int uniform_only,
             uint8_t *codes, float *s, uint16_t *ab, double *sse, int32_t *clipped,
             int nthreads)
{
    cqo_fit_joint(w, ngroups, G, B, mode, a_grid, na, b_grid, nb, alpha_grid, nalpha,
                  uniform_only, 0.0, codes, s, ab, sse, clipped, NULL, nthreads);
}

/*
 * Exact minimum SSE of ANY nlev-level scalar quantizer of the n values v
 * (the free-codebook / Lloyd-Max side of the error bound in [CQ two]).
 * Optimal 1-D clustering by dynamic programming over the sorted values
 * (Bellman; Wang & Song, "Ckmeans.1d.dp", 2011): cost(i, j) is the SSE of
 * values i..j around their mean, D[l][j] = min_i D[l-1][i-1] + cost(i, j).
 */
static int cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

double cqo_optimal_sse(const double *v_in, int n, int nlev)
{
    double *v = (double *)malloc(sizeof(double) * n);
    memcpy(v, v_in, sizeof(double) * n);
    qsort(v, n, sizeof(double), cmp_double);
    double *S1 = (double *)calloc(n + 1, sizeof(double));
    double *S2 = (double *)calloc(n + 1, sizeof(double));
    for (int i = 0; i < n; i++) {
        S1[i + 1] = S1[i] + v[i];
        S2[i + 1] = S2[i] + v[i] * v[i];
    }
    if (nlev > n) nlev = n;
    double *D = (double *)malloc(sizeof(double) * (n + 1) * (nlev + 1));
#define DD(l, j) D[(l) * (n + 1) + (j)]
    for (int j = 0; j <= n; j++) DD(0, j) = (j == 0) ? 0.0 : INFINITY;
    for (int l = 1; l <= nlev; l++) {
        DD(l, 0) = 0.0;
        for (int j = 1; j <= n; j++) {
            double best = INFINITY;
            for (int i = l; i <= j; i++) {     /* last cluster = v[i-1 .. j-1] */
                double cnt = j - i + 1;
                double s1 = S1[j] - S1[i - 1], s2 = S2[j] - S2[i - 1];
                double cost = s2 - s1 * s1 / cnt;
                if (cost < 0) cost = 0;
                double c = DD(l - 1, i - 1) + cost;
                if (c < best) best = c;
            }
            DD(l, j) = best;
        }
    }
    double r = DD(nlev, n);
#undef DD
    free(D); free(S1); free(S2); free(v);
    return r;
}

/* ------------------------------------------------------------------------ */
/* Population analysis  [CQ two]: the error bound "Lloyd-Max <= Cubic <=    */
/* best clipped INT" evaluated on a density instead of a finite sample, and */
/* the share of the INT / Lloyd-Max gap that the cubic recovers.            */
/* ------------------------------------------------------------------------ */

#define CQO_DIST_GAUSS 0     /* N(0, 1) */
#define CQO_DIST_LAPLACE 1   /* Laplace with unit variance: scale 1/sqrt(2) */

static const double kLaplaceScale = 0.70710678118654752440;   /* 1/sqrt(2) */

/* Upper-tail probability of N(0,1). */
static double gauss_q(double x) { return 0.5 * erfc(x / 1.41421356237309504880); }
static double gauss_pdf(double x) { return exp(-0.5 * x * x) * 0.39894228040143267794; }

/*
 * Partial moments m[j] = integral over [a, b] of x^j f(x), j = 0, 1, 2, for
 * 0 <= a <= b (b may be +INFINITY), in closed form:
 *   Gaussian:  m0 = Q(a) - Q(b),  m1 = pdf(a) - pdf(b),
 *              m2 = m0 + a pdf(a) - b pdf(b)            (integration by parts)
 *   Laplace (scale l): m0 = (e^{-a/l} - e^{-b/l}) / 2,
 *              m1 = ((a + l) e^{-a/l} - (b + l) e^{-b/l}) / 2,
 *              m2 = ((a^2 + 2 l a + 2 l^2) e^{-a/l} - (same at b)) / 2.
 */
static void half_moments(int dist, double a, double b, double m[3])
{
    int inf = isinf(b);
    if (dist == CQO_DIST_GAUSS) {
        double pa = gauss_pdf(a), pb = inf ? 0.0 : gauss_pdf(b);
        m[0] = gauss_q(a) - (inf ? 0.0 : gauss_q(b));
        m[1] = pa - pb;
        m[2] = m[0] + a * pa - (inf ? 0.0 : b * pb);
    } else {
        double l = kLaplaceScale;
        double ea = exp(-a / l), eb = inf ? 0.0 : exp(-b / l);
        double bb = inf ? 0.0 : b;
        m[0] = 0.5 * (ea - eb);
        m[1] = 0.5 * ((a + l) * ea - (bb + l) * eb);
        m[2] = 0.5 * ((a * a + 2 * l * a + 2 * l * l) * ea - (bb * bb + 2 * l * bb + 2 * l * l) * eb);
    }
}

/* Partial moments over any interval a < b, using the symmetry of f. */
void cqo_pop_moments(int dist, double a, double b, double *m)
{
    if (b <= 0) {
        half_moments(dist, -b, -a, m);
        m[1] = -m[1];
    } else if (a >= 0) {
        half_moments(dist, a, b, m);
    } else {
        double l[3], r[3];
        half_moments(dist, 0.0, -a, l);
        half_moments(dist, 0.0, b, r);
        m[0] = l[0] + r[0];
        m[1] = r[1] - l[1];
        m[2] = l[2] + r[2];
    }
}

/*
 * Mean squared error of the nearest-level quantizer with the n levels lv
 * (ascending) on the density: the decision thresholds are the midpoints of
 * neighbouring levels, and each cell contributes the integral of
 * (x - level)^2 f(x) = m2 - 2 level m1 + level^2 m0.
 */
double cqo_pop_mse(int dist, const double *lv, int n)
{
    double tot = 0.0;
    for (int i = 0; i < n; i++) {
        double lo = i == 0 ? -INFINITY : 0.5 * (lv[i - 1] + lv[i]);
        double hi = i == n - 1 ? INFINITY : 0.5 * (lv[i] + lv[i + 1]);
        double m[3];
        cqo_pop_moments(dist, lo, hi, m);
        tot += m[2] - 2.0 * lv[i] * m[1] + lv[i] * lv[i] * m[0];
    }
    return tot;
}

/* Inverse of an increasing function on the real line by bisection. */
static double invert(double (*F)(double), double p)
{
    double lo = -60.0, hi = 60.0;
    for (int it = 0; it < 200; it++) {
        double mid = 0.5 * (lo + hi);
        if (F(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* CDFs of the point densities proportional to f^(1/3): N(0, 3) for the
 * Gaussian, Laplace with three times the scale for the Laplace density. */
static double cdf_gauss3(double x) { return 1.0 - gauss_q(x / 1.73205080756887729353); }
static double cdf_laplace3(double x)
{
    double l = 3.0 * kLaplaceScale;
    return x < 0 ? 0.5 * exp(x / l) : 1.0 - 0.5 * exp(-x / l);
}

/*
 * Lloyd-Max quantizer with n levels (the free scalar codebook of [CQ two]'s
 * bound) by Lloyd's iteration: thresholds at the midpoints of the levels,
 * each level moved to the centroid m1/m0 of its cell, until no level moves
 * by more than tol or max_iter sweeps.  Starts from the asymptotically
 * optimal companding levels (quantiles of f^(1/3), Panter and Dite 1951).
 * Writes the ascending levels to lv and returns their MSE.
 */
double cqo_pop_lloyd_max(int dist, int n, int max_iter, double tol, double *lv)
{
    double (*F)(double) = dist == CQO_DIST_GAUSS ? cdf_gauss3 : cdf_laplace3;
    for (int i = 0; i < n; i++)
        lv[i] = invert(F, (i + 0.5) / n);
    double *nx = (double *)malloc(sizeof(double) * n);
    for (int it = 0; it < max_iter; it++) {
        double move = 0.0;
        for (int i = 0; i < n; i++) {
            double lo = i == 0 ? -INFINITY : 0.5 * (lv[i - 1] + lv[i]);
            double hi = i == n - 1 ? INFINITY : 0.5 * (lv[i] + lv[i + 1]);
            double m[3];
            cqo_pop_moments(dist, lo, hi, m);
            nx[i] = m[0] > 0 ? m[1] / m[0] : lv[i];
            double d = fabs(nx[i] - lv[i]);
            if (d > move) move = d;
        }
        memcpy(lv, nx, sizeof(double) * n);
        if (move <= tol) break;
    }
    free(nx);
    return cqo_pop_mse(dist, lv, n);
}

/*
 * Level shape of an n-level cubic grid on [-1, 1]: code i has the signed
 * coordinate (2i - (n-1)) / (n-1), i.e. t = |k| / Kc with Kc = (n-1)/2 --
 * the midrise grid for n = 2^B and the midtread grid (without its unused
 * code) for n = 2^B - 1 -- mapped through q  [CQ core].
 */
void cqo_pop_shape(int n, double a, double b, double *out)
{
    for (int i = 0; i < n; i++) {
        double k = 2.0 * i - (n - 1);
        double t = fabs(k) / (n - 1);
        out[i] = (k > 0 ? 1.0 : (k < 0 ? -1.0 : 0.0)) * cqo_q(t, a, b);
    }
}

/* Continuous counterpart of cqo_is_monotone: q'(t) > 0 on [0, 1]. */
int cqo_pop_monotone(double a, double b)
{
    double c = 1.0 - a - b;
    if (!(a > 0) || !(3.0 - 2.0 * a - b > 0))
        return 0;
    if (c > 0 && -b > 0 && -b < 3.0 * c && !(a - b * b / (3.0 * c) > 0))
        return 0;
    return 1;
}

/*
 * min over the group scale s of the MSE of the levels s * shape (the
 * clip threshold of a population quantizer is its scale): a scan of log s
 * over [0.3, 40] in 64 steps, then golden-section search between the scan
 * points around the best one.  Returns the MSE, writes s.
 */
double cqo_pop_best_scale(int dist, const double *shape, int n, double *s_out)
{
    double *lv = (double *)malloc(sizeof(double) * n);
    const double l0 = log(0.3), l1 = log(40.0);
    const int steps = 64;
    double best = INFINITY;
    int bi = 0;
    for (int j = 0; j <= steps; j++) {
        double s = exp(l0 + (l1 - l0) * j / steps);
        for (int i = 0; i < n; i++) lv[i] = s * shape[i];
        double e = cqo_pop_mse(dist, lv, n);
        if (e < best) { best = e; bi = j; }
    }
    double lo = l0 + (l1 - l0) * (bi > 0 ? bi - 1 : 0) / steps;
    double hi = l0 + (l1 - l0) * (bi < steps ? bi + 1 : steps) / steps;
    const double gr = 0.61803398874989484820;
    double x1 = hi - gr * (hi - lo), x2 = lo + gr * (hi - lo), f1, f2;
    for (int i = 0; i < n; i++) lv[i] = exp(x1) * shape[i];
    f1 = cqo_pop_mse(dist, lv, n);
    for (int i = 0; i < n; i++) lv[i] = exp(x2) * shape[i];
    f2 = cqo_pop_mse(dist, lv, n);
    for (int it = 0; it < 60; it++) {
        if (f1 < f2) {
            hi = x2; x2 = x1; f2 = f1;
            x1 = hi - gr * (hi - lo);
            for (int i = 0; i < n; i++) lv[i] = exp(x1) * shape[i];
            f1 = cqo_pop_mse(dist, lv, n);
        } else {
            lo = x1; x1 = x2; f1 = f2;
            x2 = lo + gr * (hi - lo);
            for (int i = 0; i < n; i++) lv[i] = exp(x2) * shape[i];
            f2 = cqo_pop_mse(dist, lv, n);
        }
    }
    double ls = f1 < f2 ? x1 : x2, e = f1 < f2 ? f1 : f2;
    if (best < e) {                       /* the scan point itself was better */
        e = best;
        ls = l0 + (l1 - l0) * bi / steps;
    }
    free(lv);
    if (s_out) *s_out = exp(ls);
    return e;
}

static double cubic_cost(int dist, int n, double a, double b, double *shape, double *s)
{
    if (!cqo_pop_monotone(a, b)) return INFINITY;
    cqo_pop_shape(n, a, b, shape);
    return cqo_pop_best_scale(dist, shape, n, s);
}

/*
 * Best n-level cubic quantizer of the density: min over monotone (a, b)
 * and s of the MSE ([CQ fit]: search over monotone shape candidates jointly
 * with the scale / clip).  A scan of a in [0.02, 2.92] and b in [-3, 3] with
 * step 0.1 (plus the uniform point (1, 0)), then a pattern search around
 * the best point: an 11 x 11 grid of step 0.02 that shrinks fourfold each
 * round, eleven rounds.  Returns the MSE; writes a, b, s.
 */
double cqo_pop_cubic(int dist, int n, double *a_out, double *b_out, double *s_out)
{
    double *shape = (double *)malloc(sizeof(double) * n);
    double s, ba = 1.0, bb = 0.0, bs = 0.0;
    double best = cubic_cost(dist, n, 1.0, 0.0, shape, &bs);
    for (int ia = 0; ia <= 29; ia++) {
        for (int ib = 0; ib <= 60; ib++) {
            double a = 0.02 + 0.1 * ia, b = -3.0 + 0.1 * ib;
            double e = cubic_cost(dist, n, a, b, shape, &s);
            if (e < best) { best = e; ba = a; bb = b; bs = s; }
        }
    }
    double h = 0.02;
    for (int round = 0; round < 11; round++) {
        double ca = ba, cb = bb;
        for (int ia = -5; ia <= 5; ia++) {
            for (int ib = -5; ib <= 5; ib++) {
                double a = ca + h * ia, b = cb + h * ib;
                double e = cubic_cost(dist, n, a, b, shape, &s);
                if (e < best) { best = e; ba = a; bb = b; bs = s; }
            }
        }
        h *= 0.25;
    }
    free(shape);
    if (a_out) *a_out = ba;
    if (b_out) *b_out = bb;
    if (s_out) *s_out = bs;
    return best;
}
