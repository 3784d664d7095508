/*
 * cq.h -- C ABI of libcq, the B200 (sm_100a) CubicQuant weight-only GEMM
 * library.
 *
 * The method (ModelScope article "CubicQuant：用三次曲线重塑低比特量化，Kimi
 * K3 2.5Bit 模型首发实践", cited as [CQ]) stores each weight as a B-bit code
 * u, packed densely, in groups of G weights that carry an FP32 scale s and
 * two FP16 shape parameters a, b (c = 1 - a - b is derived).  A code
 * decodes to
 *         w = s * sign(k) * q(t),   q(t) = a t + b t^2 + c t^3,
 * with k the signed integer coordinate of u and t = |k| / Kc its normalised
 * magnitude ([CQ] section "CubicQuant 核心：把直线网格“掰弯”").  The article's
 * code-to-coordinate formula was lost in extraction; this library fixes
 *   CQ_GRID_MIDRISE  (default): Kc = (2^B-1)/2, k = u - Kc, t = |k|/Kc;
 *   CQ_GRID_MIDTREAD          : Kc = 2^(B-1)-1, k = u - Kc, t = |k|/Kc,
 *                               sign(0) = 0 (code 2^B-1 is decoded by the
 *                               same formula; fitters never emit it).
 * With a = 1, b = 0 both give the symmetric uniform integer grid.
 *
 * Data layout (all row-major, all buffers owned by the caller):
 *   W      logical [N][K] weights; groups are G consecutive K-elements.
 *   packed uint8 [N][K*B/8]: code (n,k) occupies bits [k*B, k*B+B) of row n's
 *          byte stream, least significant bit first ([CQ] only says the
 *          stream is dense and contiguous, section "为什么只用两个形状参数？").
 *   scales float [N][K/G]                    -- s per group
 *   ab     uint16 (IEEE binary16) [N][K/G][2] -- (a, b) per group
 *   x      uint16 (bfloat16) [M][K] activations
 *   y      [M][N] (or [M][N/2] with CQ_EPI_SWIGLU), float or bfloat16
 * Storage per weight is B + 64/G bits ([CQ] section "存储开销是透明的").
 *
 * Conventions:
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise.
 *   - Every call is asynchronous on the given cudaStream_t (passed as void*,
 *     NULL = legacy default stream) and returns a cq_status.  Arguments are
 *     validated on the host before anything is launched; on error nothing
 *     is launched and no output is touched.
 *   - Supported: B in 1..8 for cq_pack, cq_decode, cq_gemm,
 *     cq_gemm_noalloc and the MoE layer (midtread: 2..8; the code stream of
 *     [CQ] "为什么只用两个形状参数？" is an ordinary 1..8-bit integer stream);
 *     B in {2,3,4} for the Dynamic A8 path;
 *     G a multiple of 128; K a multiple of G;
 *     N >= 1; packed / x / y / workspace 16-byte aligned; scales and ab
 *     4-byte aligned.
 *   - The library allocates no memory.  Calls that need scratch take a
 *     caller-provided workspace whose size is given by the matching
 *     *_workspace_size() query.
 *   - Device-side waits are bounded; a wait that runs out records an error
 *     that cq_get_device_error() reports as CQ_ERR_TIMEOUT.
 */
#ifndef CQ_H_
#define CQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CQ_API __attribute__((visibility("default")))
#else
#define CQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CQ_OK = 0,
    CQ_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad enum   */
    CQ_ERR_UNSUPPORTED = 2,  /* B, G, K, N or alignment not supported  */
    CQ_ERR_CUDA = 3,         /* a CUDA runtime call failed             */
    CQ_ERR_TIMEOUT = 4,      /* a bounded device wait ran out          */
    CQ_ERR_WORKSPACE = 5     /* workspace missing or too small         */
} cq_status;

enum { CQ_GRID_MIDRISE = 0, CQ_GRID_MIDTREAD = 1 };
enum { CQ_DTYPE_F32 = 0, CQ_DTYPE_BF16 = 1 };
enum { CQ_EPI_NONE = 0, CQ_EPI_SWIGLU = 1 };

/* Library version as 10000*major + 100*minor + patch. */
CQ_API int cq_version(void);

/* Static English description of a cq_status value. */
CQ_API const char *cq_status_string(int status);

/*
 * cq_pack -- pack one code per byte into the dense LSB-first bit stream.
 *   codes  uint8 [N][K], each < 2^B (higher bits are ignored)
 *   packed uint8 [N][K*B/8] (output)
 * Requires K*B % 8 == 0.  [CQ] "为什么只用两个形状参数？": codes remain an
 * ordinary 1-8 bit scalar stream that can be packed contiguously.
 */
CQ_API int cq_pack(const uint8_t *codes, int64_t N, int64_t K, int B, uint8_t *packed,
            void *stream);

/*
 * cq_decode -- expand packed codes and group parameters into weights.
 *   out_dtype CQ_DTYPE_F32: W_out float [N][K], each element the level
 *             s*sign(k)*q(t) evaluated in FP64 and rounded once to FP32;
 *   out_dtype CQ_DTYPE_BF16: W_out bfloat16 [N][K], that FP32 value rounded
 *             to nearest-even BF16.
 * B in 1..8 (midtread grid: 2..8); CQ_ERR_UNSUPPORTED otherwise.
 * [CQ] "CubicQuant 核心" (reconstruction); this is the parity tool, the GEMM
 * never materialises W ([CQ] "压缩权重必须“边解码、边计算”").
 */
CQ_API int cq_decode(const uint8_t *packed, const float *scales, const uint16_t *ab,
              int64_t N, int64_t K, int B, int G, int grid_mode, int out_dtype,
              void *W_out, void *stream);

/*
 * cq_gemm -- y[m][n] = sum_k x[m][k] * w[n][k] with FP32 accumulation, the
 * weights decoded tile by tile on chip (A16 path, [CQ] "一份 checkpoint，同时
 * 服务 A16 与 Dynamic A8" and "压缩权重必须“边解码、边计算”").
 *   x          bfloat16 [M][K]; M >= 0 (M == 0 is a no-op)
 *   epilogue   CQ_EPI_NONE: y [M][N];
 *              CQ_EPI_SWIGLU: rows [0,N/2) are gate, rows [N/2,N) are up,
 *              y[m][j] = silu(g) * u with silu(g) = g / (1 + exp(-g)),
 *              y is [M][N/2]; requires N % 128 == 0.
 *   out_dtype  CQ_DTYPE_F32 or CQ_DTYPE_BF16
 *   workspace  device scratch of at least cq_gemm_workspace_size(...) bytes
 *              (may be NULL when that size is 0).  Its first bytes hold
 *              counters that must be zero before the first call that uses
 *              the buffer; every completed call leaves them zero again.
 * Calls that share one workspace must not overlap on the GPU.
 * Paths (B in {2,3,4}): M <= 2 runs the decode-sized GEMV kernel (no
 * workspace) where its plan fits; 3 <= M <= 8 with K a multiple of 512 runs
 * the narrow-row kernel
 * ([CQ] "压缩权重必须“边解码、边计算”": the narrow-row GEMV; register-operand
 * tensor-core MMAs, 16-row x one-slice work units split evenly over the SMs,
 * row blocks shared by two CTAs summed through the workspace), also the
 * fallback of M <= 2 shapes the GEMV does not take; everything else
 * runs the tensor-core engine (128-row weight tiles, 16- to 192-token
 * activation tiles, stream-K over the K slices, partial tiles summed in a
 * fixed order).  B in {1,5,6,7,8} always runs the engine, with token tiles
 * of at most 128 and a decoder that evaluates each code's level (FP64 q(t)
 * times s, rounded to FP32 and then to BF16, as the pair tables of the other
 * widths hold it) instead of looking it up.  Results are run-to-run
 * deterministic.  All three kernels
 * are launched with programmatic dependent launch: their setup may overlap
 * the end of the preceding kernel in the stream, and they read no caller
 * memory before that kernel has completed (stream order holds).
 */
CQ_API size_t cq_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int B, int G,
                              int epilogue);
CQ_API int cq_gemm(const uint16_t *x, int64_t M, const uint8_t *packed, const float *scales,
            const uint16_t *ab, int64_t N, int64_t K, int B, int G, int grid_mode,
            int epilogue, int out_dtype, void *y, void *workspace, size_t ws_bytes,
            void *stream);

/*
 * cq_gemm_noalloc -- cq_gemm without a caller workspace, for callers that
 * cannot allocate device memory: code that runs under an allocator it does
 * not own (a plugin or operator inside another engine that hands it only
 * inputs and outputs), or a latency-critical path whose memory is planned
 * in advance and may not call cudaMalloc while serving.  Same arguments,
 * semantics and results as cq_gemm (the article has no counterpart; this is
 * a calling convenience).
 *   Scratch: a fixed 4 MiB array inside libcq (every GPU that loads the
 *   library holds it until the process exits), enough for any M <= 16 on a
 *   148-SM B200 (narrow-row kernel or engine); a problem that needs more
 *   returns CQ_ERR_WORKSPACE.
 *   The first call on a device looks up that array's device address (a CUDA
 *   runtime query, which also loads libcq's device code there) and caches
 *   it with the device's context; make that first call before any stream
 *   capture.  After a cudaDeviceReset the device has a new context and the
 *   next call looks the address up again (again: not inside a capture).
 *   Every call shares the one array: calls that overlap on the GPU (other
 *   streams, other host threads) race and must not be issued.  All argument
 *   checks run before anything is queued; a call that passes them clears
 *   the array's tile counters with cudaMemsetAsync on `stream`.  It calls
 *   no allocating or freeing routine.
 */
CQ_API int cq_gemm_noalloc(const uint16_t *x, int64_t M, const uint8_t *packed,
                           const float *scales, const uint16_t *ab, int64_t N, int64_t K, int B,
                           int G, int grid_mode, int epilogue, int out_dtype, void *y,
                           void *stream);

/*
 * cq_gemm_host -- cq_gemm for a caller whose activations and outputs live in
 * HOST memory (one decode step served from the host): queues on `stream`
 * the copy of x_host into the device staging buffer x_dev, cq_gemm on it,
 * and the copy of the output from the device staging buffer y_dev into
 * y_host.  Same arguments, semantics and results as cq_gemm otherwise (the
 * article has no counterpart; this is a calling convenience).
 *   x_host  HOST bfloat16 [M][K]; y_host HOST [M][N] (or [M][N/2] with
 *           SwiGLU) in out_dtype.  When both are page-locked (pinned) and
 *           16-byte aligned, x is copied by a small kernel that reads the
 *           host memory directly, chained to the GEMM by programmatic
 *           dependent launch, and the GEMM stores its output straight into
 *           y_host (y_dev is then not used); otherwise both copies go
 *           through the copy engine (pageable memory is staged by the
 *           driver, synchronously).  Both must stay valid until the stream
 *           has run the call's work.
 *   x_dev   DEVICE staging buffer of M*K*2 bytes; y_dev DEVICE staging
 *           buffer of the output's size; both 16-byte aligned, owned by the
 *           caller (the library allocates nothing).
 *   workspace / ws_bytes as cq_gemm (cq_gemm_workspace_size bytes).
 * Every argument and size check runs before anything is queued.
 */
CQ_API int cq_gemm_host(const uint16_t *x_host, int64_t M, const uint8_t *packed,
                        const float *scales, const uint16_t *ab, int64_t N, int64_t K, int B,
                        int G, int grid_mode, int epilogue, int out_dtype, void *y_host,
                        uint16_t *x_dev, void *y_dev, void *workspace, size_t ws_bytes,
                        void *stream);

/*
 * Dynamic A8 ([CQ] "一份 checkpoint，同时服务 A16 与 Dynamic A8"): the same
 * checkpoint served with INT8 activations.  The article's carrier and
 * activation formulas were lost in extraction; this library reads them as
 *   carrier(u) = RNE(127 * sign(k) * q(t)) (q in FP64), saturated to +-127,
 *   xq[m][k]   = RNE(x[m][k] * RN_fp32(127 / absmax[m])), saturated to
 *                +-127, absmax[m] = max_k |x[m][k]| (a zero row gives zeros),
 *   y[m][n]    = sum_g (absmax[m] / 127) * (s[n][g] / 127) * acc[m][n][g],
 *                acc the exact integer dot product of group g.
 *
 * cq_quant_rows -- per-row INT8 quantization of bfloat16 activations.
 *   x      bfloat16 [M][K];  xq int8 [M][K] (output);  absmax float [M] (output)
 * Bit-exact: the decisions are taken in FP32 as written above.
 */
CQ_API int cq_quant_rows(const uint16_t *x, int64_t M, int64_t K, int8_t *xq, float *absmax,
                         void *stream);

/*
 * cq_gemm_a8 -- the Dynamic-A8 GEMM: x is quantized per row inside the call
 * (into the workspace), the codes are decoded to their INT8 carriers tile by
 * tile on chip, the integer dot products run on the tensor cores
 * (tcgen05.mma kind::i8, INT32 accumulators in tensor memory) and are
 * scaled once per group in FP32 ([CQ] "实验结果 2. H200 内核交叉点": the A8
 * path wins from M = 64 on).  Arguments, layouts, epilogues and output
 * dtypes as cq_gemm; the workspace (cq_gemm_a8_workspace_size bytes, 256-byte
 * aligned) holds the quantized activations, their row maxima and the
 * stream-K scratch; its counters are cleared by each call.  Calls that share
 * one workspace must not overlap on the GPU.  B in {2,3,4}; run-to-run
 * deterministic.
 */
CQ_API size_t cq_gemm_a8_workspace_size(int64_t M, int64_t N, int64_t K, int B, int G,
                                        int epilogue);
CQ_API int cq_gemm_a8(const uint16_t *x, int64_t M, const uint8_t *packed, const float *scales,
                      const uint16_t *ab, int64_t N, int64_t K, int B, int G, int grid_mode,
                      int epilogue, int out_dtype, void *y, void *workspace, size_t ws_bytes,
                      void *stream);

/*
 * One quantized matrix of an expert (HOST-side description, device pointers).
 */
typedef struct {
    const uint8_t *packed;   /* [rows][cols*B/8]        */
    const float *scales;     /* [rows][cols/G]          */
    const uint16_t *ab;      /* [rows][cols/G][2] fp16  */
    int32_t B;               /* 2, 3 or 4               */
    int32_t reserved;        /* must be 0               */
} cq_matrix_desc;

typedef struct {
    cq_matrix_desc gate_up;  /* [2I][H]: gate rows [0,I), up rows [I,2I) */
    cq_matrix_desc down;     /* [H][I]                                    */
} cq_expert_desc;

/*
 * cq_moe_prepare_layer -- build the device-side table of one MoE layer:
 * for each of the E experts, the TMA descriptors of its packed gate/up and
 * down matrices and their operand descriptions.  `experts` is a HOST array
 * of E descriptions (device pointers inside); `layer` is device memory of
 * cq_moe_layer_bytes(E) bytes owned by the caller, valid as long as the
 * expert weights do not move.  Synchronous (run once per layer, at load).
 * Each matrix must satisfy the cq_gemm requirements (B in 1..8,
 * G % 128 == 0, H and I multiples of G, I % 64 == 0, packed 16-byte aligned).
 * The library remembers, by the table's address, the widths written there:
 * cq_moe_grouped_gemm takes a layer with a width outside {2,3,4} through the
 * tensor-core engine's wide-code decoder (and never the decode-sized path),
 * so such a table must be used at the address this call wrote; a copy of it
 * elsewhere is taken to hold widths 2..4 only, and its wider experts are
 * flagged on the device (cq_get_device_error) instead of computed.
 */
CQ_API size_t cq_moe_layer_bytes(int E);
CQ_API int cq_moe_prepare_layer(const cq_expert_desc *experts, int E, int64_t H, int64_t I,
                                int G, void *layer);

/*
 * cq_moe_grouped_gemm -- the routed-expert FFN of one MoE layer, with
 * per-expert CubicQuant weights (the quantized tensors of [CQ] are the
 * routed experts, section "先看结论").  For every route r = t*k + j:
 *   e = topk_ids[t][j];  g|u = W_gu[e] x_t;  h = bf16(silu(g) * u);
 *   y_r = W_dn[e] h  (FP32 accumulation)
 * and, when out != NULL, out[t] = sum_j topk_w[t][j] * y_(t,j) (j ascending,
 * FP32).  Routing is done on the device (no host synchronisation): routes
 * are grouped by expert, then one grouped launch runs every active expert's
 * gate/up tiles with the SwiGLU epilogue and one runs the down tiles.
 *   tokens     bfloat16 [T][H]
 *   topk_ids   int32 [T][k]; an id outside [0, E) drops that route (its
 *              y_r is zero) and is counted in the device error word
 *   topk_w     float [T][k] (required when out != NULL)
 *   layer      table built by cq_moe_prepare_layer for these E experts
 *   route_out  float [T*k][H] per-route outputs y_r (may be NULL)
 *   out        [T][H] combined output in out_dtype (may be NULL)
 *   workspace  device scratch of at least cq_moe_workspace_size(...) bytes
 * Calls that share one workspace must not overlap on the GPU.  A layer with
 * a 1-bit expert returns CQ_ERR_UNSUPPORTED on the midtread grid.
 */
CQ_API size_t cq_moe_workspace_size(int64_t T, int k, int E, int64_t H, int64_t I, int G);
CQ_API int cq_moe_grouped_gemm(const uint16_t *tokens, int64_t T, const int32_t *topk_ids,
                               const float *topk_w, int k, int E, const void *layer, int64_t H,
                               int64_t I, int G, int grid_mode, int out_dtype, void *route_out,
                               void *out, void *workspace, size_t ws_bytes, void *stream);

/*
 * cq_get_device_error -- synchronise `stream`, then read and clear the
 * device error word of the current device.  Returns CQ_OK when no bounded
 * wait ran out since the last call, CQ_ERR_TIMEOUT otherwise (the site code
 * of the first wait that gave up is stored in *site when site != NULL).
 */
CQ_API int cq_get_device_error(void *stream, int *site);

#ifdef __cplusplus
}
#endif

#endif /* CQ_H_ */
