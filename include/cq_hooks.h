/*
 * cq_hooks.h -- profiling and test hooks of libcq.
 *
 * These entry points are not part of the library's product interface
 * (include/cq.h); they exist so that the library's own test suite and
 * benchmark can reach paths that a normal call never takes.  They follow
 * the conventions of cq.h: device pointers, asynchronous on `stream`,
 * arguments validated on the host, a cq_status result.
 */
#ifndef CQ_HOOKS_H_
#define CQ_HOOKS_H_

#include "cq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * cq_trace_gemm -- cq_gemm (midrise grid, FP32 output) that also stores
 * per-CTA clock64() stamps and per-role cycle counters of the kernel it runs
 * into `trace`: device memory of at least (number of SMs) x 64 uint64 words,
 * written at [CTA][slot].  The slots a kernel fills are listed beside its
 * stamp macros in the kernel source.
 */
CQ_API int cq_trace_gemm(const uint16_t *x, int64_t M, const uint8_t *packed,
                         const float *scales, const uint16_t *ab, int64_t N, int64_t K, int B,
                         int G, int epilogue, void *y, void *workspace, size_t ws_bytes,
                         uint64_t *trace, void *stream);

/*
 * cq_test_gemm_bounded -- cq_gemm (midrise grid, no epilogue, FP32 output)
 * with a chosen bound for every device-side wait (`timeout_ns`).  When
 * skip_first_stage != 0 the call runs on the tensor-core engine whatever M
 * is, and the first code stage and the first activation stage are never
 * loaded, so that the waits for them run out: the kernel then records
 * CQ_ERR_TIMEOUT (read with cq_get_device_error) and returns.  Used to test
 * failure detection without a GPU fault.
 */
CQ_API int cq_test_gemm_bounded(const uint16_t *x, int64_t M, const uint8_t *packed,
                                const float *scales, const uint16_t *ab, int64_t N, int64_t K,
                                int B, int G, void *y, void *workspace, size_t ws_bytes,
                                uint64_t timeout_ns, int skip_first_stage, void *stream);

/*
 * cq_test_gemm_path -- cq_gemm on a chosen kernel: path 0 = the one cq_gemm
 * picks, 1 = the narrow-row kernel (M <= 16), 2 = the decode-sized GEMV
 * (M <= 2), 3 = the tensor-core engine.  A path that does not take the
 * problem returns CQ_ERR_UNSUPPORTED.  cq_test_gemm_path_workspace_size gives
 * the workspace that path needs.  Used to check the kernels against each
 * other on the same inputs.
 */
CQ_API size_t cq_test_gemm_path_workspace_size(int64_t M, int64_t N, int64_t K, int B, int G,
                                               int epilogue, int path);
CQ_API int cq_test_gemm_path(const uint16_t *x, int64_t M, const uint8_t *packed,
                             const float *scales, const uint16_t *ab, int64_t N, int64_t K,
                             int B, int G, int grid_mode, int epilogue, int out_dtype, void *y,
                             void *workspace, size_t ws_bytes, int path, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CQ_HOOKS_H_ */
