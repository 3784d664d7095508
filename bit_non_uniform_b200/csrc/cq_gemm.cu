// cq_gemm.cu -- host side of cq_gemm: argument checks, work partition,
// activation tensor map and the engine launch.
#include <cuda_runtime.h>

#include "cq.h"
#include "cq_hooks.h"
#include "cq_engine.cuh"
#include "cq_gemv_launch.cuh"
#include "cq_narrow_launch.cuh"
#include "cq_host.h"

namespace cq {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;   // 2 s per wait

// The widths the engine decodes through pair tables; the others (1, 5..8)
// take its wide-code decoder, with token tiles of at most 128.
static bool table_width(int B) { return B >= 2 && B <= 4; }

// Token-tile width.  Each token tile decodes the weights again, and up to
// N = 192 the decode of a slice costs more than its MMAs, so wide problems
// take wide tiles with two accumulator buffers in TMEM (beside a ring of two
// decoded slices): 192 tokens for W2/W4 and 176 for W3, whose 64-entry pair
// tables leave room for only two 192-token activation stages but three of
// 176 tokens -- unless the ragged last tile pads more than 15% (W3: 5%)
// beyond 128-token tiles.  (256-token tiles leave room for a single
// accumulator buffer: measured slower.)
static int pick_nt(int64_t M, int B) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128 || !table_width(B)) return 128;
  const int64_t pad128 = (M + 127) / 128 * 128;
  if (B == 3) {
    const int64_t pad176 = (M + 175) / 176 * 176;
    return pad176 * 100 <= pad128 * 105 ? 176 : 128;
  }
  const int64_t pad192 = (M + 191) / 192 * 192;
  return pad192 * 100 <= pad128 * 115 ? 192 : 128;
}

struct GemmPlan {
  int NT, n_tt, n_rt, spt, tiles, P;
  size_t ws_counter_bytes, ws_partial_bytes;
};

static GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int B, int epilogue, int sms) {
  GemmPlan g;
  g.n_rt = epilogue == CQ_EPI_SWIGLU ? static_cast<int>(N / kRows)
                                     : static_cast<int>((N + kRows - 1) / kRows);
  g.NT = pick_nt(M, B);
  g.n_tt = static_cast<int>((M + g.NT - 1) / g.NT);
  g.spt = static_cast<int>(K / kSlice);
  g.tiles = g.n_rt * g.n_tt;
  const int64_t W = static_cast<int64_t>(g.tiles) * g.spt;
  g.P = static_cast<int>(W < sms ? W : sms);
  g.ws_counter_bytes = ((static_cast<size_t>(g.tiles) * sizeof(int) + 255) / 256) * 256;
  g.ws_partial_bytes = static_cast<size_t>(2) * g.P * g.NT * kRows * sizeof(float);
  return g;
}

// Which kernel runs a cq_gemm call: the narrow-row kernel for up to 16 tokens
// when its plan fits, else the decode-sized GEMV (up to 2 tokens), else the
// tensor-core engine.  (The test hook may force one of them.)
enum GemmPath { PATH_AUTO = 0, PATH_NARROW = 1, PATH_GEMV = 2, PATH_ENGINE = 3 };

// The narrow-row kernel takes 3 <= M <= 8 on its own: the GEMV is faster for
// M <= 2, and past 8 tokens (two MMAs per step) the engine is (down_proj
// 7168 x 3072 W3 at M = 8: 18.2 against 20.3 us; gate_up 6144 x 7168 W2:
// 28.0 against 27.7 us; graphs of launches over weights larger than L2).
constexpr int64_t kNrAutoMinM = 3, kNrAutoMaxM = 8;
static bool narrow_wanted(int64_t M, int path) {
  return path == PATH_NARROW || (path == PATH_AUTO && M >= kNrAutoMinM && M <= kNrAutoMaxM);
}

// Scratch bytes of whichever path gemm_impl takes for this problem.
static void gemm_scratch(int64_t M, int64_t N, int64_t K, int B, int G, int epilogue, int sms,
                         size_t* counter_bytes, size_t* total, int path = PATH_AUTO) {
  if (narrow_wanted(M, path)) {
    const NrPlan nv = plan_narrow(M, N, K, B, G, epilogue, sms);
    if (nv.use) {
      *counter_bytes = nv.ws_counter_bytes;
      *total = nv.ws_counter_bytes + nv.ws_partial_bytes;
      return;
    }
  }
  const GvPlan v = path == PATH_ENGINE ? GvPlan{} : plan_gemv(M, N, K, B, G, epilogue, sms);
  if (v.use) {
    *counter_bytes = v.ws_counter_bytes;
    *total = v.ws_counter_bytes + v.ws_partial_bytes;
    return;
  }
  const GemmPlan g = plan_gemm(M, N, K, B, epilogue, sms);
  *counter_bytes = g.ws_counter_bytes;
  *total = g.ws_counter_bytes + g.ws_partial_bytes;
}

// ---------------------------------------------------------------------------
// tensor-core engine path
// ---------------------------------------------------------------------------
template <int NT, int TE>
static int launch_engine(const EngineParams& p, const CUtensorMap& map, const CUtensorMap& wmap,
                         cudaStream_t s) {
  using C = EngineCfg<NT, TE>;
  static std::atomic<uint64_t> smem_set{0};
  if (!ensure_smem_limit(engine_kernel<NT, TE>, C::SMEM, smem_set)) return CQ_ERR_CUDA;
  // programmatic dependent launch: this grid's setup (barriers, TMEM) may
  // overlap the end of the preceding one; the kernel waits for it before
  // reading any caller memory
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(p.P);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, engine_kernel<NT, TE>, p, map, wmap) != cudaSuccess)
    return CQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

// Pair tables of 64 entries for W3, 16 for W2/W4 (the smaller tables leave
// room for more activation stages); the wide-code decoder for the other
// widths (token tiles of at most 128).
template <int NT>
static int launch_engine_te(const EngineParams& p, const CUtensorMap& map,
                            const CUtensorMap& wmap, int B, cudaStream_t s) {
  if (!table_width(B)) {
    if constexpr (NT <= 128) return launch_engine<NT, 0>(p, map, wmap, s);
    return CQ_ERR_UNSUPPORTED;              // pick_nt never plans it
  }
  if (B == 3) return launch_engine<NT, 64>(p, map, wmap, s);
  return launch_engine<NT, 16>(p, map, wmap, s);
}

// Every argument and shape check of cq_gemm except the workspace: a call that
// passes launches nothing unless the problem is empty (M == 0 or N == 0).
static int validate_gemm(const uint16_t* x, int64_t M, const uint8_t* packed,
                         const float* scales, const uint16_t* ab, int64_t N, int64_t K, int B,
                         int G, int grid_mode, int epilogue, int out_dtype, const void* y) {
  int st = validate_matrix(packed, scales, ab, N, K, B, G, grid_mode, 1, 8);
  if (st != CQ_OK) return st;
  if (M < 0) return CQ_ERR_INVALID_ARG;
  if (epilogue != CQ_EPI_NONE && epilogue != CQ_EPI_SWIGLU) return CQ_ERR_INVALID_ARG;
  if (out_dtype != CQ_DTYPE_F32 && out_dtype != CQ_DTYPE_BF16) return CQ_ERR_INVALID_ARG;
  if (epilogue == CQ_EPI_SWIGLU && N % kRows != 0) return CQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return CQ_OK;
  if (K == 0) return CQ_ERR_UNSUPPORTED;
  if (!x || !y) return CQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16)) return CQ_ERR_UNSUPPORTED;
  if (M > (int64_t)1 << 24) return CQ_ERR_UNSUPPORTED;
  // tile counts are int on the device: bound them by the narrowest token tile
  if (((M + 15) / 16) * ((N + kRows - 1) / kRows) >= ((int64_t)1 << 31)) return CQ_ERR_UNSUPPORTED;
  return CQ_OK;
}

int gemm_impl(const uint16_t* x, int64_t M, const uint8_t* packed, const float* scales,
              const uint16_t* ab, int64_t N, int64_t K, int B, int G, int grid_mode,
              int epilogue, int out_dtype, void* y, void* workspace, size_t ws_bytes,
              cudaStream_t stream, uint64_t timeout_ns, int debug_skip,
              uint64_t* trace = nullptr, int path = PATH_AUTO) {
  int st = validate_gemm(x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype,
                         y);
  if (st != CQ_OK) return st;
  if (M == 0 || N == 0) return CQ_OK;
  const int sms = num_sms();
  if (sms <= 0) return CQ_ERR_CUDA;
  if (debug_skip) path = PATH_ENGINE;
  if (narrow_wanted(M, path)) {
    const NrPlan nv = plan_narrow(M, N, K, B, G, epilogue, sms);
    if (nv.use) {
      const size_t need = nv.ws_counter_bytes + nv.ws_partial_bytes;
      if (ws_bytes < need || !workspace) return CQ_ERR_WORKSPACE;
      if (!aligned(workspace, 16)) return CQ_ERR_UNSUPPORTED;
      return run_narrow(nv, x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue,
                        out_dtype, y, workspace, stream, timeout_ns, trace);
    }
    if (path == PATH_NARROW) return CQ_ERR_UNSUPPORTED;
  }
  const GvPlan v = path == PATH_ENGINE ? GvPlan{} : plan_gemv(M, N, K, B, G, epilogue, sms);
  if (path == PATH_GEMV && !v.use) return CQ_ERR_UNSUPPORTED;
  if (v.use)
    return run_gemv(v, x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype, y,
                    stream, timeout_ns, trace);
  const GemmPlan g = plan_gemm(M, N, K, B, epilogue, sms);
  const size_t need = g.ws_counter_bytes + g.ws_partial_bytes;
  if (ws_bytes < need || (need && !workspace)) return CQ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return CQ_ERR_UNSUPPORTED;

  CUtensorMap map, wmap;
  st = encode_bf16_rows_sw128(&map, x, M, K, g.NT);
  if (st != CQ_OK) return st;
  st = encode_packed_rows(&wmap, packed, N, K * B / 8, B);
  if (st != CQ_OK) return st;

  EngineParams p = {};
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = G;
  p.mode = grid_mode;
  p.epilogue = epilogue;
  p.out_bf16 = out_dtype == CQ_DTYPE_BF16;
  p.n_rt = g.n_rt;
  p.spt = g.spt;
  p.num_tiles = g.tiles;
  p.P = g.P;
  p.mat.packed = packed;
  p.mat.scales = scales;
  p.mat.ab = reinterpret_cast<const uint32_t*>(ab);
  p.mat.B = B;
  p.M = static_cast<int>(M);
  p.n_tt = g.n_tt;
  p.y = y;
  p.ldy = epilogue == CQ_EPI_SWIGLU ? N / 2 : N;
  p.y_rows = M;
  p.partial_slots = 2 * g.P;
  p.counter_len = g.tiles;
  p.counter = reinterpret_cast<int*>(workspace);
  p.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + g.ws_counter_bytes);
  p.timeout_ns = timeout_ns;
  p.debug_skip_first_stage = debug_skip;
  p.trace = trace;

  switch (g.NT) {
    case 16: return launch_engine_te<16>(p, map, wmap, B, stream);
    case 32: return launch_engine_te<32>(p, map, wmap, B, stream);
    case 64: return launch_engine_te<64>(p, map, wmap, B, stream);
    case 128: return launch_engine_te<128>(p, map, wmap, B, stream);
    case 176: return launch_engine_te<176>(p, map, wmap, B, stream);
    default: return launch_engine_te<192>(p, map, wmap, B, stream);
  }
}

size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K, int B, int G, int epilogue,
                           int sms, int path = PATH_AUTO) {
  if (M <= 0 || N <= 0 || K <= 0 || K % kSlice != 0 || G <= 0 || G % kSlice != 0 ||
      K % G != 0 || M > (int64_t)1 << 24 || N > (int64_t)1 << 30 ||
      ((M + 15) / 16) * ((N + kRows - 1) / kRows) >= ((int64_t)1 << 31))
    return 0;                                     // cq_gemm rejects these shapes
  size_t counters = 0, total = 0;
  gemm_scratch(M, N, K, B, G, epilogue, sms, &counters, &total, path);
  return total;
}

}  // namespace cq

using namespace cq;

extern "C" size_t cq_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int B, int G,
                                         int epilogue) {
  int sms = num_sms();
  if (sms <= 0) sms = 148;
  return gemm_workspace_size(M, N, K, B, G, epilogue, sms);
}

extern "C" int cq_gemm(const uint16_t* x, int64_t M, const uint8_t* packed, const float* scales,
                       const uint16_t* ab, int64_t N, int64_t K, int B, int G, int grid_mode,
                       int epilogue, int out_dtype, void* y, void* workspace, size_t ws_bytes,
                       void* stream) {
  return gemm_impl(x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype, y,
                   workspace, ws_bytes, static_cast<cudaStream_t>(stream), kDefaultTimeoutNs, 0);
}

// ---------------------------------------------------------------------------
// host-buffer GEMM: the copy of x from page-locked host memory as a kernel
// chained to the GEMM by programmatic dependent launch (a copy-engine
// transfer before a kernel breaks the chain and adds its own start latency),
// and the GEMM's stores straight into a page-locked y
// ---------------------------------------------------------------------------
constexpr int kCopyThreads = 256;

// dst[0, bytes) = src[0, bytes); both 16-byte aligned.  Waits for the
// preceding grid before writing (the previous GEMM may still read dst, or
// the GEMM this copy follows may still write src).
__global__ void __launch_bounds__(kCopyThreads)
    host_copy_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int64_t bytes) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t n16 = bytes >> 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kCopyThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kCopyThreads + threadIdx.x; i < n16;
       i += stride)
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  if (blockIdx.x == 0 && threadIdx.x < (bytes & 15))
    dst[n16 * 16 + threadIdx.x] = src[n16 * 16 + threadIdx.x];
}

static int launch_host_copy(const void* src, void* dst, int64_t bytes, int sms, cudaStream_t s) {
  if (bytes <= 0) return CQ_OK;
  const int64_t n16 = (bytes + 15) >> 4;
  int64_t blocks = (n16 + kCopyThreads - 1) / kCopyThreads;
  if (blocks > sms) blocks = sms;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kCopyThreads);
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, host_copy_kernel, static_cast<const uint8_t*>(src),
                         static_cast<uint8_t*>(dst), bytes) != cudaSuccess)
    return CQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

// Whether p is page-locked host memory a kernel can address (registered or
// allocated by the runtime as pinned).
static bool device_addressable_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();                    // pageable memory may report an error: clear it
    return false;
  }
  return a.type == cudaMemoryTypeHost && a.devicePointer == p;
}

extern "C" int cq_gemm_host(const uint16_t* x_host, int64_t M, const uint8_t* packed,
                            const float* scales, const uint16_t* ab, int64_t N, int64_t K, int B,
                            int G, int grid_mode, int epilogue, int out_dtype, void* y_host,
                            uint16_t* x_dev, void* y_dev, void* workspace, size_t ws_bytes,
                            void* stream) {
  // every check before anything is queued
  int st = validate_gemm(x_dev, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue,
                         out_dtype, y_dev);
  if (st != CQ_OK) return st;
  if (M == 0 || N == 0) return CQ_OK;
  if (!x_host || !y_host) return CQ_ERR_INVALID_ARG;
  int sms = num_sms();
  if (sms <= 0) return CQ_ERR_CUDA;
  const size_t need = gemm_workspace_size(M, N, K, B, G, epilogue, sms);
  if (ws_bytes < need || (need && !workspace)) return CQ_ERR_WORKSPACE;
  if (need && !aligned(workspace, 16)) return CQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t x_bytes = static_cast<size_t>(M) * K * 2;
  const int64_t ncol = epilogue == CQ_EPI_SWIGLU ? N / 2 : N;
  const size_t y_bytes = static_cast<size_t>(M) * ncol * (out_dtype == CQ_DTYPE_BF16 ? 2 : 4);
  // page-locked buffers on both sides: three chained kernels; otherwise the
  // copy engine (the driver stages pageable memory itself)
  const bool kernels = aligned(x_host, 16) && aligned(y_host, 16) &&
                       device_addressable_host(x_host) && device_addressable_host(y_host);
  if (kernels) {
    st = launch_host_copy(x_host, x_dev, static_cast<int64_t>(x_bytes), sms, s);
  } else {
    st = cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, s) == cudaSuccess
             ? CQ_OK : CQ_ERR_CUDA;
  }
  if (st != CQ_OK) return st;
  // a page-locked y_host takes the GEMM's stores directly (every kernel only
  // stores to its output); otherwise y_dev is staged and copied back
  st = gemm_impl(x_dev, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype,
                 kernels ? y_host : y_dev, workspace, ws_bytes, s, kDefaultTimeoutNs, 0);
  if (st != CQ_OK || kernels) return st;
  return cudaMemcpyAsync(y_host, y_dev, y_bytes, cudaMemcpyDeviceToHost, s) == cudaSuccess
             ? CQ_OK : CQ_ERR_CUDA;
}

// Profiling hook (declared in cq_hooks.h): cq_gemm that also writes per-CTA
// event timestamps to trace ([grid][64] uint64 words of device memory).
extern "C" CQ_API int cq_trace_gemm(const uint16_t* x, int64_t M, const uint8_t* packed,
                                    const float* scales, const uint16_t* ab, int64_t N,
                                    int64_t K, int B, int G, int epilogue, void* y,
                                    void* workspace, size_t ws_bytes, uint64_t* trace,
                                    void* stream) {
  return gemm_impl(x, M, packed, scales, ab, N, K, B, G, CQ_GRID_MIDRISE, epilogue,
                   CQ_DTYPE_F32, y, workspace, ws_bytes, static_cast<cudaStream_t>(stream),
                   kDefaultTimeoutNs, 0, trace);
}

// Test hook (declared in cq_hooks.h): cq_gemm with a chosen wait limit and,
// optionally, with the first stage loads withheld so that the bounded waits
// run out; the caller then reads CQ_ERR_TIMEOUT from cq_get_device_error().
extern "C" CQ_API int cq_test_gemm_bounded(const uint16_t* x, int64_t M, const uint8_t* packed,
                                    const float* scales, const uint16_t* ab, int64_t N, int64_t K,
                                    int B, int G, void* y, void* workspace, size_t ws_bytes,
                                    uint64_t timeout_ns, int skip_first_stage, void* stream) {
  return gemm_impl(x, M, packed, scales, ab, N, K, B, G, CQ_GRID_MIDRISE, CQ_EPI_NONE,
                   CQ_DTYPE_F32, y, workspace, ws_bytes, static_cast<cudaStream_t>(stream),
                   timeout_ns, skip_first_stage);
}

// Test hook (declared in cq_hooks.h): cq_gemm on a chosen kernel, and the
// workspace that choice needs.
extern "C" CQ_API size_t cq_test_gemm_path_workspace_size(int64_t M, int64_t N, int64_t K, int B,
                                                         int G, int epilogue, int path) {
  int sms = num_sms();
  if (sms <= 0) sms = 148;
  return gemm_workspace_size(M, N, K, B, G, epilogue, sms, path);
}

extern "C" CQ_API int cq_test_gemm_path(const uint16_t* x, int64_t M, const uint8_t* packed,
                                        const float* scales, const uint16_t* ab, int64_t N,
                                        int64_t K, int B, int G, int grid_mode, int epilogue,
                                        int out_dtype, void* y, void* workspace, size_t ws_bytes,
                                        int path, void* stream) {
  if (path < PATH_AUTO || path > PATH_ENGINE) return CQ_ERR_INVALID_ARG;
  return gemm_impl(x, M, packed, scales, ab, N, K, B, G, grid_mode, epilogue, out_dtype, y,
                   workspace, ws_bytes, static_cast<cudaStream_t>(stream), kDefaultTimeoutNs, 0,
                   nullptr, path);
}
