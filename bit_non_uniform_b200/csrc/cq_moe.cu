// cq_moe.cu -- grouped MoE entry points (routing, grouped GEMMs, combine).
#include <cuda_runtime.h>

#include "cq.h"

extern "C" size_t cq_moe_workspace_size(int64_t T, int k, int E, int64_t H, int64_t I, int G) {
  (void)T; (void)k; (void)E; (void)H; (void)I; (void)G;
  return 0;
}

extern "C" int cq_moe_grouped_gemm(const uint16_t* tokens, int64_t T, const int32_t* topk_ids,
                                   const float* topk_w, int k, int E,
                                   const cq_expert_desc* experts, int64_t H, int64_t I, int G,
                                   int grid_mode, int out_dtype, void* route_out, void* out,
                                   void* workspace, size_t ws_bytes, void* stream) {
  (void)tokens; (void)T; (void)topk_ids; (void)topk_w; (void)k; (void)E; (void)experts;
  (void)H; (void)I; (void)G; (void)grid_mode; (void)out_dtype; (void)route_out; (void)out;
  (void)workspace; (void)ws_bytes; (void)stream;
  return CQ_ERR_UNSUPPORTED;
}
