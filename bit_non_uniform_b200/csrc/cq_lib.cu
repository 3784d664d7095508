// cq_lib.cu -- libcq is compiled as one translation unit so that the device
// error word and the kernels share one module without relocatable device code.
#include "cq_api.cu"
#include "cq_gemm.cu"
#include "cq_moe.cu"
#include "cq_noalloc.cu"
#include "cq_a8.cu"
