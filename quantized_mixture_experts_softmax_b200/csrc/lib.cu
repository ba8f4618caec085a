// Single translation unit of the CUDA library (libmoe.so): the kernels share the device
// status word and helpers without relocatable device code.
#include "route_align.cu"
#include "permute_combine.cu"
#include "gemm_w4a16.cu"
#include "gemm_fp8.cu"
#include "gemm_w4i8.cu"
#include "gemm_mx.cu"
#include "api.cu"
#include "align_noalloc.cu"
