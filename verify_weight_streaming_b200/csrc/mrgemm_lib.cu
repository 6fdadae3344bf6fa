// The whole library is one translation unit, so the device-side error word
// has exactly one definition shared by every kernel.
#include "api.cu"
#include "mrgemv.cu"
#include "router_topk.cu"
#include "gemm_f16.cu"
#include "cast_bf16.cu"
