// Single translation unit for libmoe_fp8.so: one copy of the device error
// word and of the host-side caches.
#include "quant.cu"
#include "route.cu"
#include "permute.cu"
#include "permute_noalloc.cu"
#include "gemm.cu"
#include "combine.cu"
#include "ep.cu"
#include "backward.cu"
