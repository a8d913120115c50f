// Kernel instantiations for element type bf16, head dimension 64.
#define KVS_T __nv_bfloat16
#define KVS_D 64
#define KVS_SUFFIX bf16_d64
#include "instantiate.cuh"
