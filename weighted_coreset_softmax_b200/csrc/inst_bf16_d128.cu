// Kernel instantiations for element type bf16, head dimension 128.
#define KVS_T __nv_bfloat16
#define KVS_D 128
#define KVS_SUFFIX bf16_d128
#include "instantiate.cuh"
