// Kernel instantiations for element type f32, head dimension 64.
#define KVS_T float
#define KVS_D 64
#define KVS_SUFFIX f32_d64
#include "instantiate.cuh"
