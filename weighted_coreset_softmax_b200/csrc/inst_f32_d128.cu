// Kernel instantiations for element type f32, head dimension 128.
#define KVS_T float
#define KVS_D 128
#define KVS_SUFFIX f32_d128
#include "instantiate.cuh"
