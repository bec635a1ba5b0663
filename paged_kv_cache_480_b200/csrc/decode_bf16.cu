// Decode and merge kernels instantiated for one element type.
#include "decode_launch.cuh"

PKV_DEFINE_DTYPE(bf16, __nv_bfloat16)
