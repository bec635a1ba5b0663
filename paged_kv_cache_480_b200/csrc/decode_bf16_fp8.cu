// Decode kernels for bf16 q and out over an FP8 (E4M3) cache.
#include "decode_launch.cuh"

PKV_DEFINE_TYPES(bf16_fp8, __nv_bfloat16, fp8e4m3)
