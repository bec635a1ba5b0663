// Decode kernels for f16 q and out over an FP8 (E4M3) cache.
#include "decode_launch.cuh"

PKV_DEFINE_TYPES(f16_fp8, __half, fp8e4m3)
