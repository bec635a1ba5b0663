// Decode kernels for f32 q and out over an FP8 (E4M3) cache.
#include "decode_launch.cuh"

PKV_DEFINE_TYPES(f32_fp8, float, fp8e4m3)
