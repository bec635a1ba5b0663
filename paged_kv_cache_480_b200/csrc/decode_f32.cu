// Decode and merge kernels for f32 q, out and caches.
#include "decode_launch.cuh"

PKV_DEFINE_TYPES(f32, float, float)
PKV_DEFINE_MERGE(f32, float)
