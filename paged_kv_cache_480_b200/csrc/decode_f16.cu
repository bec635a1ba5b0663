// Decode and merge kernels for f16 q, out and caches.
#include "decode_launch.cuh"

PKV_DEFINE_TYPES(f16, __half, __half)
PKV_DEFINE_MERGE(f16, __half)
