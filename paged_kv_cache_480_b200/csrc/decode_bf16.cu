// Decode and merge kernels for bf16 q, out and caches.
#include "decode_launch.cuh"

PKV_DEFINE_TYPES(bf16, __nv_bfloat16, __nv_bfloat16)
PKV_DEFINE_MERGE(bf16, __nv_bfloat16)
