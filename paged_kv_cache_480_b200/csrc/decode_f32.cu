// Decode and merge kernels instantiated for one element type.
#include "decode_launch.cuh"

PKV_DEFINE_DTYPE(f32, float)
