// decode_f32_f32.cu -- decode kernel instances for q float, cache float.
#include "decode_launch.cuh"

PKV_DEFINE_DECODE(launch_decode_f32_f32, float, float)
