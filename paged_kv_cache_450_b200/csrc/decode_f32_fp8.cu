// decode_f32_fp8.cu -- decode kernel instances for q float, cache __nv_fp8_e4m3.
#include "decode_launch.cuh"

PKV_DEFINE_DECODE(launch_decode_f32_fp8, float, __nv_fp8_e4m3)
