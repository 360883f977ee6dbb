// decode_bf16_fp8.cu -- decode kernel instances for q __nv_bfloat16, cache __nv_fp8_e4m3.
#include "decode_launch.cuh"

PKV_DEFINE_DECODE(launch_decode_bf16_fp8, __nv_bfloat16, __nv_fp8_e4m3)
