// decode_bf16_bf16.cu -- decode kernel instances for q __nv_bfloat16, cache __nv_bfloat16.
#include "decode_launch.cuh"

PKV_DEFINE_DECODE(launch_decode_bf16_bf16, __nv_bfloat16, __nv_bfloat16)
