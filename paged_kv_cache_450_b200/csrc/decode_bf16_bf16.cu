// decode_bf16_bf16.cu -- decode kernel instances for q __nv_bfloat16, cache __nv_bfloat16.
#include "decode_launch.cuh"

PKV_DEFINE_DECODE(launch_decode_bf16_bf16, __nv_bfloat16, __nv_bfloat16)

namespace pkv {

cudaError_t launch_decode_shared_prefix_bf16(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                                             int group, int num_kv_heads, int grid_partitions, cudaStream_t st) {
  cudaError_t e;
  switch (p.block_size) {
    case 16: e = dispatch_grouped_group<16>(kmap, vmap, p, group, num_kv_heads, grid_partitions, st); break;
    case 32: e = dispatch_grouped_group<32>(kmap, vmap, p, group, num_kv_heads, grid_partitions, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_reduce<__nv_bfloat16, 128>(p, st);
}

}  // namespace pkv
