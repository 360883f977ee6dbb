// multiquery_fp8.cu -- the mma.sync multi-query kernel over fp8 (E4M3) caches.
#include "multiquery_launch.cuh"

namespace pkv {

cudaError_t launch_multiquery_mma_fp8(const CUtensorMap& kmap, const CUtensorMap& vmap, const MultiQueryParams& p,
                                      int group, int rows_per_seq, bool reduce, cudaStream_t st) {
  return launch_multiquery_mma_t<true>(kmap, vmap, p, group, rows_per_seq, reduce, st);
}

}  // namespace pkv
