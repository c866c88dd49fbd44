// Decode-attention kernels for head dimension 256 (all b, query-row and QJL variants).
#include "octo_decode_kernel.cuh"

namespace octo {

cudaError_t launch_decode_d256(const DecodeArgs& a, const TmaDesc& tm, int b, int G, bool qjl, dim3 grid, cudaStream_t st) {
  return launch_decode_d<256>(a, tm, b, G, qjl, grid, st);
}

}  // namespace octo
