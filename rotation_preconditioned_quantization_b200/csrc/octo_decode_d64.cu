// Decode-attention kernels for head dimension 64 (all b, query-row and QJL variants).
#include "octo_decode_kernel.cuh"

namespace octo {

cudaError_t launch_decode_d64(const DecodeArgs& a, const TmaDesc& tm, int b, int G, bool qjl, dim3 grid, cudaStream_t st) {
  return launch_decode_d<64>(a, tm, b, G, qjl, grid, st);
}

}  // namespace octo
