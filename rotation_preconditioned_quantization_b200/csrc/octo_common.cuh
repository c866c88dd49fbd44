// Device helpers shared by the encode and decode kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/octopus.h"

namespace octo {

constexpr int kWarp = 32;

// Launch set-up that does not change between calls of one kernel on one
// device: the dynamic shared-memory opt-in and the number of blocks that can
// be resident at once (SMs x blocks per SM). Each launcher keeps one cache per
// kernel instantiation; the first call on a device fills its entry.
constexpr int kLaunchCacheDevices = 64;
struct LaunchCache {
  std::atomic<int> resident[kLaunchCacheDevices];  // 0: not known yet
};

template <typename Kern>
inline cudaError_t launch_setup(Kern kern, LaunchCache& c, int threads, size_t smem, int& resident) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < kLaunchCacheDevices;
  int v = cached ? c.resident[dev].load(std::memory_order_acquire) : 0;
  if (v == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (e != cudaSuccess) return e;
    v = sms * (per_sm > 0 ? per_sm : 1);
    if (cached) c.resident[dev].store(v, std::memory_order_release);
  }
  resident = v;
  return cudaSuccess;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Walsh-Hadamard butterflies (Sylvester order) on a vector of D values held
// E = D/32 per lane, lane l owning coordinates [l*E, l*E + E). Unnormalised.
// The explainer ("engineering implementation") describes the encoder's WHT as
// an in-place Kronecker-factored butterfly: here the E-point factor runs in
// registers and the 32-point factor across lanes with shuffles.
template <int E>
__device__ __forceinline__ void fwht_warp(float (&v)[E], int lane) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if ((e & h) == 0) {
        const float a = v[e], b = v[e + h];
        v[e] = a + b;
        v[e + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    // lower lane: v + o, upper lane: o - v, as one fma with a +-1 factor
    // (the product is exact, so the result is the correctly rounded sum)
    const float sg = (lane & m) != 0 ? -1.0f : 1.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = fmaf(sg, v[e], __shfl_xor_sync(0xffffffffu, v[e], m));
  }
}

// Inverse octahedral map of (a, b) = (xi, eta), normalised (explainer,
// "octahedral folding": r = 1 - |xi| - |eta|; unfold when r < 0; normalise).
__device__ __forceinline__ float3 oct_inverse(float a, float b) {
  const float r = 1.0f - fabsf(a) - fabsf(b);
  float x = a, y = b;
  if (r < 0.0f) {
    x = copysignf(1.0f - fabsf(b), a);
    y = copysignf(1.0f - fabsf(a), b);
    // sgn(0) = +1 (copysignf keeps +0's positive sign; -0 cannot reach here
    // from a centroid table)
  }
  const float inv = 1.0f / sqrtf(x * x + y * y + r * r);
  return make_float3(x * inv, y * inv, r * inv);
}

// Ordered codebook cells (ix, iy) of a code's 2(B+1)-bit direction field
// m_x | m_y << B | s_x << 2B | s_y << (2B + 1): a cell is stored as its
// sign (1 = lower half, negative levels) and the rank m of |level| among the
// positive levels of the odd-symmetric codebook.
template <int B>
__device__ __forceinline__ void direction_cells(uint32_t field, int& ix, int& iy) {
  constexpr uint32_t half = 1u << B, ones = (2u << B) - 1u;
  const uint32_t mx = field & (half - 1u), my = (field >> B) & (half - 1u);
  const uint32_t sx = (field >> (2 * B)) & 1u, sy = (field >> (2 * B + 1)) & 1u;
  ix = static_cast<int>((half | mx) ^ (sx ? ones : 0u));
  iy = static_cast<int>((half | my) ^ (sy ? ones : 0u));
}

}  // namespace octo
