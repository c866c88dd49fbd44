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

// Packed fp32 pairs (sm_100 add/sub/mul/fma .f32x2): one instruction does
// the two lanes' IEEE round-to-nearest operations, so results are the same
// as with scalar operations.
#define OCTO_F32X2_OP(name, op)                                                                         \
  __device__ __forceinline__ float2 name(float2 a, float2 b) {                                         \
    float2 d;                                                                                           \
    asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n " op           \
        ".rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"                                            \
        : "=f"(d.x), "=f"(d.y)                                                                          \
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));                                                      \
    return d;                                                                                           \
  }
OCTO_F32X2_OP(add_f32x2, "add")
OCTO_F32X2_OP(sub_f32x2, "sub")
OCTO_F32X2_OP(mul_f32x2, "mul")
#undef OCTO_F32X2_OP
__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rc, {%6, %7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// Walsh-Hadamard butterflies over the 32 register coordinates of a lane
// (coordinate bits 0-4, Sylvester order): the stage over bit 0 pairs
// neighbouring registers and runs scalar; the stages over bits 1-4 pair
// register pairs (2i, 2i+1), two butterflies per packed add and sub.
__device__ __forceinline__ void fwht32_regs(float (&v)[32]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float a = v[e], b = v[e + 1];
    v[e] = a + b;
    v[e + 1] = a - b;
  }
#pragma unroll
  for (int hh = 2; hh < 32; hh <<= 1) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      if ((e & hh) == 0) {
        const float2 a = make_float2(v[e], v[e + 1]), b = make_float2(v[e + hh], v[e + hh + 1]);
        const float2 s = add_f32x2(a, b), d = sub_f32x2(a, b);
        v[e] = s.x; v[e + 1] = s.y; v[e + hh] = d.x; v[e + hh + 1] = d.y;
      }
    }
  }
}

// The butterfly stages across the LK lanes of a key, lane j of the key
// being lane j * STRIDE of the warp (lane bits log2(STRIDE) and up): lower
// lane v + o, upper lane o - v, as fma(+-1, v, o) on register pairs.
template <int LK, int STRIDE>
__device__ __forceinline__ void fwht32_lanes(float (&v)[32], int lane) {
#pragma unroll
  for (int m = STRIDE; m < LK * STRIDE; m <<= 1) {
    const float sg = (lane & m) != 0 ? -1.0f : 1.0f;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, v[e], m), __shfl_xor_sync(0xffffffffu, v[e + 1], m));
      const float2 r = fma_f32x2(make_float2(sg, sg), make_float2(v[e], v[e + 1]), o);
      v[e] = r.x; v[e + 1] = r.y;
    }
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
