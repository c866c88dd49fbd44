// octo_decode_attn_static: the decode step for callers that cannot allocate
// device memory (see octopus.h). The split-merge scratch lives in a fixed
// file-scope device array; nothing here calls cudaMalloc or cudaFree.

#include <cuda_runtime.h>

#include <mutex>

#include "../../include/octopus.h"

namespace {

// The scratch: status word, arrival counters and split partials of
// octo_decode_attn, reserved on every device that loads this library.
__device__ __align__(256) unsigned char g_static_scratch[OCTO_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device. In host code the
// array's name only stands for the symbol; the address a kernel may use
// comes from cudaGetSymbolAddress, looked up once per device with that
// device current.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OCTO_ECUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return OCTO_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return OCTO_OK;
}

}  // namespace

extern "C" int octo_decode_attn_static(const octo_layout* L, const octo_tables* tables, const void* q, int q_dtype,
                                       int B, int Hq, int Hkv, int Lq, int64_t kv_len, int64_t cache_cap,
                                       const uint32_t* packed, const float* gamma, const uint32_t* qjl_bits,
                                       const float* qjl_norm, const void* V, float scale, float* out, float* logits,
                                       octo_stream_t stream) {
  const size_t need = octo_decode_attn_workspace(L, B, Hq, Hkv, Lq, kv_len);
  if (need == 0) {  // sizes the decode step rejects: too many query rows per KV head, or invalid
    const bool shaped = L && B >= 1 && Hkv >= 1 && Hq >= Hkv && Hq % Hkv == 0 && Lq >= 1;
    return shaped && (Hq / Hkv) * Lq > 8 ? OCTO_EUNSUPPORTED : OCTO_EINVAL;
  }
  if (need > OCTO_STATIC_SCRATCH_BYTES) return OCTO_EWORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != OCTO_OK) return rc;
  // the status word (bytes [0, 256)) and the arrival counters (bytes
  // [256, 256 + 4*B*Hkv)) must start at zero; the array keeps whatever the
  // previous call left
  const size_t zero = 256 + ((sizeof(int) * static_cast<size_t>(B) * Hkv + 255) / 256) * 256;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, zero, st) != cudaSuccess) return OCTO_ECUDA;
  return octo_decode_attn(L, tables, q, q_dtype, B, Hq, Hkv, Lq, kv_len, cache_cap, packed, gamma, qjl_bits,
                          qjl_norm, V, scale, out, logits, scratch, OCTO_STATIC_SCRATCH_BYTES, stream);
}
