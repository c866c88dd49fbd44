// octo_decode_attn_static: the decode step for callers that cannot allocate
// device memory (see octopus.h). The split-merge scratch lives in a fixed
// file-scope device array; nothing here calls cudaMalloc or cudaFree.

#include <cuda_runtime.h>

#include <mutex>

#include "../../include/octopus.h"
#include "octo_decode_check.h"

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
  // octo_decode_attn's own checks first (same codes, same order): a rejected
  // call touches neither the GPU nor the shared array
  size_t need = 0;
  const int vc = octo::decode_validate(L, tables, q, q_dtype, B, Hq, Hkv, Lq, kv_len, cache_cap, packed, gamma,
                                       qjl_bits, qjl_norm, V, scale, out, logits, &need);
  if (vc != OCTO_OK) return vc;
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

extern "C" int octo_decode_attn_static_status(int* status, octo_stream_t stream) {
  if (!status) return OCTO_EINVAL;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != OCTO_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyAsync(&word, scratch, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return OCTO_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return OCTO_ECUDA;
  *status = word;
  return OCTO_OK;
}

extern "C" int octo_decode_attn_static_fill(int byte, octo_stream_t stream) {
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != OCTO_OK) return rc;
  const cudaError_t e = cudaMemsetAsync(scratch, byte & 0xff, OCTO_STATIC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? OCTO_OK : OCTO_ECUDA;
}
