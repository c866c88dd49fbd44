// OCTOPUS fused decode attention: host entry points (argument checks,
// split planning, workspace carve-up, dispatch to the per-D kernels).

#include <cuda_runtime.h>

#include <algorithm>

#include "octo_decode_kernel.cuh"

namespace octo {

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return sms;
}

// Split the cache of each head into n_splits contiguous slices so that the
// grid (heads x splits) fills the SMs in whole waves: minimise
// ceil(heads * s / sms) / s over s, slices of at least 256 keys.
static void choose_splits(int64_t heads, int64_t kv_len, int sms, int& n_splits, int64_t& per) {
  const int64_t max_s = std::max<int64_t>(1, std::min<int64_t>(1024, (kv_len + 255) / 256));
  double best = 1e300;
  int64_t best_s = 1;
  for (int64_t s = 1; s <= max_s; ++s) {
    const int64_t waves = (heads * s + sms - 1) / sms;
    const double cost = static_cast<double>(waves) / s + 1e-4 * s;  // tiny bias against needless splits
    if (cost < best - 1e-12) { best = cost; best_s = s; }
  }
  per = (kv_len + best_s - 1) / best_s;
  per = ((per + 63) / 64) * 64;  // slices start at multiples of 64 keys (16-byte aligned copies)
  n_splits = static_cast<int>(std::max<int64_t>(1, (kv_len + per - 1) / per));
}

static int rows_template(int Gq) { return Gq <= 1 ? 1 : (Gq <= 4 ? 4 : 8); }

}  // namespace octo

namespace {

// Workspace: a status word (own 256-byte line), the per-head arrival
// counters, then the per-split (m, l) and O partials.
struct WsLayout {
  size_t status, counters, m, l, o, total;
};

WsLayout ws_layout(int64_t heads, int n_splits, int G, int D) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  WsLayout w{};
  w.status = 0;
  w.counters = 256;
  w.m = w.counters + up(sizeof(int) * heads);
  w.l = w.m + up(sizeof(float) * heads * n_splits * G);
  w.o = w.l + up(sizeof(float) * heads * n_splits * G);
  w.total = w.o + up(sizeof(float) * heads * n_splits * G * D);
  return w;
}

int check_layout(const octo_layout* L) {
  if (!L) return OCTO_EINVAL;
  if (L->d != 64 && L->d != 128 && L->d != 256) return OCTO_EUNSUPPORTED;
  if (L->b < 2 || L->b > 4) return OCTO_EUNSUPPORTED;
  octo_layout chk;
  if (octo_layout_init(&chk, L->d, L->b, L->qjl, L->rounding) != OCTO_OK) return OCTO_EINVAL;
  if (chk.words != L->words || chk.T != L->T || chk.code_bits != L->code_bits) return OCTO_EINVAL;
  return OCTO_OK;
}

}  // namespace

extern "C" size_t octo_decode_attn_workspace(const octo_layout* L, int B, int Hq, int Hkv, int Lq, int64_t kv_len) {
  if (check_layout(L) != OCTO_OK) return 0;
  if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || Lq < 1 || kv_len < 0) return 0;
  const int Gq = (Hq / Hkv) * Lq;
  if (Gq > 8) return 0;
  const int G = octo::rows_template(Gq);
  int n_splits;
  int64_t per;
  octo::choose_splits(static_cast<int64_t>(B) * Hkv, std::max<int64_t>(kv_len, 1), octo::sm_count(), n_splits, per);
  return ws_layout(static_cast<int64_t>(B) * Hkv, n_splits, G, L->d).total;
}

extern "C" int octo_decode_attn(const octo_layout* L, const octo_tables* tab, const void* q, int q_dtype, int B,
                                int Hq, int Hkv, int Lq, int64_t kv_len, int64_t cache_cap,
                                const uint32_t* packed, const float* gamma, const uint32_t* qjl_bits,
                                const float* qjl_norm, const void* V, float scale, float* out, float* logits,
                                void* workspace, size_t ws_bytes, octo_stream_t stream) {
  const int lc = check_layout(L);
  if (lc != OCTO_OK) return lc;
  if (!tab || !q || !packed || !gamma || !tab->dir_c || !tab->rho_c || !tab->signs || tab->n_heads < 1)
    return OCTO_EINVAL;
  if (q_dtype != OCTO_F32 && q_dtype != OCTO_BF16) return OCTO_EINVAL;
  if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || Lq < 1) return OCTO_EINVAL;
  if (kv_len < 0 || cache_cap < 0 || kv_len > cache_cap) return OCTO_EINVAL;
  if (!V && !logits) return OCTO_EINVAL;
  if (V && !out) return OCTO_EINVAL;
  if (L->qjl && (!qjl_bits || !qjl_norm || !tab->qjl_S)) return OCTO_EINVAL;
  auto misaligned = [](const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 != 0; };
  if (V && misaligned(V)) return OCTO_EINVAL;
  // code rows are staged by 16-byte bulk copies
  if (cache_cap % 4 != 0 || misaligned(packed) || misaligned(gamma)) return OCTO_EINVAL;
  if (L->qjl && (misaligned(qjl_bits) || misaligned(qjl_norm))) return OCTO_EINVAL;
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return OCTO_EINVAL;
  if (!(scale == scale)) return OCTO_EINVAL;
  const int g = Hq / Hkv, Gq = g * Lq;
  if (Gq > 8) return OCTO_EUNSUPPORTED;
  if (static_cast<int64_t>(B) * Hkv > 65535) return OCTO_EUNSUPPORTED;  // grid.y limit
  const int D = L->d;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t heads = static_cast<int64_t>(B) * Hkv;

  if (kv_len == 0) {
    if (V) {
      const cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * static_cast<size_t>(B) * Hq * Lq * D, st);
      return e == cudaSuccess ? OCTO_OK : OCTO_ECUDA;
    }
    return OCTO_OK;
  }

  octo::DecodeArgs a{};
  a.q = q;
  a.q_bf16 = q_dtype == OCTO_BF16;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Lq = Lq; a.g = g; a.Gq = Gq;
  a.kv_len = kv_len;
  a.cache_cap = cache_cap;
  a.packed = packed;
  a.gamma = gamma;
  a.qjl_bits = qjl_bits;
  a.qjl_norm = qjl_norm;
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = out;
  a.logits = logits;
  a.dir_c = tab->dir_c;
  a.rho_c = tab->rho_c;
  a.signs = tab->signs;
  a.qjl_S = tab->qjl_S;
  a.table_heads = tab->n_heads;
  const int G = octo::rows_template(Gq);

  octo::choose_splits(heads, kv_len, octo::sm_count(), a.n_splits, a.keys_per_split);
  const WsLayout w = ws_layout(heads, a.n_splits, G, D);
  if (ws_bytes < w.total) return OCTO_EWORKSPACE;
  char* base = static_cast<char*>(workspace);
  a.status = reinterpret_cast<int*>(base + w.status);
  a.counters = reinterpret_cast<int*>(base + w.counters);
  a.part_m = reinterpret_cast<float*>(base + w.m);
  a.part_l = reinterpret_cast<float*>(base + w.l);
  a.part_o = reinterpret_cast<float*>(base + w.o);
  const dim3 grid(static_cast<unsigned>(a.n_splits), static_cast<unsigned>(heads));
  cudaError_t e;
  switch (D) {
    case 64: e = octo::launch_decode_d64(a, L->b, G, L->qjl != 0, grid, st); break;
    case 128: e = octo::launch_decode_d128(a, L->b, G, L->qjl != 0, grid, st); break;
    default: e = octo::launch_decode_d256(a, L->b, G, L->qjl != 0, grid, st); break;
  }
  return e == cudaSuccess ? OCTO_OK : OCTO_ECUDA;
}
