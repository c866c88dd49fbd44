// OCTOPUS fused decode attention: host entry points (argument checks,
// split planning, workspace carve-up, dispatch to the per-D kernels).

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstring>

#include "octo_decode_check.h"
#include "octo_decode_kernel.cuh"

namespace octo {

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int sm_count() {
  static std::atomic<int> known[kLaunchCacheDevices];  // 0: not queried yet
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const bool cached = dev >= 0 && dev < kLaunchCacheDevices;
  if (cached && (sms = known[dev].load(std::memory_order_relaxed)) > 0) return sms;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  if (cached) known[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

// Split the cache of each head into n_splits contiguous slices. A CTA
// (one per SM) pays a fixed cost (prologue, first data, split merge: about
// 8 us measured on B200) plus its slice's bytes at about 30 GB/s per SM, and
// CTAs run in waves of the SM count; pick the split count that minimises
//   waves(s) * (fixed + (kv_len / s) * unit_bytes / per_sm_rate).
// Slices start at multiples of 16 keys (one consumer chunk of the kernels).
static void choose_splits(int64_t heads, int64_t kv_len, int sms, int64_t unit_bytes, int& n_splits,
                          int64_t& per) {
  constexpr double kFixedUs = 8.0, kBytesPerUs = 30.0e3;
  const int64_t max_s = std::max<int64_t>(1, std::min<int64_t>(1024, (kv_len + 63) / 64));
  double best = 1e300;
  int64_t best_s = 1;
  for (int64_t s = 1; s <= max_s; ++s) {
    const int64_t waves = (heads * s + sms - 1) / sms;
    const double keys = static_cast<double>((kv_len + s - 1) / s);
    const double cost = static_cast<double>(waves) * (kFixedUs + keys * static_cast<double>(unit_bytes) / kBytesPerUs);
    if (cost < best * (1.0 - 1e-9)) { best = cost; best_s = s; }
  }
  per = (kv_len + best_s - 1) / best_s;
  per = ((per + 15) / 16) * 16;  // slices start on 16-key boundaries (the copies need 4)
  n_splits = static_cast<int>(std::max<int64_t>(1, (kv_len + per - 1) / per));
}

// The slice plan of a call. When the CTAs span several waves and the last
// one is partly empty, some heads take one slice more (so smaller slices)
// until the CTAs fill whole waves: heads [0, heads_lo) keep n_lo slices of
// per_lo keys, heads [heads_lo, heads) take n slices of per keys. Blocks are
// dispatched in grid order as SMs free up, so the larger slices (lower
// heads) start first and the smaller ones fill in behind them.
struct SplitPlan {
  int n;
  int64_t per;
  int heads_lo, n_lo;
  int64_t per_lo;
};

static SplitPlan plan_splits(int64_t heads, int64_t kv_len, int sms, int64_t unit_bytes) {
  int n;
  int64_t per;
  choose_splits(heads, kv_len, sms, unit_bytes, n, per);
  SplitPlan p{n, per, 0, n, per};
  const int64_t ctas = heads * n, rem = ctas % sms;
  if (kv_len > 0 && ctas > sms && rem != 0 && sms - rem < heads) {
    const int64_t per_hi = ((kv_len + n) / (n + 1) + 15) / 16 * 16;
    if ((kv_len + per_hi - 1) / per_hi == n + 1)
      p = SplitPlan{n + 1, per_hi, static_cast<int>(heads - (sms - rem)), n, per};
  }
  return p;
}

// Bytes one (token, KV head) costs decode: code words, gamma, V row (and
// the sketch words and residual norm).
static int64_t unit_bytes(const octo_layout* L) {
  return 4 * L->words + 4 + 2 * L->d + (L->qjl ? 4 * (L->d / 32) + 4 : 0);
}

static int rows_template(int Gq) { return Gq <= 1 ? 1 : (Gq <= 4 ? 4 : 8); }

}  // namespace octo

namespace {

// Workspace: a status word (own 256-byte line), the per-head arrival
// counters, then the per-split (m, l) and O partials.
struct WsLayout {
  size_t status, counters, m, l, o, prep, total;
};

// Floats per head of the OCTOPUS-QJL query preparation (the tensor-core
// kernel's query scratch image: G rotated rows of tc_qrow(d) floats, then
// p = S q_rot, G rows of d floats); none otherwise.
int64_t prep_floats(bool qjl, int G, int D) {
  return qjl && D <= 128 ? static_cast<int64_t>(G) * (octo::tc_qrow(D) + D) : 0;
}

WsLayout ws_layout(int64_t heads, int n_splits, int G, int D, bool qjl) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  WsLayout w{};
  w.status = 0;
  w.counters = 256;
  w.m = w.counters + up(sizeof(int) * heads);
  w.l = w.m + up(sizeof(float) * heads * n_splits * G);
  w.o = w.l + up(sizeof(float) * heads * n_splits * G);
  w.prep = w.o + up(sizeof(float) * heads * n_splits * G * D);
  w.total = w.prep + up(sizeof(float) * heads * prep_floats(qjl, G, D));
  return w;
}

int check_layout(const octo_layout* L) {
  if (!L) return OCTO_EINVAL;
  if (L->d != 64 && L->d != 128 && L->d != 256) return OCTO_EUNSUPPORTED;
  if (L->b < 2 || L->b > 4) return OCTO_EUNSUPPORTED;
  if (L->b_dir != L->b + 1 || L->b_rho != L->b - 1) return OCTO_EUNSUPPORTED;  // fused decode: the OCTOPUS split
  octo_layout chk;
  if (octo_layout_init(&chk, L->d, L->b, L->qjl, L->rounding) != OCTO_OK) return OCTO_EINVAL;
  if (chk.words != L->words || chk.T != L->T || chk.code_bits != L->code_bits) return OCTO_EINVAL;
  return OCTO_OK;
}

// ---- tensor maps of the tensor-core kernel (host) ----------------------------
// The encoder comes from the driver through the runtime's entry-point query,
// so the library needs no link against the driver library.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType type, cuuint32_t rank, const void* base, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle) {
  const auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint32_t elem[3] = {1, 1, 1};
  return enc(m, type, rank, const_cast<void*>(base), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token extents are kv_len (not the capacity), so boxes that run past the
// last token arrive zero-filled.
bool build_maps(octo::TmaDesc& tm, const octo_layout* L, int64_t heads, int64_t kv_len, int64_t cap,
                const uint32_t* packed, const float* gamma, const uint32_t* qjl_bits, const float* qjl_norm,
                const void* V) {
  std::memset(&tm, 0, sizeof(tm));
  const cuuint64_t kv = static_cast<cuuint64_t>(kv_len), H = static_cast<cuuint64_t>(heads);
  const cuuint64_t row = static_cast<cuuint64_t>(cap) * 4;  // bytes between token rows of a plane
  const cuuint32_t KW = 16, RK = static_cast<cuuint32_t>(octo::tc_round_keys(L->d, L->b));
  const int W = L->words, QW = L->d / 32, D = L->d;
  {
    const cuuint64_t dims[3] = {kv, static_cast<cuuint64_t>(W), H}, str[2] = {row, row * W};
    const cuuint32_t box[3] = {KW, static_cast<cuuint32_t>(W), 1};
    if (!make_map(&tm.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, packed, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  {
    const cuuint64_t dims[2] = {kv, H}, str[1] = {row};
    const cuuint32_t box[2] = {RK, 1};
    if (!make_map(&tm.gamma, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, gamma, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
    if (L->qjl &&
        !make_map(&tm.qnorm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, qjl_norm, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  if (L->qjl) {
    const cuuint64_t dims[3] = {kv, static_cast<cuuint64_t>(QW), H}, str[2] = {row, row * QW};
    const cuuint32_t box[3] = {RK, static_cast<cuuint32_t>(QW), 1};
    if (!make_map(&tm.qbits, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, qjl_bits, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  if (V) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), kv, H};
    const cuuint64_t str[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(cap) * D * 2};
    const cuuint32_t box[3] = {64, RK, 1};
    if (!make_map(&tm.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  }
  return true;
}

}  // namespace

extern "C" size_t octo_decode_attn_workspace(const octo_layout* L, int B, int Hq, int Hkv, int Lq, int64_t kv_len) {
  if (check_layout(L) != OCTO_OK) return 0;
  if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || Lq < 1 || kv_len < 0) return 0;
  const int Gq = (Hq / Hkv) * Lq;
  if (Gq > 8) return 0;
  const int G = octo::rows_template(Gq);
  const octo::SplitPlan sp = octo::plan_splits(static_cast<int64_t>(B) * Hkv, std::max<int64_t>(kv_len, 1),
                                               octo::sm_count(), octo::unit_bytes(L));
  return ws_layout(static_cast<int64_t>(B) * Hkv, sp.n, G, L->d, L->qjl != 0).total;
}

int octo::decode_validate(const octo_layout* L, const octo_tables* tab, const void* q, int q_dtype, int B, int Hq,
                          int Hkv, int Lq, int64_t kv_len, int64_t cache_cap, const uint32_t* packed,
                          const float* gamma, const uint32_t* qjl_bits, const float* qjl_norm, const void* V,
                          float scale, const float* out, const float* logits, size_t* ws_need) {
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
  if (L->qjl && (misaligned(qjl_bits) || misaligned(qjl_norm) || misaligned(tab->qjl_S))) return OCTO_EINVAL;
  if (!(scale == scale)) return OCTO_EINVAL;
  if ((Hq / Hkv) * Lq > 8) return OCTO_EUNSUPPORTED;
  if (static_cast<int64_t>(B) * Hkv > 65535) return OCTO_EUNSUPPORTED;  // grid.y limit
  if (kv_len > INT_MAX) return OCTO_EUNSUPPORTED;                         // 32-bit token coordinates
  if (ws_need) *ws_need = octo_decode_attn_workspace(L, B, Hq, Hkv, Lq, kv_len);
  return OCTO_OK;
}

extern "C" int octo_decode_attn(const octo_layout* L, const octo_tables* tab, const void* q, int q_dtype, int B,
                                int Hq, int Hkv, int Lq, int64_t kv_len, int64_t cache_cap,
                                const uint32_t* packed, const float* gamma, const uint32_t* qjl_bits,
                                const float* qjl_norm, const void* V, float scale, float* out, float* logits,
                                void* workspace, size_t ws_bytes, octo_stream_t stream) {
  size_t need = 0;
  const int vc = octo::decode_validate(L, tab, q, q_dtype, B, Hq, Hkv, Lq, kv_len, cache_cap, packed, gamma,
                                       qjl_bits, qjl_norm, V, scale, out, logits, &need);
  if (vc != OCTO_OK) return vc;
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return OCTO_EINVAL;
  const int g = Hq / Hkv, Gq = g * Lq;
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

  const octo::SplitPlan sp = octo::plan_splits(heads, kv_len, octo::sm_count(), octo::unit_bytes(L));
  a.n_splits = sp.n;
  a.keys_per_split = sp.per;
  a.heads_lo = sp.heads_lo;
  a.n_splits_lo = sp.n_lo;
  a.keys_per_split_lo = sp.per_lo;
  const WsLayout w = ws_layout(heads, a.n_splits, G, D, L->qjl != 0);
  if (ws_bytes < w.total) return OCTO_EWORKSPACE;
  char* base = static_cast<char*>(workspace);
  a.status = reinterpret_cast<int*>(base + w.status);
  a.counters = reinterpret_cast<int*>(base + w.counters);
  a.part_m = reinterpret_cast<float*>(base + w.m);
  a.part_l = reinterpret_cast<float*>(base + w.l);
  a.part_o = reinterpret_cast<float*>(base + w.o);
  a.prep = reinterpret_cast<float*>(base + w.prep);
  a.prep_stride = prep_floats(L->qjl != 0, G, D);
  const dim3 grid(static_cast<unsigned>(a.n_splits), static_cast<unsigned>(heads));
  // tensor maps for the tensor-core kernel (d <= 128)
  octo::TmaDesc tm;
  std::memset(&tm, 0, sizeof(tm));
  if (D <= 128 &&
      !build_maps(tm, L, heads, kv_len, cache_cap, packed, gamma, qjl_bits, qjl_norm, V))
    return OCTO_ECUDA;
  cudaError_t e;
  switch (D) {
    case 64: e = octo::launch_decode_d64(a, tm, L->b, G, L->qjl != 0, grid, st); break;
    case 128: e = octo::launch_decode_d128(a, tm, L->b, G, L->qjl != 0, grid, st); break;
    default: e = octo::launch_decode_d256(a, tm, L->b, G, L->qjl != 0, grid, st); break;
  }
  return e == cudaSuccess ? OCTO_OK : OCTO_ECUDA;
}
