// OCTOPUS key reconstruction for sm_100a: k_hat = gamma * R^T u_hat.
//
// The explainer's "triplet decomposition" read backwards (the codec used to
// compress and reconstruct a cache rather than to attend over it): unpack the
// T triplet codes of a key, decode each to rho_hat * n_hat (inverse
// octahedral map of the two direction levels, section "octahedral folding",
// scaled by the norm level), concatenate into the rotated direction u_hat
// (padding dropped), and undo the rotation R = (1/sqrt(d)) H diag(s). H is
// symmetric, so R^T u = (1/sqrt(d)) s * (H u): the encoder's warp-shuffle
// Walsh-Hadamard butterflies followed by a per-coordinate scale
// gamma * s_j / sqrt(d). The QJL sketch plays no part: it estimates inner
// products, it does not correct the key.
//
// Kernel structure: a persistent grid walks tiles of KT consecutive tokens
// of one head. Phase 1 stages the tile's code words ([W][KT], token-
// contiguous in the cache, so each word plane is one coalesced row) and
// gammas in shared memory; it is issued one tile ahead, into registers, so
// the loads overlap the previous tile's work. Phase 2 runs one thread per (key, triplet) over
// the tile and writes the decoded triplet into the key's shared-memory row;
// decoded triplets of the positive-level quadrant come from a replicated
// table and the code's two direction signs flip x and y. Phase 3 runs one
// warp per key: d/32 coordinates per lane, butterflies, scale, one vector
// store per lane (fp32 or bf16 rows). The output bytes dominate the
// traffic (4d or 2d bytes per key against 4W + 4 read).

#include <cuda_runtime.h>

#include <algorithm>

#include "octo_common.cuh"

namespace octo {

struct DequantArgs {
  const uint32_t* packed;
  const float* gamma;
  const float* dir_c;
  const float* rho_c;
  const float* signs;
  void* out;
  int out_bf16;
  int64_t n_heads, n_tokens, cache_cap, token_offset, table_heads;
  int64_t tiles_per_head, n_tiles;
};

template <int D, int B>
struct DqCfg {
  static constexpr int T = (D + 2) / 3;
  static constexpr int BD = B + 1, BR = B - 1;
  static constexpr int C = 2 * BD + BR;
  static constexpr int W = (T * C + 31) / 32;
  static constexpr int NDIR = 1 << BD, NRHO = 1 << BR;
  static constexpr int NE = 1 << (3 * B - 1);  // positive quadrant: (m_xi, m_eta, i_rho)
  static constexpr int REP = NE <= 256 ? 8 : 2;  // replicas: lanes of a quarter-warp in distinct bank groups
  static constexpr int E = D / 32;               // coordinates per lane in phase 3
  static constexpr int KT = 64;                  // keys per tile
  static constexpr int US = (3 * T + 3) / 4 * 4;  // row stride of the decoded directions (floats, 16-byte rows)
  static constexpr int THREADS = 256;
  static constexpr int NWARP = THREADS / 32;
  static constexpr size_t TABLE = sizeof(float4) * NE * REP;
  static constexpr size_t UROWS = sizeof(float) * KT * US;
  // word planes [W + 1][CS] (+ a zero plane, see phase 2); the odd stride puts
  // the planes of one key in distinct banks
  static constexpr int CS = KT + 1;
  static constexpr size_t CODES = (sizeof(uint32_t) * (W + 1) * CS + 15) / 16 * 16;
  static constexpr size_t SMEM = TABLE + UROWS + CODES + sizeof(float) * KT;
  static_assert(TABLE % 16 == 0 && UROWS % 16 == 0 && CODES % 16 == 0, "16-byte aligned parts");
};

template <int D, int B>
__global__ void __launch_bounds__(256) dequant_kernel(DequantArgs a) {
  using Cfg = DqCfg<D, B>;
  constexpr int T = Cfg::T, C = Cfg::C, W = Cfg::W, E = Cfg::E, KT = Cfg::KT, US = Cfg::US, CS = Cfg::CS;
  constexpr int NE = Cfg::NE, REP = Cfg::REP, NWARP = Cfg::NWARP, THREADS = Cfg::THREADS;
  constexpr uint32_t HALF = 1u << B;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  float4* table = reinterpret_cast<float4*>(smem_raw);                                  // [NE][REP]
  float* U = reinterpret_cast<float*>(smem_raw + Cfg::TABLE);                           // [KT][US]
  uint32_t* cw = reinterpret_cast<uint32_t*>(smem_raw + Cfg::TABLE + Cfg::UROWS);       // [W + 1][CS]
  float* gs = reinterpret_cast<float*>(smem_raw + Cfg::TABLE + Cfg::UROWS + Cfg::CODES);  // [KT]
  __shared__ float s_dir_c[32], s_rho_c[8];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < Cfg::NDIR) s_dir_c[tid] = a.dir_c[tid];
  if (tid < Cfg::NRHO) s_rho_c[tid] = a.rho_c[tid];
  __syncthreads();
  // rho_hat * n_hat for the cells (HALF + m_xi, HALF + m_eta) and norm level i_rho
  for (int e = tid; e < NE; e += THREADS) {
    const float3 n = oct_inverse(s_dir_c[HALF + (e & (HALF - 1))], s_dir_c[HALF + ((e >> B) & (HALF - 1))]);
    const float r = s_rho_c[e >> (2 * B)];
    const float4 v = make_float4(n.x * r, n.y * r, n.z * r, 0.0f);
#pragma unroll
    for (int k = 0; k < REP; ++k) table[e * REP + k] = v;
  }
  // a zero word plane after the last: the code that ends in word W - 1 reads it as its "next" word
  for (int k = tid; k < KT; k += THREADS) cw[W * CS + k] = 0u;
  const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
  const int rep_off = lane & (REP - 1);
  __syncthreads();

  // Phase 1 for tile tl: this thread's share of the code words (PW of them,
  // coalesced along the tokens) and one gamma, into registers; stored to
  // shared memory once the previous tile no longer needs the buffers, so the
  // loads overlap the previous tile's phases 2 and 3.
  constexpr int PW = (W * KT + THREADS - 1) / THREADS;
  uint32_t nw[PW];
  float ng = 0.0f;
  auto fetch = [&](int64_t tl) {
    const int64_t fh = tl / a.tiles_per_head;
    const int64_t ft0 = (tl - fh * a.tiles_per_head) * KT;
    const int fnk = static_cast<int>(min(static_cast<int64_t>(KT), a.n_tokens - ft0));
    const uint32_t* ph = a.packed + fh * W * a.cache_cap + a.token_offset + ft0;
#pragma unroll
    for (int j = 0; j < PW; ++j) {
      const int i = tid + j * THREADS, w = i / KT, k = i - w * KT;
      nw[j] = (i < W * KT && k < fnk) ? __ldg(ph + static_cast<int64_t>(w) * a.cache_cap + k) : 0u;
    }
    ng = tid < fnk ? __ldg(a.gamma + fh * a.cache_cap + a.token_offset + ft0 + tid) : 0.0f;
  };
  auto stash_words = [&]() {
#pragma unroll
    for (int j = 0; j < PW; ++j) {
      const int i = tid + j * THREADS;
      if (i < W * KT) cw[(i / KT) * CS + (i % KT)] = nw[j];
    }
  };
  static_assert(KT <= THREADS, "one gamma per thread");
  if (static_cast<int64_t>(blockIdx.x) < a.n_tiles) {
    fetch(blockIdx.x);
    stash_words();
    if (tid < KT) gs[tid] = ng;
  }
  __syncthreads();

  for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x) {
    const int64_t h = tile / a.tiles_per_head;
    const int64_t t0 = (tile - h * a.tiles_per_head) * KT;  // first token of the tile, from token_offset
    const int nk = static_cast<int>(min(static_cast<int64_t>(KT), a.n_tokens - t0));
    const int64_t next = tile + gridDim.x;
    if (next < a.n_tiles) fetch(next);

    // phase 2: one thread per (key, triplet); code i of a key sits at stream bit i*C
    for (int i = tid; i < nk * T; i += THREADS) {
      const int k = i / T, t = i - k * T;
      const int bit = t * C, w0 = bit >> 5, sh = bit & 31;
      const uint32_t code = __funnelshift_r(cw[w0 * CS + k], cw[(w0 + 1) * CS + k], sh) & ((1u << C) - 1u);
      const uint32_t q = (code & ((1u << (2 * B)) - 1u)) | ((code >> (2 * B + 2)) << (2 * B));
      float4 v = table[q * REP + rep_off];
      // the codebook is odd-symmetric and the inverse map odd in x and in y
      v.x = __uint_as_float(__float_as_uint(v.x) ^ (((code >> (2 * B)) & 1u) << 31));
      v.y = __uint_as_float(__float_as_uint(v.y) ^ (((code >> (2 * B + 1)) & 1u) << 31));
      float* u = U + k * US + 3 * t;
      u[0] = v.x;
      u[1] = v.y;
      u[2] = v.z;
    }
    __syncthreads();
    if (next < a.n_tiles) stash_words();  // phase 3 does not read the words

    // phase 3: one warp per key: H u_hat, then gamma * s_j / sqrt(d)
    float sg[E];
    const float* srow = a.signs + (h % a.table_heads) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) sg[e] = __ldg(srow + e) * inv_sqrt_d;
    auto load_row = [&](int k, float (&v)[E]) {
      const float* u = U + k * US + lane * E;
      if constexpr (E == 2) {
        const float2 x = *reinterpret_cast<const float2*>(u);
        v[0] = x.x; v[1] = x.y;
      } else {
#pragma unroll
        for (int e = 0; e < E; e += 4) {
          const float4 x = *reinterpret_cast<const float4*>(u + e);
          v[e] = x.x; v[e + 1] = x.y; v[e + 2] = x.z; v[e + 3] = x.w;
        }
      }
    };
    auto store_row = [&](int k, float (&v)[E]) {
      const float g = gs[k];
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] *= g * sg[e];
      const int64_t off = ((h * a.n_tokens + t0 + k) * D) + lane * E;
      if (a.out_bf16) {
        uint32_t p[E / 2];
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[e], v[e + 1]);
          p[e / 2] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.out) + off;
        if constexpr (E == 2) {
          *reinterpret_cast<uint32_t*>(o) = p[0];
        } else if constexpr (E == 4) {
          *reinterpret_cast<uint2*>(o) = make_uint2(p[0], p[1]);
        } else {
#pragma unroll
          for (int e = 0; e < E / 2; e += 4)
            *reinterpret_cast<uint4*>(o + 2 * e) = make_uint4(p[e], p[e + 1], p[e + 2], p[e + 3]);
        }
      } else {
        float* o = static_cast<float*>(a.out) + off;
        if constexpr (E == 2) {
          *reinterpret_cast<float2*>(o) = make_float2(v[0], v[1]);
        } else {
#pragma unroll
          for (int e = 0; e < E; e += 4)
            *reinterpret_cast<float4*>(o + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
    };
    for (int k = warp; k < nk; k += NWARP) {
      float v[E];
      load_row(k, v);
      fwht_warp<E>(v, lane);
      store_row(k, v);
    }
    __syncthreads();  // the rows and gammas are reused by the next tile
    if (next < a.n_tiles && tid < KT) gs[tid] = ng;
  }
}

template <int D, int B>
static cudaError_t launch_dequant(const DequantArgs& a0, cudaStream_t st) {
  using Cfg = DqCfg<D, B>;
  DequantArgs a = a0;
  a.tiles_per_head = (a.n_tokens + Cfg::KT - 1) / Cfg::KT;
  a.n_tiles = a.tiles_per_head * a.n_heads;
  auto kern = dequant_kernel<D, B>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(Cfg::SMEM));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cfg::THREADS, Cfg::SMEM);
  if (per_sm < 1) per_sm = 1;
  const int64_t grid = std::min<int64_t>(a.n_tiles, static_cast<int64_t>(sms) * per_sm);
  kern<<<static_cast<unsigned>(grid), Cfg::THREADS, Cfg::SMEM, st>>>(a);
  return cudaGetLastError();
}

template <int D>
static cudaError_t dequant_dispatch_b(const DequantArgs& a, int b, cudaStream_t st) {
  switch (b) {
    case 2: return launch_dequant<D, 2>(a, st);
    case 3: return launch_dequant<D, 3>(a, st);
    default: return launch_dequant<D, 4>(a, st);
  }
}

}  // namespace octo

extern "C" int octo_dequant(const octo_layout* L, const octo_tables* tab, int64_t n_heads, int64_t n_tokens,
                            int64_t cache_cap, int64_t token_offset, const uint32_t* packed, const float* gamma,
                            void* out, int out_dtype, octo_stream_t stream) {
  using namespace octo;
  if (!L || !tab) return OCTO_EINVAL;
  if (L->d != 64 && L->d != 128 && L->d != 256) return OCTO_EUNSUPPORTED;
  if (L->b < 2 || L->b > 4) return OCTO_EUNSUPPORTED;
  octo_layout chk;
  if (octo_layout_init(&chk, L->d, L->b, L->qjl, L->rounding) != OCTO_OK) return OCTO_EINVAL;
  if (chk.words != L->words || chk.T != L->T || chk.code_bits != L->code_bits) return OCTO_EINVAL;
  if (out_dtype != OCTO_F32 && out_dtype != OCTO_BF16) return OCTO_EINVAL;
  if (n_heads < 0 || n_tokens < 0 || token_offset < 0 || cache_cap < 0) return OCTO_EINVAL;
  if (token_offset + n_tokens > cache_cap) return OCTO_EINVAL;
  if (n_heads == 0 || n_tokens == 0) return OCTO_OK;
  if (!packed || !gamma || !out || !tab->dir_c || !tab->rho_c || !tab->signs || tab->n_heads < 1)
    return OCTO_EINVAL;
  if (reinterpret_cast<uintptr_t>(out) % 16 != 0) return OCTO_EINVAL;
  DequantArgs a{};
  a.packed = packed;
  a.gamma = gamma;
  a.dir_c = tab->dir_c;
  a.rho_c = tab->rho_c;
  a.signs = tab->signs;
  a.out = out;
  a.out_bf16 = out_dtype == OCTO_BF16;
  a.n_heads = n_heads;
  a.n_tokens = n_tokens;
  a.cache_cap = cache_cap;
  a.token_offset = token_offset;
  a.table_heads = tab->n_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (L->d) {
    case 64: e = dequant_dispatch_b<64>(a, L->b, st); break;
    case 128: e = dequant_dispatch_b<128>(a, L->b, st); break;
    default: e = dequant_dispatch_b<256>(a, L->b, st); break;
  }
  return e == cudaSuccess ? OCTO_OK : OCTO_ECUDA;
}
