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
// Kernel structure: each block walks a contiguous range of tiles of KT
// consecutive tokens of one head. A tile's code words ([W][KT], token-
// contiguous in the cache, so each word plane is one coalesced row) and
// gammas are staged in shared memory by asynchronous copies, one tile ahead
// (two buffers). A key is handled by d/32 lanes, each owning 32 consecutive
// coordinates: the lane decodes the 12 triplets that cover them straight
// into registers (codes from a window of the key's words; decoded triplets
// of the positive-level quadrant from a replicated table, the code's two
// direction signs flipping x and y), runs 5 butterfly stages in registers
// and the remaining log2(d/32) across its lanes, scales and stores its 32
// outputs (fp32 or bf16). The output bytes dominate the traffic (4d or 2d
// bytes per key against 4W + 4 read).

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
  int out_v8;  // out is 32-byte aligned: 32-byte stores (whole sectors per lane)
  int in_v4;   // token offset, capacity and cache pointers allow 16-byte staging copies
  int64_t n_heads, n_tokens, cache_cap, token_offset, table_heads;
  int64_t tiles_per_head, n_tiles;
};

// BD_ bits for each of xi and eta, BR_ for rho (the OCTOPUS allocation is
// (b + 1, b - 1); other splits serve the bit-allocation sweep).
template <int D, int BD_, int BR_>
struct DqCfg {
  static constexpr int T = (D + 2) / 3;
  static constexpr int BD = BD_, BR = BR_;
  static constexpr int B = BD - 1;  // magnitude bits of a direction cell
  static constexpr int C = 2 * BD + BR;
  static constexpr int W = (T * C + 31) / 32;
  static constexpr int NDIR = 1 << BD, NRHO = 1 << BR;
  static constexpr int NE = 1 << (2 * B + BR);     // positive quadrant: (m_xi, m_eta, i_rho)
  static constexpr int REP = NE <= 256 ? 8 : 2;    // replicas: lanes of a quarter-warp in distinct bank groups
  static constexpr int LK = D / 32;                // lanes per key, 32 coordinates each
  static constexpr int LKB = LK == 2 ? 1 : (LK == 4 ? 2 : 3);
  static constexpr int KW = 32 / LK;               // keys per warp and pass
  static constexpr int THREADS = 256, NWARP = THREADS / 32;
  static constexpr int KT = 128;                   // keys per tile
  static constexpr int PASSES = KT / (NWARP * KW);
  // A lane decodes the NT triplets from floor(32 j / 3) on: 36 coordinates,
  // which hold its 32 at any offset 0..2. Their codes lie in a window of NWL
  // words (one more than the last code's first word, for its upper bits).
  static constexpr int NT = 12;
  static constexpr int NWL = ((NT - 1) * C) / 32 + 3;
  static constexpr int WMAX = ((32 * (LK - 1) / 3) * C) / 32 + NWL;  // end of the last lane's window
  static constexpr int WP = WMAX > W ? WMAX : W;   // word planes held; planes >= W stay zero
  // plane stride: 16-byte rows for the 16-byte staging copies; 4 mod 32
  // words, so the lanes of a key (different planes, same column) mostly
  // fall in different banks
  static constexpr int CS = KT + 4;
  static constexpr size_t TABLE = sizeof(float4) * NE * REP;
  static constexpr size_t CBUF = (sizeof(uint32_t) * WP * CS + 15) / 16 * 16;
  static constexpr size_t SMEM = TABLE + 2 * CBUF + 2 * sizeof(float) * KT;  // two tile buffers
  static_assert(PASSES * NWARP * KW == KT && NT * 3 >= 32 + 2, "tile and lane coverage");
  static_assert(TABLE % 16 == 0, "16-byte aligned parts");
};

// 4-byte asynchronous global -> shared copy; bytes = 0 writes a zero.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(bytes)
               : "memory");
}
// 16-byte asynchronous global -> shared copy (both addresses 16-byte
// aligned); only the first `bytes` come from global memory, the rest are zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(bytes)
               : "memory");
}
// 32-byte global store (sm_100): eight 32-bit words, 32-byte aligned address.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

template <int D, int BD_, int BR_>
__global__ void __launch_bounds__(256, 3) dequant_kernel(DequantArgs a) {
  using Cfg = DqCfg<D, BD_, BR_>;
  constexpr int B = Cfg::B;
  constexpr int C = Cfg::C, W = Cfg::W, KT = Cfg::KT, CS = Cfg::CS, LK = Cfg::LK, LKB = Cfg::LKB, KW = Cfg::KW;
  constexpr int NE = Cfg::NE, REP = Cfg::REP, NWARP = Cfg::NWARP, THREADS = Cfg::THREADS, NT = Cfg::NT;
  constexpr int NWL = Cfg::NWL, WP = Cfg::WP;
  constexpr uint32_t HALF = 1u << B, CM = (1u << C) - 1u;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  float4* table = reinterpret_cast<float4*>(smem_raw);  // [NE][REP]
  uint32_t* cwb = reinterpret_cast<uint32_t*>(smem_raw + Cfg::TABLE);  // [2][WP][CS]
  float* gsb = reinterpret_cast<float*>(smem_raw + Cfg::TABLE + 2 * Cfg::CBUF);  // [2][KT]
  __shared__ float s_dir_c[32], s_rho_c[32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = lane & (LK - 1);  // this lane's coordinates: [32 j, 32 j + 32) of its key
  const int t0 = (32 * j) / 3, roff = 32 * j - 3 * t0;  // first triplet; its offset before 32 j (0..2)
  const int wa = (t0 * C) >> 5, boff = (t0 * C) & 31;  // code window: first word, bit offset in it

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
  // word planes past the key's last word read as zeros (both buffers)
  if constexpr (WP > W) {
    for (int i = tid; i < 2 * (WP - W) * CS; i += THREADS) {
      const int bb = i / ((WP - W) * CS), r = i - bb * (WP - W) * CS;
      cwb[bb * (Cfg::CBUF / 4) + W * CS + r] = 0u;
    }
  }
  const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
  const int rep_off = lane & (REP - 1);

  // this block's contiguous range of tiles (a head changes rarely along it)
  const int64_t per = (a.n_tiles + gridDim.x - 1) / gridDim.x;
  const int64_t tbeg = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t tend = min(a.n_tiles, tbeg + per);

  // tile tl's code words and gammas into buffer bb (cp.async, zero past the end)
  auto stage = [&](int64_t tl, int bb) {
    const int64_t h = tl / a.tiles_per_head;
    const int64_t ft0 = (tl - h * a.tiles_per_head) * KT;
    const int fnk = static_cast<int>(min(static_cast<int64_t>(KT), a.n_tokens - ft0));
    const int64_t tok0 = a.token_offset + ft0;
    const uint32_t* ph = a.packed + h * W * a.cache_cap + tok0;
    uint32_t* cw = cwb + bb * (Cfg::CBUF / 4);
    if (a.in_v4) {
      // four tokens a copy; past the last token the copies read less (zeros)
      constexpr int K4 = KT / 4;
      for (int i = tid; i < W * K4; i += THREADS) {
        const int w = i / K4, k = 4 * (i - w * K4);
        const int n = max(0, min(4, fnk - k));
        cp_async16(cw + w * CS + k, ph + static_cast<int64_t>(w) * a.cache_cap + (n > 0 ? k : 0), 4u * n);
      }
      if (tid < K4) {
        const int k = 4 * tid, n = max(0, min(4, fnk - k));
        cp_async16(gsb + bb * KT + k, a.gamma + h * a.cache_cap + tok0 + (n > 0 ? k : 0), 4u * n);
      }
    } else {
      for (int i = tid; i < W * KT; i += THREADS) {
        const int w = i / KT, k = i - w * KT;
        cp_async4(cw + w * CS + k, ph + static_cast<int64_t>(w) * a.cache_cap + min(k, fnk - 1), k < fnk ? 4u : 0u);
      }
      if (tid < KT)
        cp_async4(gsb + bb * KT + tid, a.gamma + h * a.cache_cap + tok0 + min(tid, fnk - 1), tid < fnk ? 4u : 0u);
    }
  };

  uint32_t smask = 0;  // bit p: s_j < 0 for this lane's coordinate 32 j + p, for head sg_head
  int64_t sg_head = -1;
  if (tbeg < tend) stage(tbeg, 0);
  cp_async_commit_wait();
  __syncthreads();

  int bb = 0;
  for (int64_t tile = tbeg; tile < tend; ++tile, bb ^= 1) {
    const int64_t h = tile / a.tiles_per_head;
    const int64_t t0tok = (tile - h * a.tiles_per_head) * KT;
    const int nk = static_cast<int>(min(static_cast<int64_t>(KT), a.n_tokens - t0tok));
    if (tile + 1 < tend) stage(tile + 1, bb ^ 1);  // overlaps this tile's work
    if (h != sg_head) {
      const float* srow = a.signs + (h % a.table_heads) * D + 32 * j;
      smask = 0;
#pragma unroll
      for (int p = 0; p < 32; ++p) smask |= (__ldg(srow + p) < 0.0f ? 1u : 0u) << p;
      sg_head = h;
    }
    const uint32_t* cw = cwb + bb * (Cfg::CBUF / 4);
    const float* gs = gsb + bb * KT;
#pragma unroll 1
    for (int pass = 0; pass < Cfg::PASSES; ++pass) {
      const int kk = (pass * NWARP + warp) * KW + (lane >> LKB);  // key of this lane's group in the tile
      // this lane's code window
      uint32_t wr[NWL];
#pragma unroll
      for (int m = 0; m < NWL; ++m) wr[m] = cw[(wa + m) * CS + kk];
      // decode triplets t0 .. t0 + NT - 1 into v[3 i + c] (coordinate 32 j - roff + 3 i + c)
      float v[3 * NT];
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        const int qi = (i * C) >> 5;                     // word of the code's first bit, without boff
        const int o = boff + ((i * C) & 31);             // its bit in word qi (may carry into qi + 1)
        const bool carry = o >= 32;
        const uint32_t lo = carry ? wr[qi + 1] : wr[qi];
        const uint32_t hi = carry ? wr[qi + 2] : wr[qi + 1];
        const uint32_t code = __funnelshift_r(lo, hi, o & 31) & CM;
        const uint32_t q = (code & ((1u << (2 * B)) - 1u)) | ((code >> (2 * B + 2)) << (2 * B));
        const float4 e = table[q * REP + rep_off];
        // the codebook is odd-symmetric and the inverse map odd in x and in y
        v[3 * i] = __uint_as_float(__float_as_uint(e.x) ^ ((code << (31 - 2 * B)) & 0x80000000u));
        v[3 * i + 1] = __uint_as_float(__float_as_uint(e.y) ^ ((code << (30 - 2 * B)) & 0x80000000u));
        v[3 * i + 2] = e.z;
      }
      // shift by roff: x[p] = v[p + roff]
#pragma unroll
      for (int p = 0; p < 32; ++p) v[p] = roff == 0 ? v[p] : (roff == 1 ? v[p + 1] : v[p + 2]);
      // H over the 32 register coordinates, then across the LK lanes of the key
#pragma unroll
      for (int hh = 1; hh < 32; hh <<= 1) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          if ((e & hh) == 0) {
            const float x = v[e], y = v[e + hh];
            v[e] = x + y;
            v[e + hh] = x - y;
          }
        }
      }
#pragma unroll
      for (int m = 1; m < LK; m <<= 1) {
        const float sgn = (lane & m) != 0 ? -1.0f : 1.0f;
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = fmaf(sgn, v[e], __shfl_xor_sync(0xffffffffu, v[e], m));
      }
      if (kk < nk) {
        const float g = gs[kk] * inv_sqrt_d;
        // k_hat_j = gamma s_j (H u_hat)_j / sqrt(d): scale, then the sign bit of s_j
        auto outv = [&](int p) {
          return __uint_as_float(__float_as_uint(v[p] * g) ^ ((smask << (31 - p)) & 0x80000000u));
        };
        const int64_t off = (h * a.n_tokens + t0tok + kk) * D + 32 * j;
        uint32_t w[32];  // the 32 outputs as fp32 bits, or packed bf16 pairs in w[0..15]
        if (a.out_bf16) {
#pragma unroll
          for (int p = 0; p < 32; p += 2) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(outv(p), outv(p + 1));
            w[p / 2] = *reinterpret_cast<const uint32_t*>(&b2);
          }
        } else {
#pragma unroll
          for (int p = 0; p < 32; ++p) w[p] = __float_as_uint(outv(p));
        }
        unsigned char* o = static_cast<unsigned char*>(a.out) + off * (a.out_bf16 ? 2 : 4);
        const int nw = a.out_bf16 ? 16 : 32;
        if (a.out_v8) {
#pragma unroll
          for (int q = 0; q < 32; q += 8) {
            if (q < nw) {
              const uint32_t w8[8] = {w[q], w[q + 1], w[q + 2], w[q + 3], w[q + 4], w[q + 5], w[q + 6], w[q + 7]};
              st_global_v8(o + 4 * q, w8);
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; q += 4)
            if (q < nw) *reinterpret_cast<uint4*>(o + 4 * q) = make_uint4(w[q], w[q + 1], w[q + 2], w[q + 3]);
        }
      }
    }
    cp_async_commit_wait();  // the next tile's words are in
    __syncthreads();         // and every warp is done with this tile's buffer
  }
}

template <int D, int BD, int BR>
static cudaError_t launch_dequant(const DequantArgs& a0, cudaStream_t st) {
  using Cfg = DqCfg<D, BD, BR>;
  DequantArgs a = a0;
  a.tiles_per_head = (a.n_tokens + Cfg::KT - 1) / Cfg::KT;
  a.n_tiles = a.tiles_per_head * a.n_heads;
  auto kern = dequant_kernel<D, BD, BR>;
  static LaunchCache cache;
  int resident = 0;
  const cudaError_t e = launch_setup(kern, cache, Cfg::THREADS, Cfg::SMEM, resident);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(a.n_tiles, resident);
  kern<<<static_cast<unsigned>(grid), Cfg::THREADS, Cfg::SMEM, st>>>(a);
  return cudaGetLastError();
}

// The OCTOPUS split for every d; at d = 128 also the bit-allocation sweep's
// other splits (the encoder's set).
template <int D>
static cudaError_t dequant_dispatch_split(const DequantArgs& a, int b_dir, int b_rho, cudaStream_t st) {
  if (b_dir == 3 && b_rho == 1) return launch_dequant<D, 3, 1>(a, st);
  if (b_dir == 4 && b_rho == 2) return launch_dequant<D, 4, 2>(a, st);
  if (b_dir == 5 && b_rho == 3) return launch_dequant<D, 5, 3>(a, st);
  if constexpr (D == 128) {
    if (b_dir == 2 && b_rho == 4) return launch_dequant<D, 2, 4>(a, st);
    if (b_dir == 3 && b_rho == 3) return launch_dequant<D, 3, 3>(a, st);
    if (b_dir == 5 && b_rho == 1) return launch_dequant<D, 5, 1>(a, st);
    if (b_dir == 3 && b_rho == 5) return launch_dequant<D, 3, 5>(a, st);
    if (b_dir == 4 && b_rho == 4) return launch_dequant<D, 4, 4>(a, st);
  }
  return cudaErrorNotSupported;
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
  const int lc = octo_layout_init_delta(&chk, L->d, L->b, L->b_dir - L->b, L->qjl, L->rounding);
  if (lc != OCTO_OK) return lc;
  // the OCTOPUS split for every d; the bit-allocation sweep's splits at d = 128 without the sketch
  const bool octopus_split = L->b_dir == L->b + 1;
  if (!octopus_split && (L->d != 128 || L->qjl)) return OCTO_EUNSUPPORTED;
  if (chk.words != L->words || chk.T != L->T || chk.code_bits != L->code_bits || chk.b_rho != L->b_rho)
    return OCTO_EINVAL;
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
  a.out_v8 = reinterpret_cast<uintptr_t>(out) % 32 == 0;
  a.in_v4 = token_offset % 4 == 0 && cache_cap % 4 == 0 && reinterpret_cast<uintptr_t>(packed) % 16 == 0 &&
            reinterpret_cast<uintptr_t>(gamma) % 16 == 0;
  a.n_heads = n_heads;
  a.n_tokens = n_tokens;
  a.cache_cap = cache_cap;
  a.token_offset = token_offset;
  a.table_heads = tab->n_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (L->d) {
    case 64: e = dequant_dispatch_split<64>(a, L->b_dir, L->b_rho, st); break;
    case 128: e = dequant_dispatch_split<128>(a, L->b_dir, L->b_rho, st); break;
    default: e = dequant_dispatch_split<256>(a, L->b_dir, L->b_rho, st); break;
  }
  if (e == cudaErrorNotSupported) return OCTO_EUNSUPPORTED;  // a split without a built kernel (nothing launched)
  return e == cudaSuccess ? OCTO_OK : OCTO_ECUDA;
}
