// OCTOPUS key encoder for sm_100a.
//
// Per key (explainer, "triplet decomposition"): gamma = ||k|| (fp32),
// u = k / gamma; rotate u by the sign-flipped Walsh-Hadamard transform
// (section "rotation"); cut the rotated direction into triplets, zero-padded
// at the end; per triplet take rho = ||t|| and the octahedral coordinates
// (xi, eta) of its direction (section "octahedral folding"); index xi and eta
// with the (b+1)-bit codebook and rho with the (b-1)-bit codebook, then (by
// default) refine by the 3x3 joint search of section "joint rounding"; pack
// the (3b+1)-bit codes into the key's bit stream. With OCTOPUS-QJL (section
// "optional residual correction") also store sign(S e) and ||e|| for the
// rotated residual e = u_rot - u_rot_hat.
//
// Kernel structure: each block walks a contiguous range of tiles of KT
// consecutive tokens of one head (KT as large as leaves room for three
// blocks per SM). Phase 1: d/32 lanes per key, 32 coordinates per lane -
// vector loads, the norm by a short shuffle reduction, sign flips from a lane
// bit mask, 5 butterfly stages in registers and the rest across the key's
// lanes; the rotated direction goes to shared memory. Phase 2: one thread
// per triplet over the whole tile (balanced whatever T is) - octahedral map,
// indexing, and the joint search as the largest s = n_hat . t over a
// bordered shared-memory table of decoded unit directions. Phase 3: one
// thread per (key, word) assembles the packed words and stores them
// token-contiguously (coalesced). Phase 4 (QJL): the projection S e
// register-blocked - each warp d/8 rows of S, each lane a few keys - and the
// sign bits gathered per key in shared memory.

#include <cuda_runtime.h>

#include <algorithm>

#include "octo_common.cuh"

namespace octo {

struct EncodeArgs {
  const void* keys;
  int key_bf16;
  int64_t n_heads, n_tokens, head_stride, token_stride, cache_cap, token_offset;
  uint32_t* packed;
  float* gamma;
  uint32_t* qjl_bits;
  float* qjl_norm;
  const float* dir_c;
  const float* dir_t;
  const float* rho_c;
  const float* rho_t;
  const float* signs;
  const float* qjl_S;
  int64_t table_heads;
  int joint;
  int64_t n_tiles, tiles_per_head;
};

// BD_ bits for each of xi and eta, BR_ for rho (the OCTOPUS allocation is
// (b + 1, b - 1); other splits serve the bit-allocation sweep).
template <int D, int BD_, int BR_>
struct EncCfg {
  static constexpr int T = (D + 2) / 3;
  static constexpr int BD = BD_, BR = BR_;
  static constexpr int MB = BD - 1;  // magnitude bits of a direction cell
  static constexpr int C = 2 * BD + BR;
  static constexpr int W = (T * C + 31) / 32;
  static constexpr int NDIR = 1 << BD, NRHO = 1 << BR;
  // row stride of the rotated directions (floats), at least 3T. From d = 128
  // on it is 4 mod 32, so that 8 rows x 4 consecutive columns (an MMA B
  // fragment of the sketch projection) hit 32 banks; at d = 64 it is odd, so
  // that one row per lane (the FMA projection) does.
  static constexpr int US = D >= 128 ? 3 * T + ((4 - 3 * T) % 32 + 32) % 32
                                     : ((3 * T) % 2 == 0 ? 3 * T + 1 : 3 * T);
  static constexpr int THREADS = 256;
  // the n_hat table has a border of one cell on every side (NaN vectors), so
  // that the 3x3 neighbourhood of any cell is inside it
  static constexpr int NB = NDIR + 2;
  // n_hat replicas: 8 put the lanes of a quarter-warp in distinct bank
  // groups; the 34 x 34 table of b = 4 keeps 4
  static constexpr int REP = NB * NB * 8 * 16 <= 48 * 1024 ? 8 : 4;
  static constexpr size_t TABLE = sizeof(float4) * NB * NB * REP;
  // keys per tile: as many as leave room for BLOCKS blocks per SM (decoded
  // rows and codes per key), at most 8192 / D, a multiple of the 8 warps
  static constexpr int BLOCKS = TABLE <= 48 * 1024 ? 3 : 2;
  static constexpr size_t PER_KEY = sizeof(float) * US + sizeof(uint16_t) * T;
  static constexpr int KT_FIT = static_cast<int>((227 * 1024 / BLOCKS - 1024 - TABLE) / PER_KEY) / 8 * 8;
  static constexpr int KT = KT_FIT < 8192 / D ? KT_FIT : 8192 / D;
  static constexpr size_t SMEM = TABLE + sizeof(float) * KT * US + sizeof(uint16_t) * KT * T;
  static_assert(KT >= 8, "tile of keys");
};

// x as a tf32 head (rounded to nearest) plus the exact fp32 remainder x -
// head. The remainder is passed to the MMA as it is: the tensor core reads
// the tf32 part of the register (truncating it), which is within 2^-10 of
// the remainder, itself at most 2^-11 |x| - so head + remainder carries x to
// about 2^-21.
__device__ __forceinline__ void tf32_split(float x, uint32_t& hi, uint32_t& lo) {
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
  lo = __float_as_uint(x - __uint_as_float(hi));
}

// D += A B for one m16n8k8 tile with tf32 operands and fp32 accumulation.
__device__ __forceinline__ void mma_tf32_1688(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Read-only load of VB bytes (4, 8 or 16; aligned) as 32-bit words.
template <int VB>
__device__ __forceinline__ void ld_words(const unsigned char* p, uint32_t* w) {
  if constexpr (VB == 4) {
    w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
  } else if constexpr (VB == 8) {
    const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = x.x; w[1] = x.y;
  } else {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
  }
}

template <int D, int BD_, int BR_, bool QJL>
__global__ void __launch_bounds__(256, QJL ? 2 : 3) encode_kernel(EncodeArgs a) {
  using Cfg = EncCfg<D, BD_, BR_>;
  constexpr int B = Cfg::MB;  // magnitude bits of a direction cell (b for the OCTOPUS split)
  constexpr int T = Cfg::T, KT = Cfg::KT, US = Cfg::US, W = Cfg::W, C = Cfg::C;
  constexpr int NDIR = Cfg::NDIR, NRHO = Cfg::NRHO;

  constexpr int REP = Cfg::REP;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int NB = Cfg::NB;
  float4* nhat = reinterpret_cast<float4*>(smem_raw);                 // [NB*NB][REP], cell (ix, iy) at (ix+1, iy+1)
  float* U = reinterpret_cast<float*>(nhat + NB * NB * REP);          // [KT][US]
  uint16_t* codes = reinterpret_cast<uint16_t*>(U + KT * US);         // [KT][T]
  __shared__ float s_dir_c[32], s_dir_t[32], s_rho_c[32], s_rho_t[32];
  // Cell search tables: s_tpad[i] = threshold i - 1 (-inf, +inf at the ends),
  // so cell i is s_tpad[i] <= x < s_tpad[i + 1]; s_bin[k] = the cell of the
  // left edge of bin k of 128 equal bins over [-1, 1]. With at most one
  // threshold per bin, the bin's cell is within one of x's cell.
  __shared__ float s_tpad[34];
  __shared__ uint8_t s_bin[128];
  // code-field parts of a direction cell: x's (m | s << 2B) and y's (m << B | s << 2B + 1)
  __shared__ uint16_t s_fx[32], s_fy[32];
  __shared__ int s_bins_ok;
  __shared__ uint32_t sketch[QJL ? KT * (D / 32) : 1];  // [KT][D/32] sketch words of the tile (QJL)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NWARP = Cfg::THREADS / 32;

  if (tid < NDIR) s_dir_c[tid] = a.dir_c[tid];
  if (tid < NDIR - 1) s_dir_t[tid] = a.dir_t[tid];
  if (tid < NRHO) s_rho_c[tid] = a.rho_c[tid];
  if (tid < NRHO - 1) s_rho_t[tid] = a.rho_t[tid];
  if (tid == 0) s_bins_ok = 1;
  __syncthreads();
  if (tid <= NDIR) s_tpad[tid] = tid == 0 ? -INFINITY : (tid == NDIR ? INFINITY : s_dir_t[tid - 1]);
  if (tid < 128) {
    const float left = -1.0f + static_cast<float>(tid) * (1.0f / 64.0f);
    int c = 0;
    for (int k = 0; k < NDIR - 1; ++k) c += s_dir_t[k] <= left;
    s_bin[tid] = static_cast<uint8_t>(c);
  }
  if (tid < NDIR - 2) {  // two thresholds in one bin: the bin search would be off by two
    const int b0 = static_cast<int>(floorf((s_dir_t[tid] + 1.0f) * 64.0f));
    const int b1 = static_cast<int>(floorf((s_dir_t[tid + 1] + 1.0f) * 64.0f));
    if (b0 == b1) atomicAnd(&s_bins_ok, 0);
  }
  if (tid < NDIR) {
    constexpr uint32_t half = 1u << B, ones = (2u << B) - 1u;
    const uint32_t sg = static_cast<uint32_t>(tid) < half;
    const uint32_t m = (static_cast<uint32_t>(tid) ^ (sg ? ones : 0u)) & (half - 1u);
    s_fx[tid] = static_cast<uint16_t>(m | (sg << (2 * B)));
    s_fy[tid] = static_cast<uint16_t>((m << B) | (sg << (2 * B + 1)));
  }
  __syncthreads();
  // a border cell holds NaN: its s = n . t is NaN, and "s > best" is false
  for (int e = tid; e < NB * NB; e += Cfg::THREADS) {
    const int bx = e / NB - 1, by = e % NB - 1;
    float4 v = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000), __int_as_float(0x7fc00000), 0.0f);
    if (bx >= 0 && bx < NDIR && by >= 0 && by < NDIR) {
      const float3 n = oct_inverse(s_dir_c[bx], s_dir_c[by]);
      v = make_float4(n.x, n.y, n.z, 0.0f);
    }
#pragma unroll
    for (int k = 0; k < REP; ++k) nhat[e * REP + ((k + lane) & (REP - 1))] = v;
  }
  __syncthreads();
  // the norm codebook lives in registers: thresholds and centroids
  float rt[NRHO > 1 ? NRHO - 1 : 1], rc[NRHO];
#pragma unroll
  for (int k = 0; k < NRHO - 1; ++k) rt[k] = s_rho_t[k];
#pragma unroll
  for (int k = 0; k < NRHO; ++k) rc[k] = s_rho_c[k];
  const int rep_off = lane & (REP - 1);
  // Cell of x in the direction codebook: start from the uniform-grid cell
  // and step to the exact one (cell i has t[i-1] <= x < t[i]; the Lloyd-Max
  // thresholds are close to uniform, so this takes 0-1 steps).
  const bool bins_ok = s_bins_ok != 0;
  auto dir_index = [&](float x) -> int {
    if (bins_ok) {
      // bin of x by rounding (x + 1) * 64 to an integer in the mantissa of
      // 1.5 * 2^23 + (x + 1) * 64; the bin's cell, then one step either way
      const int bi = min(__float_as_int(fmaf(x, 64.0f, 12582912.0f + 64.0f)) - 0x4B400000, 127);
      int i = s_bin[bi];
      i += x >= s_tpad[i + 1];
      i -= x < s_tpad[i];
      return i;
    }
    int i = __float2int_rd((x + 1.0f) * (0.5f * NDIR));
    i = i < 0 ? 0 : (i > NDIR - 1 ? NDIR - 1 : i);
    while (i > 0 && x < s_dir_t[i - 1]) --i;
    while (i < NDIR - 1 && x >= s_dir_t[i]) ++i;
    return i;
  };
  // Norm level nearest to v (count of thresholds <= v) and its centroid.
  auto rho_level = [&](float v, int& ir, float& rh) {
    ir = 0;
    rh = rc[0];
#pragma unroll
    for (int k = 0; k < NRHO - 1; ++k) {
      const bool up = v >= rt[k];
      ir += up;
      rh = up ? rc[k + 1] : rh;
    }
  };

  const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));

  // Phase 1 layout: LK = D/32 lanes per key, lane jq owning coordinates
  // [32 jq, 32 jq + 32): 5 butterfly stages run in registers and log2(LK)
  // across the key's lanes; a warp holds 32/LK keys at once.
  constexpr int LK = D / 32, KWP = 32 / LK;
  // lane = jq * KWP + kslot: a quarter-warp holds 8 keys (or all of them) at
  // one coordinate block, so its stores of the rotated rows (rows 4 mod 32
  // words apart) fall in distinct bank groups
  const int jq = lane / KWP, kslot = lane % KWP;
  uint32_t smask = 0;  // bit p: s < 0 at coordinate 32 jq + p of head smask_head
  int64_t smask_head = -1;

  // each block walks a contiguous range of tiles (the head, hence the sign
  // vector, changes rarely along it)
  const int64_t per = (a.n_tiles + gridDim.x - 1) / gridDim.x;
  const int64_t tbeg = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t tend = a.n_tiles < tbeg + per ? a.n_tiles : tbeg + per;
  for (int64_t tile = tbeg; tile < tend; ++tile) {
    const int64_t h = tile / a.tiles_per_head;
    const int64_t n0 = (tile % a.tiles_per_head) * KT;
    const int nk = static_cast<int>(a.n_tokens - n0 < KT ? a.n_tokens - n0 : KT);
    if (h != smask_head) {
      const float* srow = a.signs + (h % a.table_heads) * D + 32 * jq;
      smask = 0;
#pragma unroll
      for (int p = 0; p < 32; ++p) smask |= (__ldg(srow + p) < 0.0f ? 1u : 0u) << p;
      smask_head = h;
    }
    __syncthreads();  // previous tile's shared buffers are free
    if constexpr (QJL)
      for (int i = tid; i < KT * (D / 32); i += Cfg::THREADS) sketch[i] = 0u;

    // ---------------- phase 1: LK lanes per key
    // the key's 32 elements of this lane, in loads of the alignment the API
    // guarantees (min(16, D/32 x element size) bytes)
    for (int k0 = warp * KWP; k0 < nk; k0 += NWARP * KWP) {
      const int k = k0 + kslot;
      const bool valid = k < nk;
      float v[32];
      if (!valid) {
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = 0.0f;
      } else if (a.key_bf16) {
        constexpr int VB = (D / 32) * 2 < 16 ? (D / 32) * 2 : 16;
        const unsigned char* p = reinterpret_cast<const unsigned char*>(
            static_cast<const __nv_bfloat16*>(a.keys) + h * a.head_stride + (n0 + k) * a.token_stride + 32 * jq);
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 64 / VB; ++q) ld_words<VB>(p + q * VB, w + q * (VB / 4));
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          v[2 * q] = bf16_lo(w[q]);
          v[2 * q + 1] = bf16_hi(w[q]);
        }
      } else {
        constexpr int VB = (D / 32) * 4 < 16 ? (D / 32) * 4 : 16;
        const unsigned char* p = reinterpret_cast<const unsigned char*>(
            static_cast<const float*>(a.keys) + h * a.head_stride + (n0 + k) * a.token_stride + 32 * jq);
        uint32_t w[32];
#pragma unroll
        for (int q = 0; q < 128 / VB; ++q) ld_words<VB>(p + q * VB, w + q * (VB / 4));
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(w[q]);
      }
      float ss = 0.0f;
#pragma unroll
      for (int q = 0; q < 32; ++q) ss = fmaf(v[q], v[q], ss);
#pragma unroll
      for (int m = KWP; m < LK * KWP; m <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
      const float g = sqrtf(ss);
      // u_rot = H (s * k) / (gamma sqrt(d)): the signs s (exact) on the raw
      // key, the butterflies, then one scale (0 for a zero key)
      const float scale = g > 0.0f ? inv_sqrt_d / g : 0.0f;
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(__float_as_uint(v[q]) ^ ((smask << (31 - q)) & 0x80000000u));
      // H: coordinate bits 0-4 in registers, then bits 5.. across the key's lanes
      fwht32_regs(v);
      fwht32_lanes<LK, KWP>(v, lane);
      if (valid) {
        float* row = U + k * US;
#pragma unroll
        for (int q = 0; q < 32; ++q) row[32 * jq + q] = v[q] * scale;
        if (jq == 0) {
          for (int q = D; q < 3 * T; ++q) row[q] = 0.0f;  // the zero pad of the last triplet
          a.gamma[h * a.cache_cap + a.token_offset + n0 + k] = g;
        }
      }
    }
    __syncthreads();

    // ---------------- phase 2: thread per triplet
    for (int j = tid; j < nk * T; j += Cfg::THREADS) {
      const int k = j / T, i = j - k * T;
      float* tp = U + k * US + 3 * i;
      const float x = tp[0], y = tp[1], z = tp[2];
      const float ax = fabsf(x), ay = fabsf(y);
      const float l1 = ax + ay + fabsf(z);
      // p = t / ||t||_1 (a zero triplet maps to the north pole); the lower
      // hemisphere (p_z < 0) folds to ((1 - |p_y|) sgn p_x, (1 - |p_x|) sgn p_y)
      const float il = l1 > 0.0f ? __fdividef(1.0f, l1) : 0.0f;
      const bool lower = z < 0.0f;
      const float fx = lower ? fmaf(-ay, il, 1.0f) : ax * il;
      const float fy = lower ? fmaf(-ax, il, 1.0f) : ay * il;
      const float xi = x >= 0.0f ? fx : -fx;
      const float eta = y >= 0.0f ? fy : -fy;
      int ix = dir_index(xi);
      int iy = dir_index(eta);
      int ir;
      float rh;
      const float4* nc = nhat + ((ix + 1) * NB + (iy + 1)) * REP + rep_off;  // the centre cell
      float4 nb = *nc;
      if (!a.joint) {
        rho_level(sqrtf(x * x + y * y + z * z), ir, rh);  // rho, only scalar rounding uses it
      } else {
        // For a fixed direction n_hat the best norm level is the centroid
        // nearest s = n_hat . t, and the error is rho^2 + min_l (c_l^2 -
        // 2 c_l s). Every norm centroid c_l is positive, so that error falls
        // strictly as s grows: the candidate of least error is the one with
        // the largest s, and the norm level is searched once, for it.
        // Centre first, then (dx, dy) row-major; replace only on a strictly
        // larger s (a strictly smaller error). Neighbours outside the
        // codebook are border cells whose s is NaN and never wins.
        float sbest = nb.x * x + nb.y * y + nb.z * z;
        int kbest = 4;  // (dx + 1) * 3 + (dy + 1)
#pragma unroll
        for (int k = 0; k < 9; ++k) {
          if (k == 4) continue;
          const float4 n = nc[((k / 3 - 1) * NB + (k % 3 - 1)) * REP];
          const float sc = n.x * x + n.y * y + n.z * z;
          if (sc > sbest) { sbest = sc; kbest = k; }
        }
        ix += kbest / 3 - 1;
        iy += kbest % 3 - 1;
        if constexpr (QJL) nb = nc[((kbest / 3 - 1) * NB + (kbest % 3 - 1)) * REP];
        rho_level(sbest, ir, rh);
      }
      codes[k * T + i] = static_cast<uint16_t>(s_fx[ix] | s_fy[iy] | (ir << (2 * Cfg::BD)));
      if constexpr (QJL) {
        // residual e = t - rho_hat n_hat, in place (the pad coordinate is dropped later)
        tp[0] = x - rh * nb.x;
        tp[1] = y - rh * nb.y;
        tp[2] = z - rh * nb.z;
      }
    }
    __syncthreads();

    // ---------------- phase 3: thread per (key, word), token-contiguous stores
    for (int j = tid; j < nk * W; j += Cfg::THREADS) {
      const int w = j / nk, k = j - w * nk;
      const int first = (32 * w) / C;
      const int last = min(T - 1, (32 * w + 31) / C);
      uint32_t word = 0;
      for (int i = first; i <= last; ++i) {
        const uint32_t code = codes[k * T + i];
        const int sh = i * C - 32 * w;
        word |= sh >= 0 ? (code << sh) : (code >> (-sh));
      }
      a.packed[(h * W + w) * a.cache_cap + a.token_offset + n0 + k] = word;
    }

    if constexpr (QJL) {
      // ---------------- phase 4: sketch bits = [ (S e)_r >= 0 ], nu = ||e||
      // Tensor cores from d = 128 on; at d = 64 the projection is small and
      // the register-blocked FMA form is faster.
      constexpr int QW = D / 32;  // sketch words per key
      if constexpr (D >= 128) {
        // P = S E^T for the tile (rows of S x keys) on tensor cores: mma.sync
        // m16n8k8 with tf32 operands, each operand split into a tf32 head and a
        // tf32 remainder and three products summed (head.head + head.rem +
        // rem.head), about 2^-21 of sum |S_rm e_m| from the fp32 result. A warp
        // takes one 16-row tile of S and a group of up to 4 eight-key tiles; the
        // S fragments of a k-step serve the whole group.
        constexpr int MT = D / 16;                  // row tiles of S
        constexpr int NT = (KT + 7) / 8;            // key tiles
        // key tiles per work item: all of the tile's when that gives one item per
        // warp (the S fragments of a k-step are split once for every key)
        constexpr int NGT = (MT == NWARP && NT <= 8) ? NT : 4;
        constexpr int NG = (NT + NGT - 1) / NGT;
        const float* Sh = a.qjl_S + (h % a.table_heads) * D * D;
        const int g8 = lane >> 2, c4 = lane & 3;
        for (int item = warp; item < MT * NG; item += NWARP) {
          const int mt = item % MT, ng = item / MT;
          float acc[NGT][4];
  #pragma unroll
          for (int t = 0; t < NGT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
          const float* s0 = Sh + (16 * mt + g8) * D + c4;  // A rows g8 and g8 + 8, columns c4 and c4 + 4
  #pragma unroll 2
          for (int k0 = 0; k0 < D; k0 += 8) {
            uint32_t ah[4], al[4];
            tf32_split(__ldg(s0 + k0), ah[0], al[0]);
            tf32_split(__ldg(s0 + 8 * D + k0), ah[1], al[1]);
            tf32_split(__ldg(s0 + k0 + 4), ah[2], al[2]);
            tf32_split(__ldg(s0 + 8 * D + k0 + 4), ah[3], al[3]);
  #pragma unroll
            for (int t = 0; t < NGT; ++t) {
              const int key = (ng * NGT + t) * 8 + g8;   // B column g8: this lane's key of the tile
              if (ng * NGT + t < NT) {
                const float* e = U + (key < KT ? key : 0) * US + k0 + c4;
                uint32_t bh[2], bl[2];
                tf32_split(e[0], bh[0], bl[0]);
                tf32_split(e[4], bh[1], bl[1]);
                mma_tf32_1688(acc[t], al, bh);
                mma_tf32_1688(acc[t], ah, bl);
                mma_tf32_1688(acc[t], ah, bh);
              }
            }
          }
          // rows 16 mt + g8 (+8), keys 8 (ng NGT + t) + 2 c4 (+1)
  #pragma unroll
          for (int t = 0; t < NGT; ++t) {
  #pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = 16 * mt + g8 + 8 * (i >> 1);
              const int key = (ng * NGT + t) * 8 + 2 * c4 + (i & 1);
              if (ng * NGT + t < NT && key < nk && acc[t][i] >= 0.0f)
                atomicOr(&sketch[key * QW + row / 32], 1u << (row % 32));
            }
          }
        }
      } else {
        // Warp w takes rows [w RW, w RW + RW) of S, lane l the keys l + 32 kk:
        // one accumulator per (row, key), so each S value loaded feeds KPL
        // keys and each residual value RW rows. Every sum runs over m in
        // ascending order, as a plain dot product would.
        constexpr int RW = D / NWARP;               // rows per warp
        constexpr int KPL = (KT + 31) / 32;         // keys per lane
        const float* S = a.qjl_S + (h % a.table_heads) * D * D + warp * RW * D;
        float acc[RW][KPL];
  #pragma unroll
        for (int r = 0; r < RW; ++r)
  #pragma unroll
          for (int kk = 0; kk < KPL; ++kk) acc[r][kk] = 0.0f;
        for (int m = 0; m < D; m += 4) {
          float ev[KPL][4];
  #pragma unroll
          for (int kk = 0; kk < KPL; ++kk) {
            const int k = lane + 32 * kk;
            const float* e = U + (k < nk ? k : 0) * US + m;
  #pragma unroll
            for (int i = 0; i < 4; ++i) ev[kk][i] = e[i];
          }
  #pragma unroll
          for (int r = 0; r < RW; ++r) {
            const float4 sv = __ldg(reinterpret_cast<const float4*>(S + r * D + m));
  #pragma unroll
            for (int kk = 0; kk < KPL; ++kk) {
              float t = acc[r][kk];
              t = fmaf(sv.x, ev[kk][0], t);
              t = fmaf(sv.y, ev[kk][1], t);
              t = fmaf(sv.z, ev[kk][2], t);
              acc[r][kk] = fmaf(sv.w, ev[kk][3], t);
            }
          }
        }
        // this warp's RW bits of each key into the key's sketch words
        static_assert(32 % RW == 0 || RW % 32 == 0, "rows per warp and sketch words");
  #pragma unroll
        for (int kk = 0; kk < KPL; ++kk) {
          const int k = lane + 32 * kk;
          if (k < nk) {
  #pragma unroll
            for (int r0 = 0; r0 < RW; r0 += 32) {
              uint32_t bits = 0;
  #pragma unroll
              for (int r = r0; r < r0 + 32 && r < RW; ++r) bits |= (acc[r][kk] >= 0.0f ? 1u : 0u) << (r - r0);
              const int row = warp * RW + r0;  // first sketch row of these bits
              atomicOr(&sketch[k * QW + row / 32], bits << (row % 32));
            }
          }
        }
      }
      for (int k = tid; k < nk; k += Cfg::THREADS) {
        const float* e = U + k * US;
        float ss = 0.0f;
        for (int m = 0; m < D; ++m) ss = fmaf(e[m], e[m], ss);
        a.qjl_norm[h * a.cache_cap + a.token_offset + n0 + k] = sqrtf(ss);
      }
      __syncthreads();
      for (int i = tid; i < nk * QW; i += Cfg::THREADS) {
        const int qw = i / nk, k = i - qw * nk;
        a.qjl_bits[(h * QW + qw) * a.cache_cap + a.token_offset + n0 + k] = sketch[k * QW + qw];
      }
    }
  }
}

template <int D, int BD, int BR, bool QJL>
static cudaError_t launch_encode(const EncodeArgs& a0, cudaStream_t st) {
  using Cfg = EncCfg<D, BD, BR>;
  EncodeArgs a = a0;
  a.tiles_per_head = (a.n_tokens + Cfg::KT - 1) / Cfg::KT;
  a.n_tiles = a.tiles_per_head * a.n_heads;
  const size_t smem = Cfg::SMEM;
  auto kern = encode_kernel<D, BD, BR, QJL>;
  static LaunchCache cache;
  int resident = 0;
  const cudaError_t e = launch_setup(kern, cache, Cfg::THREADS, smem, resident);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(a.n_tiles, resident);
  kern<<<static_cast<unsigned>(grid), Cfg::THREADS, smem, st>>>(a);
  return cudaGetLastError();
}

// The OCTOPUS split (b + 1, b - 1) for every d, with or without the sketch;
// at d = 128 also the other splits of the bit-allocation sweep (direction
// b + delta, norm b - delta for b = 3 with delta in {-1, 0, 2} and b = 4 with
// delta in {-1, 0}), without the sketch.
template <int D>
static cudaError_t dispatch_split(const EncodeArgs& a, int b_dir, int b_rho, bool qjl, cudaStream_t st) {
#define OCTO_ENC(BD, BR)                                                                                 \
  if (b_dir == BD && b_rho == BR)                                                                      \
    return qjl ? launch_encode<D, BD, BR, true>(a, st) : launch_encode<D, BD, BR, false>(a, st);
  OCTO_ENC(3, 1)
  OCTO_ENC(4, 2)
  OCTO_ENC(5, 3)
#undef OCTO_ENC
  if constexpr (D == 128) {
    if (!qjl) {
      if (b_dir == 2 && b_rho == 4) return launch_encode<D, 2, 4, false>(a, st);
      if (b_dir == 3 && b_rho == 3) return launch_encode<D, 3, 3, false>(a, st);
      if (b_dir == 5 && b_rho == 1) return launch_encode<D, 5, 1, false>(a, st);
      if (b_dir == 3 && b_rho == 5) return launch_encode<D, 3, 5, false>(a, st);
      if (b_dir == 4 && b_rho == 4) return launch_encode<D, 4, 4, false>(a, st);
    }
  }
  return cudaErrorNotSupported;
}

}  // namespace octo

extern "C" int octo_encode(const octo_layout* L, const octo_tables* tab, const void* keys, int key_dtype,
                           int64_t n_heads, int64_t n_tokens, int64_t head_stride, int64_t token_stride,
                           int64_t cache_cap, int64_t token_offset, uint32_t* packed, float* gamma,
                           uint32_t* qjl_bits, float* qjl_norm, octo_stream_t stream) {
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
  if (key_dtype != OCTO_F32 && key_dtype != OCTO_BF16) return OCTO_EINVAL;
  if (n_heads < 0 || n_tokens < 0 || token_offset < 0 || cache_cap < 0) return OCTO_EINVAL;
  if (token_offset + n_tokens > cache_cap) return OCTO_EINVAL;
  if (n_heads == 0 || n_tokens == 0) return OCTO_OK;
  if (!keys || !packed || !gamma || !tab->dir_c || !tab->dir_t || !tab->rho_c || !tab->signs ||
      tab->n_heads < 1)
    return OCTO_EINVAL;
  if (L->n_rho > 1 && !tab->rho_t) return OCTO_EINVAL;
  if (L->qjl && (!qjl_bits || !qjl_norm || !tab->qjl_S)) return OCTO_EINVAL;
  if (L->qjl && reinterpret_cast<uintptr_t>(tab->qjl_S) % 16 != 0) return OCTO_EINVAL;
  if (head_stride < 0 || token_stride < 0) return OCTO_EINVAL;
  const int esz = key_dtype == OCTO_F32 ? 4 : 2;
  // each lane loads D/32 contiguous elements with one vector load
  const int64_t vec = std::min<int64_t>(16, static_cast<int64_t>(L->d / 32) * esz);
  if (reinterpret_cast<uintptr_t>(keys) % vec != 0 || (head_stride * esz) % vec != 0 ||
      (token_stride * esz) % vec != 0)
    return OCTO_EINVAL;
  EncodeArgs a{};
  a.keys = keys;
  a.key_bf16 = key_dtype == OCTO_BF16;
  a.n_heads = n_heads;
  a.n_tokens = n_tokens;
  a.head_stride = head_stride;
  a.token_stride = token_stride;
  a.cache_cap = cache_cap;
  a.token_offset = token_offset;
  a.packed = packed;
  a.gamma = gamma;
  a.qjl_bits = qjl_bits;
  a.qjl_norm = qjl_norm;
  a.dir_c = tab->dir_c;
  a.dir_t = tab->dir_t;
  a.rho_c = tab->rho_c;
  a.rho_t = tab->rho_t;
  a.signs = tab->signs;
  a.qjl_S = tab->qjl_S;
  a.table_heads = tab->n_heads;
  a.joint = L->rounding == OCTO_ROUND_JOINT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (L->d) {
    case 64: e = dispatch_split<64>(a, L->b_dir, L->b_rho, L->qjl != 0, st); break;
    case 128: e = dispatch_split<128>(a, L->b_dir, L->b_rho, L->qjl != 0, st); break;
    default: e = dispatch_split<256>(a, L->b_dir, L->b_rho, L->qjl != 0, st); break;
  }
  if (e == cudaErrorNotSupported) return OCTO_EUNSUPPORTED;  // a split without a built kernel (nothing launched)
  return e == cudaSuccess ? OCTO_OK : OCTO_ECUDA;
}
