// OCTOPUS fused decode attention for sm_100a: the kernel template.
//
// One step of decode attention over a compressed key cache (explainer,
// "engineering implementation": decompression, dot products and online
// softmax happen on chip, the uncompressed keys are never written out; the
// abstract: keys are reconstructed on the fly without materialising them).
//
// Math per KV head (b, h) with query rows r (GQA group x query tokens):
//   q_rot_r = (1/sqrt(d)) H (s_h * q_r)                    (rotated once)
//   logit_rn = gamma_n * sum_i rho_hat_in (q_rot_r,i . n_hat_in)
//              [+ gamma_n nu_n sqrt(pi/2)/d <S q_rot_r, 2 bits_n - 1>]  (QJL)
//   out_r = softmax_n(scale * logit_rn) V_n
// Because R is orthogonal, q . k_hat = gamma q_rot . u_rot_hat, so the keys
// are never inverse-rotated.
//
// The file holds three kernels. decode_tc_kernel (further below) serves
// every head dimension up to 128: logits and P.V on tensor cores, whole
// rounds of keys staged by TMA tensor copies from a producer warp, 10 to 12
// consumer warps. With OCTOPUS-QJL it is preceded by decode_prep_kernel,
// which rotates the query rows and forms p = S q_rot once per KV head.
// decode_kernel, described here, serves d = 256 (where the tensor-core
// layout does not fit in shared memory):
//
// Structure of decode_kernel (one CTA = one KV head x one contiguous slice
// of the cache, 8 warps, every warp a consumer, thread 0 also the producer):
//  * The slice is cut into stages of CK = 512 keys. For each stage thread 0
//    issues TMA bulk copies (cp.async.bulk, completion on an mbarrier) of the
//    stage's code words and gammas (and sketch words and residual norms)
//    into a ring of NS shared-memory buffers, and a bulk L2 prefetch of the
//    stage's V rows. NS stages are in flight; a buffer is refilled after the
//    block-wide barrier that ends its stage.
//  * prologue (overlapping the first copies): codebooks -> a shared-memory
//    table of decoded triplets, replicated 8x so that the 8 lanes of a
//    quarter-warp read distinct bank groups (b = 2: rho_hat * n_hat for every
//    full code; b >= 3: n_hat for every direction code, rho_hat from a
//    4/8-entry table); queries rotated by warp-shuffle WHT into a compact
//    triplet-major layout; for QJL, p = S q_rot and a 4-bit lookup table of
//    signed partial sums of p.
//  * per stage and warp: 64 keys, two per lane. Logits by table lookups and
//    FMAs; online softmax (m, l) per query row in base 2; P.V on tensor
//    cores (mma.sync m16n8k16 bf16; P split into bf16 hi + lo so the product
//    keeps ~16 mantissa bits) with V read from L2 straight into A-fragment
//    registers (16-byte loads + byte permutes).
//  * epilogue: warps merge (m, l, O) in shared memory (reusing the stage
//    ring); CTAs of a head merge
//    through the workspace, the last-arriving CTA (atomic ticket, no
//    spinning) writes the normalised output and resets the ticket.
//  * Every wait on an mbarrier is bounded; on expiry the kernel records
//    OCTO_DEVICE_TIMEOUT in the workspace status word and returns.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "octo_common.cuh"

namespace octo {

constexpr int OCTO_DEVICE_TIMEOUT = 1;  // status-word bit: a bounded device wait expired

struct DecodeArgs {
  const void* q;
  int q_bf16;
  int B, Hq, Hkv, Lq, g, Gq;  // g = Hq / Hkv, Gq = g * Lq query rows per KV head
  int64_t kv_len, cache_cap;
  const uint32_t* packed;
  const float* gamma;
  const uint32_t* qjl_bits;
  const float* qjl_norm;
  const __nv_bfloat16* V;
  float scale_log2;  // scale * log2(e)
  float* out;
  float* logits;
  const float* dir_c;
  const float* rho_c;
  const float* signs;
  const float* qjl_S;
  int64_t table_heads;
  // Slices of the cache per head: heads [heads_lo, B * Hkv) have n_splits
  // slices of keys_per_split keys, heads [0, heads_lo) n_splits_lo slices of
  // keys_per_split_lo keys (n_splits_lo <= n_splits; the grid is n_splits
  // wide, and the partials take n_splits slots per head).
  int n_splits;
  int64_t keys_per_split;
  int heads_lo, n_splits_lo;
  int64_t keys_per_split_lo;
  int* status;
  int* counters;
  // OCTOPUS-QJL, tensor-core kernel: per KV head, the rotated query rows and
  // p = S q_rot as the kernel's query scratch image ([G][QROW] then [G][D]
  // floats, prep_stride floats a head), written by decode_prep_kernel
  float* prep;
  int64_t prep_stride;
  float* part_m;
  float* part_l;
  float* part_o;
};

// Build-time tuning knobs (the defaults are the measured best on B200).
#ifndef OCTO_DECODE_MAX_WARPS
#define OCTO_DECODE_MAX_WARPS 8   // warps per CTA (16 only if shared memory allows)
#endif
#ifndef OCTO_DECODE_KPL
#define OCTO_DECODE_KPL 4         // keys per lane per chunk (d <= 128; half of it for d = 256)
#endif
#ifndef OCTO_DECODE_FOLD_BITS
#define OCTO_DECODE_FOLD_BITS 10  // full-code table when a triplet code has at most this many bits
#endif

template <int D, int B, int G, bool QJL>
struct DecCfg {
  static constexpr int T = (D + 2) / 3;
  static constexpr int BD = B + 1, BR = B - 1;
  static constexpr int C = 2 * BD + BR;
  static constexpr int W = (T * C + 31) / 32;
  static constexpr int NDIR = 1 << BD, NRHO = 1 << BR;
  static constexpr bool FOLD = C <= OCTO_DECODE_FOLD_BITS;  // table indexed by the full code (b <= 3)
  static constexpr int NE = FOLD ? (1 << C) : (1 << (2 * BD));
  static constexpr int REP = NE <= 256 ? 8 : 4;           // replicas per entry (bank groups)
  static constexpr int KPL = D <= 128 ? OCTO_DECODE_KPL : (OCTO_DECODE_KPL + 1) / 2;  // keys per lane per chunk
  static constexpr int KW = 32 * KPL;                      // keys per chunk (one warp's unit of work)
  static constexpr int NS_MAX = 2;                         // chunks in flight per warp (at most)
  static constexpr int QF = 3 * G;                         // rotated-query floats per triplet
  static constexpr int QV = (QF + 3) / 4;                  // ... as float4
  static constexpr int QW = D / 32;                        // sketch words per key
  static constexpr int PSTRIDE = 40;                       // floats per P row (bank-conflict-free reads)
  static constexpr int MT = D / 16;                        // m-tiles of O^T
  static constexpr int NCH = D / 64;                       // 16-byte V chunks per key per lane
  static constexpr int GV = (G + 3) / 4;                   // float4 per LUT entry
  // one chunk buffer: W code rows, a gamma row (+ QW sketch rows, a norm row)
  static constexpr int ROWS = W + 1 + (QJL ? QW + 1 : 0);
  static constexpr size_t CHUNK = sizeof(uint32_t) * ROWS * KW;
  static constexpr size_t TABLE = sizeof(float4) * NE * REP;
  static constexpr size_t QT = sizeof(float4) * T * QV;
  static constexpr size_t LUT = QJL ? sizeof(float4) * (D / 4) * 16 * GV : 0;
  static constexpr size_t QROW = D + 4;                    // floats per scratch query row
  static constexpr size_t SCRATCH = sizeof(float) * G * (QROW + (QJL ? D : 0));
  static constexpr size_t BUDGET = 227 * 1024 - 2048;
  // per-warp bytes: its P buffer and its chunk ring (the ring is reused for
  // the warp's (m, l, O) in the epilogue)
  static constexpr size_t PER_WARP_P = sizeof(float) * G * PSTRIDE;
  // a warp's ring also holds its (m, l, O) in the epilogue, and the rings
  // together the split-merge weights (G x up to 1024 splits, 8+ warps)
  static constexpr size_t cmax(size_t x, size_t y) { return x > y ? x : y; }
  static constexpr size_t ring_bytes(int ns) {
    return (cmax(cmax(ns * CHUNK, sizeof(float) * G * (D + 2)), sizeof(float) * G * 1024 / 8) + 127) / 128 * 128;
  }
  static constexpr size_t FIXED = TABLE + QT + LUT + SCRATCH;
  static constexpr bool fits(int nw, int ns) { return FIXED + nw * (PER_WARP_P + ring_bytes(ns)) <= BUDGET; }
  // prefer 16 warps (latency hiding), then double buffering
  static constexpr int NWARP = (OCTO_DECODE_MAX_WARPS >= 16 && fits(16, 1)) ? 16 : 8;
  static_assert(fits(8, 1), "shared memory budget");
  static constexpr int NS = fits(NWARP, NS_MAX) ? NS_MAX : 1;
  static constexpr size_t RING = ring_bytes(NS);  // keeps every ring 128-byte aligned
  static_assert(RING * 8 >= sizeof(float) * G * 1024, "split-merge weights fit in the rings");
  static constexpr int THREADS = 32 * NWARP;
  static constexpr size_t PBUF = PER_WARP_P * NWARP;
  static constexpr size_t SMEM = FIXED + PBUF + RING * NWARP;
  static_assert(SMEM <= BUDGET, "shared memory budget");
};

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  // a pure register operation: not volatile, so the scheduler may interleave it
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// hi + lo bf16 split of two fp32 values: x ~= hi + lo with |x - hi - lo| <~ 2^-17 |x|.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(x0, x1);
  const float r0 = x0 - bf16_lo(hi), r1 = x1 - bf16_hi(hi);
  lo = pack_bf16x2(r0, r1);
}

// split_bf16x2 of a pair with the two subtractions as one packed operation
__device__ __forceinline__ void split_bf16x2_v(float2 v, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(v.x, v.y);
  const float2 r = sub_f32x2(v, make_float2(bf16_lo(hi), bf16_hi(hi)));
  lo = pack_bf16x2(r.x, r.y);
}

// bf16 hi + lo of (z, 0): the zero half needs no arithmetic.
__device__ __forceinline__ void split_bf16_z0(float z, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(z, 0.0f);
  lo = pack_bf16x2(z - bf16_lo(hi), 0.0f);
}

// 2^x with the hardware approximation (PTX ex2.approx: relative error about
// 2^-22, 2^-inf = 0); softmax weights need far less.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- mbarrier / bulk-copy helpers (PTX) -----------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: false if the phase did not complete within the limit.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  for (int it = 0; it < (1 << 22); ++it)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// global -> shared bulk copy completing on `bar`; 16-byte aligned, size % 16 == 0
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

template <int D, int B, int G, bool QJL>
__global__ void __launch_bounds__(DecCfg<D, B, G, QJL>::THREADS, 1) decode_kernel(DecodeArgs a) {
  using Cfg = DecCfg<D, B, G, QJL>;
  constexpr int T = Cfg::T, C = Cfg::C, W = Cfg::W, BD = Cfg::BD, NDIR = Cfg::NDIR;
  constexpr int NE = Cfg::NE, REP = Cfg::REP, NWARP = Cfg::NWARP, QW = Cfg::QW;
  constexpr int PS = Cfg::PSTRIDE, MT = Cfg::MT, NCH = Cfg::NCH, GV = Cfg::GV;
  constexpr int KPL = Cfg::KPL, KW = Cfg::KW, QV = Cfg::QV, NS = Cfg::NS, ROWS = Cfg::ROWS;

  extern __shared__ __align__(128) unsigned char smem_raw[];
  float4* table = reinterpret_cast<float4*>(smem_raw);                                   // [NE*REP]
  float4* qt = reinterpret_cast<float4*>(smem_raw + Cfg::TABLE);                         // [T][QV]
  float4* lut = reinterpret_cast<float4*>(smem_raw + Cfg::TABLE + Cfg::QT);              // [D/4][16][GV]
  float* scratch = reinterpret_cast<float*>(smem_raw + Cfg::TABLE + Cfg::QT + Cfg::LUT);
  float* pbuf = reinterpret_cast<float*>(smem_raw + Cfg::FIXED);                         // [NWARP][G][PS]
  unsigned char* rings = smem_raw + Cfg::FIXED + Cfg::PBUF;                              // [NWARP] RING bytes
  constexpr int QROW = static_cast<int>(Cfg::QROW);
  __shared__ __align__(8) uint64_t full[NWARP][NS];
  __shared__ float s_rho_c[8];
  __shared__ float s_dir_c[32];
  __shared__ int s_last;
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x;
  const int bh = blockIdx.y;  // b * Hkv + h_kv
  const int bidx = bh / a.Hkv, hkv = bh - bidx * a.Hkv;
  const int64_t trow = bh % a.table_heads;
  const bool with_v = a.V != nullptr;

  const bool lo_head = bh < a.heads_lo;
  const int n_sl = lo_head ? a.n_splits_lo : a.n_splits;  // this head's slices
  const int64_t kps = lo_head ? a.keys_per_split_lo : a.keys_per_split;
  if (split >= n_sl) return;  // a grid slot this head does not use (nothing touched yet)
  const int64_t k_begin = static_cast<int64_t>(split) * kps;
  const int64_t k_end = min(a.kv_len, k_begin + kps);
  // chunks of KW keys, dealt to warps round-robin: warp w takes chunks w, w + NWARP, ...
  const int n_chunks = static_cast<int>((k_end - k_begin + KW - 1) / KW);
  const int my_chunks = warp < n_chunks ? (n_chunks - warp + NWARP - 1) / NWARP : 0;
  const uint32_t* pk = a.packed + static_cast<int64_t>(bh) * W * a.cache_cap;
  const float* gm = a.gamma + static_cast<int64_t>(bh) * a.cache_cap;
  const __nv_bfloat16* Vh = with_v ? a.V + static_cast<int64_t>(bh) * a.cache_cap * D : nullptr;
  const uint32_t* qbp = QJL ? a.qjl_bits + static_cast<int64_t>(bh) * QW * a.cache_cap : nullptr;
  const float* qnp = QJL ? a.qjl_norm + static_cast<int64_t>(bh) * a.cache_cap : nullptr;
  uint32_t* ring = reinterpret_cast<uint32_t*>(rings + warp * Cfg::RING);                // [NS][ROWS][KW]

  // This warp's i-th chunk: lane 0 arms the barrier, lanes < ROWS each copy
  // one row (code words, gammas, sketch words, norms) into ring slot i % NS,
  // lane ROWS prefetches the chunk's V rows into L2. Keys are copied in
  // groups of 4 (16 bytes); the capacity is a multiple of 4 and chunks start
  // at multiples of KW, so the rounded-up copy stays inside the cache rows.
  auto issue_chunk = [&](int i) {
    const int64_t s0 = k_begin + static_cast<int64_t>(warp + NWARP * i) * KW;
    const int n = static_cast<int>(k_end - s0 < KW ? k_end - s0 : KW);
    const uint32_t bytes = static_cast<uint32_t>(((n + 3) & ~3) * 4);
    uint32_t* buf = ring + (i % NS) * ROWS * KW;
    uint64_t* bar = &full[warp][i % NS];
    if (lane == 0) mbar_expect_tx(bar, bytes * ROWS);
    __syncwarp();
    for (int r = lane; r <= ROWS; r += 32) {
      if (r < W) {
        bulk_g2s(buf + r * KW, pk + r * a.cache_cap + s0, bytes, bar);
      } else if (r == W) {
        bulk_g2s(buf + W * KW, gm + s0, bytes, bar);
      } else if (QJL && r < W + 1 + QW) {
        const int w = r - W - 1;
        bulk_g2s(buf + (W + 1 + w) * KW, qbp + w * a.cache_cap + s0, bytes, bar);
      } else if (QJL && r == W + 1 + QW) {
        bulk_g2s(buf + (W + 1 + QW) * KW, qnp + s0, bytes, bar);
      } else if (r == ROWS && with_v) {
        bulk_prefetch_l2(Vh + s0 * D, static_cast<uint32_t>(n) * D * 2);
      }
    }
  };

  // The few small global reads of the prologue go first, ahead of the bulk
  // traffic that the chunk copies start: codebooks, and one query row per
  // warp (sign-flipped, in registers).
  constexpr int E = D / 32;
  float qraw[E];
  if (tid < NDIR) s_dir_c[tid] = a.dir_c[tid];
  if (tid < Cfg::NRHO) s_rho_c[tid] = a.rho_c[tid];
  {
    const int r = warp;
    if (r < G && r < a.Gq) {
      const int gi = r / a.Lq, lq = r - gi * a.Lq;
      const int64_t qoff = ((static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq) * D + lane * E;
      const float* sg = a.signs + trow * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float x = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[qoff + e])
                                 : static_cast<const float*>(a.q)[qoff + e];
        qraw[e] = x * __ldg(sg + e);
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) qraw[e] = 0.0f;
    }
  }
  if (tid == 0) {
    s_abort = 0;
    for (int w = 0; w < NWARP; ++w)
      for (int s = 0; s < NS; ++s) mbar_init(&full[w][s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  for (int i = 0; i < NS && i < my_chunks; ++i) issue_chunk(i);

  // ------------------------------------------------ prologue (overlaps the first copies)
  for (int e = tid; e < NE; e += Cfg::THREADS) {
    int ix, iy;
    direction_cells<B>(static_cast<uint32_t>(e), ix, iy);
    float3 n = oct_inverse(s_dir_c[ix], s_dir_c[iy]);
    if constexpr (Cfg::FOLD) {
      const float r = s_rho_c[e >> (2 * BD)];
      n.x *= r; n.y *= r; n.z *= r;
    }
    const float4 v = make_float4(n.x, n.y, n.z, 0.0f);
    // replica order rotated by lane so that each store instruction hits distinct bank groups
#pragma unroll
    for (int k = 0; k < REP; ++k) table[e * REP + ((k + lane) & (REP - 1))] = v;
  }
  // rotate the query rows: warp r handles row r (G <= 8 <= NWARP)
  static_assert(G <= NWARP, "one warp per query row");
  if (warp < G) {
    fwht_warp<E>(qraw, lane);
    const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
    float* qrow = scratch + warp * QROW;  // padded rotated row
#pragma unroll
    for (int e = 0; e < E; ++e) qrow[lane * E + e] = qraw[e] * inv_sqrt_d;
    if (lane < 3 * T - D) qrow[D + lane] = 0.0f;
  }
  __syncthreads();
  // compact triplet-major layout: triplet i holds (row0 xyz, row1 xyz, ...) padded to QV float4
  for (int j = tid; j < T * QV * 4; j += Cfg::THREADS) {
    const int i = j / (QV * 4), f = j - i * (QV * 4);
    const int r = f / 3, c = f - 3 * r;
    reinterpret_cast<float*>(qt)[j] = r < G ? scratch[r * QROW + 3 * i + c] : 0.0f;
  }
  if constexpr (QJL) {
    // p_r = S q_rot_r (D outputs per row), then the 4-bit signed-sum table.
    float* p = scratch + G * QROW;  // [G][D]
    const float* S = a.qjl_S + trow * D * D;
    for (int j = tid; j < G * D; j += Cfg::THREADS) {
      const int r = j / D, m = j - r * D;
      const float* qrow = scratch + r * QROW;
      const float* srow = S + static_cast<int64_t>(m) * D;
      float acc = 0.0f;
      for (int t = 0; t < D; ++t) acc = fmaf(__ldg(srow + t), qrow[t], acc);
      p[j] = acc;
    }
    __syncthreads();
    for (int j = tid; j < (D / 4) * 16; j += Cfg::THREADS) {
      const int grp = j >> 4, nib = j & 15;
      float vals[4 * GV];
#pragma unroll
      for (int r = 0; r < 4 * GV; ++r) {
        float s = 0.0f;
        if (r < G) {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float pv = p[r * D + 4 * grp + t];
            s += ((nib >> t) & 1) ? pv : -pv;
          }
        }
        vals[r] = s;
      }
#pragma unroll
      for (int v4 = 0; v4 < GV; ++v4)
        lut[j * GV + v4] = make_float4(vals[4 * v4], vals[4 * v4 + 1], vals[4 * v4 + 2], vals[4 * v4 + 3]);
    }
  }
  __syncthreads();

  // ------------------------------------------------ main loop: this warp's chunks
  const int g8 = lane >> 2, c4 = lane & 3;
  const int rep_off = lane & (REP - 1);

  float m_run[G], l_run[G];
#pragma unroll
  for (int r = 0; r < G; ++r) { m_run[r] = -INFINITY; l_run[r] = 0.0f; }
  float acc_o[MT][4];
#pragma unroll
  for (int t = 0; t < MT; ++t) acc_o[t][0] = acc_o[t][1] = acc_o[t][2] = acc_o[t][3] = 0.0f;
  float* pw = pbuf + warp * G * PS;
  int aborted_at = -1;

  // V fragments of 16-key step j of a chunk (keys s0 + 16 j + {2c4, 2c4+1,
  // 2c4+8, 2c4+9}, 16-byte columns 8 g8 + 64 hh); step j + 1 is loaded while
  // step j multiplies, step 0 while the chunk's logits are computed.
  constexpr bool VPIPE = NCH <= 2;
  auto load_v_step = [&](uint4 (&dst)[4][NCH], int64_t s0v, int j) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int64_t vk = s0v + 16 * j + 2 * c4 + (kk & 1) + 8 * (kk >> 1);
#pragma unroll
      for (int hh = 0; hh < NCH; ++hh)
        dst[kk][hh] = vk < k_end ? __ldg(reinterpret_cast<const uint4*>(Vh + vk * D + 64 * hh + 8 * g8))
                                 : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 vcur[4][NCH], vnext[4][NCH];  // vnext is dead unless VPIPE

  for (int ci = 0; ci < my_chunks; ++ci) {
    const uint32_t* buf = ring + (ci % NS) * ROWS * KW;
    const int64_t s0 = k_begin + static_cast<int64_t>(warp + NWARP * ci) * KW;
    if (VPIPE && with_v) load_v_step(vcur, s0, 0);  // in flight during the wait and the logits
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[warp][ci % NS], (ci / NS) & 1))) {
      aborted_at = ci;  // warp-uniform
      break;
    }

    int lk[KPL];
    bool valid[KPL];
    float gk[KPL];
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      lk[k] = 32 * k + lane;
      valid[k] = s0 + lk[k] < k_end;
      gk[k] = valid[k] ? __uint_as_float(buf[W * KW + lk[k]]) : 0.0f;
    }

    float lg[KPL][G];
#pragma unroll
    for (int k = 0; k < KPL; ++k)
#pragma unroll
      for (int r = 0; r < G; ++r) lg[k][r] = 0.0f;

#pragma unroll
    for (int i = 0; i < T; ++i) {
      float qv[4 * QV];
#pragma unroll
      for (int v = 0; v < QV; ++v) {
        const float4 t4 = qt[i * QV + v];
        qv[4 * v] = t4.x; qv[4 * v + 1] = t4.y; qv[4 * v + 2] = t4.z; qv[4 * v + 3] = t4.w;
      }
      constexpr uint32_t mask = (1u << C) - 1u;
      const int pos = i * C, wi = pos >> 5, sh = pos & 31;
#pragma unroll
      for (int k = 0; k < KPL; ++k) {
        uint32_t code;
        if (sh + C <= 32) code = (buf[wi * KW + lk[k]] >> sh) & mask;
        else code = __funnelshift_r(buf[wi * KW + lk[k]], buf[(wi + 1) * KW + lk[k]], sh) & mask;
        float4 u;
        if constexpr (Cfg::FOLD) {
          u = table[code * REP + rep_off];
        } else {
          const float4 n = table[(code & ((1u << (2 * BD)) - 1u)) * REP + rep_off];
          const float rh = s_rho_c[code >> (2 * BD)];
          u = make_float4(n.x * rh, n.y * rh, n.z * rh, 0.0f);
        }
#pragma unroll
        for (int r = 0; r < G; ++r)
          lg[k][r] = fmaf(qv[3 * r], u.x, fmaf(qv[3 * r + 1], u.y, fmaf(qv[3 * r + 2], u.z, lg[k][r])));
      }
    }

#pragma unroll
    for (int k = 0; k < KPL; ++k) {
#pragma unroll
      for (int r = 0; r < G; ++r) lg[k][r] *= gk[k];
      if constexpr (QJL) {
        float corr[4 * GV];
#pragma unroll
        for (int r = 0; r < 4 * GV; ++r) corr[r] = 0.0f;
#pragma unroll
        for (int w = 0; w < QW; ++w) {
          const uint32_t word = buf[(W + 1 + w) * KW + lk[k]];
#pragma unroll
          for (int j8 = 0; j8 < 8; ++j8) {
            const uint32_t nib = (word >> (4 * j8)) & 15u;
            const int j = 8 * w + j8;
#pragma unroll
            for (int v4 = 0; v4 < GV; ++v4) {
              const float4 t = lut[(j * 16 + nib) * GV + v4];
              corr[4 * v4] += t.x; corr[4 * v4 + 1] += t.y; corr[4 * v4 + 2] += t.z; corr[4 * v4 + 3] += t.w;
            }
          }
        }
        const float nu = valid[k] ? __uint_as_float(buf[(W + 1 + QW) * KW + lk[k]]) : 0.0f;
        const float f = gk[k] * nu * (1.2533141373155003f / static_cast<float>(D));  // sqrt(pi/2)/m, m = d
#pragma unroll
        for (int r = 0; r < G; ++r) lg[k][r] = fmaf(f, corr[r], lg[k][r]);
      }
    }
    // this warp is done with the chunk's rows: refill the slot with chunk ci + NS
    __syncwarp();
    if (ci + NS < my_chunks) issue_chunk(ci + NS);

    if (a.logits != nullptr) {
#pragma unroll
      for (int k = 0; k < KPL; ++k) {
        if (!valid[k]) continue;
#pragma unroll
        for (int r = 0; r < G; ++r) {
          if (r < a.Gq) {
            const int gi = r / a.Lq, lq = r - gi * a.Lq;
            const int64_t row = (static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq;
            a.logits[row * a.kv_len + s0 + lk[k]] = lg[k][r];
          }
        }
      }
    }
    if (!with_v) continue;

    // online softmax over the chunk, base 2
    bool grew = false;
    float alpha[G];
#pragma unroll
    for (int r = 0; r < G; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < KPL; ++k) {
        lg[k][r] = valid[k] ? lg[k][r] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, lg[k][r]);
      }
      const float mn = fmaxf(m_run[r], warp_max(mx));
      grew |= mn > m_run[r];
      alpha[r] = fast_exp2(m_run[r] - mn);  // m_run = -inf -> 0
      float ps = 0.0f;
#pragma unroll
      for (int k = 0; k < KPL; ++k) {
        lg[k][r] = fast_exp2(lg[k][r] - mn);  // invalid keys: 2^-inf = 0
        ps += lg[k][r];
      }
      l_run[r] = l_run[r] * alpha[r] + ps;
      m_run[r] = mn;
    }
    if (grew) {  // warp-uniform: the maxima are warp-wide
      float sa0 = 0.0f, sa1 = 0.0f;  // this lane's accumulator columns are rows 2*c4, 2*c4+1
#pragma unroll
      for (int r = 0; r < G; ++r) {
        sa0 = (r == 2 * c4) ? alpha[r] : sa0;
        sa1 = (r == 2 * c4 + 1) ? alpha[r] : sa1;
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        acc_o[t][0] *= sa0; acc_o[t][1] *= sa1; acc_o[t][2] *= sa0; acc_o[t][3] *= sa1;
      }
    }

    // P.V: KPL sub-chunks of 32 keys (lane = key), each two 16-key k-steps.
#pragma unroll
    for (int j = 0; j < 2 * KPL; ++j) {
      const int k = j >> 1, ks = j & 1;
      const int64_t kb = s0 + 32 * k;
      if (kb >= k_end) break;  // warp-uniform
      if (ks == 0) {
#pragma unroll
        for (int r = 0; r < G; ++r) pw[r * PS + lane] = lg[k][r];
        __syncwarp();
      }
      if constexpr (VPIPE) {
        if (j + 1 < 2 * KPL) load_v_step(vnext, s0, j + 1);  // keys past the end load as zeros
      } else {
        load_v_step(vcur, s0, j);
      }
      uint32_t bh0 = 0, bl0 = 0, bh1 = 0, bl1 = 0;
      if (g8 < G) {
        const float* prow = pw + g8 * PS + 16 * ks + 2 * c4;
        const float2 p01 = *reinterpret_cast<const float2*>(prow);
        const float2 p89 = *reinterpret_cast<const float2*>(prow + 8);
        split_bf16x2(p01.x, p01.y, bh0, bl0);
        split_bf16x2(p89.x, p89.y, bh1, bl1);
      }
#pragma unroll
      for (int hh = 0; hh < NCH; ++hh) {
        const uint4 k0 = vcur[0][hh], k1 = vcur[1][hh], k8 = vcur[2][hh], k9 = vcur[3][hh];
        const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w}, w1[4] = {k1.x, k1.y, k1.z, k1.w};
        const uint32_t w8[4] = {k8.x, k8.y, k8.z, k8.w}, w9[4] = {k9.x, k9.y, k9.z, k9.w};
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const uint32_t a0 = __byte_perm(w0[e2], w1[e2], 0x5410);
          const uint32_t a1 = __byte_perm(w0[e2], w1[e2], 0x7632);
          const uint32_t a2 = __byte_perm(w8[e2], w9[e2], 0x5410);
          const uint32_t a3 = __byte_perm(w8[e2], w9[e2], 0x7632);
          mma_bf16_16816(acc_o[hh * 4 + e2], a0, a1, a2, a3, bh0, bh1);
          mma_bf16_16816(acc_o[hh * 4 + e2], a0, a1, a2, a3, bl0, bl1);
        }
      }
      if constexpr (VPIPE) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
          for (int hh = 0; hh < NCH; ++hh) vcur[kk][hh] = vnext[kk][hh];
      }
      if (ks == 1) __syncwarp();  // the P rows of this sub-chunk are consumed
    }
  }

  if (aborted_at >= 0 && lane == 0) {
    atomicOr(a.status, OCTO_DEVICE_TIMEOUT);
    s_abort = 1;
    // chunks issued but not consumed (the one that timed out and up to NS-1
    // after it) must land before the shared memory is reused or released
    for (int c = aborted_at; c < aborted_at + NS && c < my_chunks; ++c)
      mbar_wait_bounded(&full[warp][c % NS], (c / NS) & 1);
  }
  __syncthreads();
  if (s_abort || !with_v) return;

  // ------------------------------------------------ epilogue: merge warps (in each warp's ring)
#pragma unroll
  for (int r = 0; r < G; ++r) l_run[r] = warp_sum(l_run[r]);
  auto wm = [&](int w) { return reinterpret_cast<float*>(rings + w * Cfg::RING); };          // [G] m
  auto wl = [&](int w) { return reinterpret_cast<float*>(rings + w * Cfg::RING) + G; };      // [G] l
  auto wo = [&](int w) { return reinterpret_cast<float*>(rings + w * Cfg::RING) + 2 * G; };  // [G][D] O
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < G; ++r) { wm(warp)[r] = m_run[r]; wl(warp)[r] = l_run[r]; }
  }
  {
    float* o = wo(warp);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int hh = t >> 2, e2 = t & 3;
      const int d0 = 64 * hh + 8 * g8 + 2 * e2;
      const int q0 = 2 * c4, q1 = 2 * c4 + 1;
      if (q0 < G) { o[q0 * D + d0] = acc_o[t][0]; o[q0 * D + d0 + 1] = acc_o[t][2]; }
      if (q1 < G) { o[q1 * D + d0] = acc_o[t][1]; o[q1 * D + d0 + 1] = acc_o[t][3]; }
    }
  }
  __syncthreads();

  const int S = n_sl, SW = a.n_splits;  // this head's slices; partial slots per head
  float* pm = a.part_m + (static_cast<int64_t>(bh) * SW + split) * G;
  float* pl = a.part_l + (static_cast<int64_t>(bh) * SW + split) * G;
  float* po = a.part_o + (static_cast<int64_t>(bh) * SW + split) * G * D;
  for (int j = tid; j < G * D; j += Cfg::THREADS) {
    const int r = j / D, d = j - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) M = fmaxf(M, wm(w)[r]);
    float o = 0.0f, l = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NWARP; ++w) {
        const float f = fast_exp2(wm(w)[r] - M);
        o = fmaf(f, wo(w)[r * D + d], o);
        l = fmaf(f, wl(w)[r], l);
      }
    }
    if (S == 1) {
      if (r < a.Gq) {
        const int gi = r / a.Lq, lq = r - gi * a.Lq;
        const int64_t row = (static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq;
        a.out[row * D + d] = l > 0.0f ? o / l : 0.0f;
      }
    } else {
      po[j] = o;
      if (d == 0) { pm[r] = M; pl[r] = l; }
    }
  }
  if (S == 1) return;

  // ------------------------------------------------ epilogue: merge splits (last CTA of this head)
  __syncthreads();
  if (tid == 0) {
    // release our partials (written by this CTA, ordered by the barrier) and,
    // for the last arrival, acquire everyone else's
    int ticket;
    asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(ticket) : "l"(a.counters + bh) : "memory");
    s_last = ticket == S - 1;
  }
  __syncthreads();
  if (!s_last) return;
  const float* bm = a.part_m + static_cast<int64_t>(bh) * SW * G;
  const float* bl = a.part_l + static_cast<int64_t>(bh) * SW * G;
  const float* bo = a.part_o + static_cast<int64_t>(bh) * SW * G * D;
  // every thread loads its (row, column)'s S partials plus the row's (m, l)
  // in one round (independent, coalesced over d), then combines them
  for (int j = tid; j < a.Gq * D; j += Cfg::THREADS) {
    const int r = j / D, d = j - r * D;
    float M = -INFINITY;
#pragma unroll 8
    for (int s2 = 0; s2 < S; ++s2) M = fmaxf(M, __ldcg(bm + s2 * G + r));
    float o = 0.0f, l = 0.0f;
    if (M != -INFINITY) {
#pragma unroll 8
      for (int s2 = 0; s2 < S; ++s2) {
        const float f = fast_exp2(__ldcg(bm + s2 * G + r) - M);
        o = fmaf(f, __ldcg(bo + (static_cast<int64_t>(s2) * G + r) * D + d), o);
        l = fmaf(f, __ldcg(bl + s2 * G + r), l);
      }
    }
    const int gi = r / a.Lq, lq = r - gi * a.Lq;
    const int64_t row = (static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq;
    a.out[row * D + d] = l > 0.0f ? o / l : 0.0f;
  }
  if (tid == 0) atomicExch(a.counters + bh, 0);  // ready for the next call
}

// ---------------------------------------------------------------------------
// Tensor-core logits (d <= 128, every bit budget b in {2, 3, 4}).
//
// For a GQA group the logits of a tile of keys are a dense contraction,
// logits[key][row] = sum_c u_hat[key][c] q_rot[row][c], so they run on
// mma.sync m16n8k16 bf16 with keys as M, query rows as N and rotated
// coordinates as K. Each 16-wide k-step holds 4 triplets: lane column c4
// carries triplet 4s + c4 as (x, y | z, 0), so a lane decodes one triplet
// code per key per k-step. For b = 3 the shared-memory table holds the
// decoded triplets rho_hat * n_hat of the positive-level quadrant (codes with
// both direction signs clear), already split into bf16 hi + lo halves in
// exactly the A-fragment register order ({xy_hi, z0_hi, xy_lo, z0_lo}); a
// code's two direction signs flip the sign bits of x and y in the fragment
// registers (the codebook is odd-symmetric and the octahedral inverse map is
// odd in each coordinate, so this is exact). b = 2 indexes a table of every
// signed code, and b = 4 looks up the direction and the signed norm apart
// (TcCfg). The rotated queries are B fragments held in registers for the
// whole CTA.
//
// OCTOPUS-QJL: the sketch sum <S q_rot, 2 bits - 1> runs on the 8-bit
// integer tensor cores (mma.sync m16n8k32, unsigned 0/1 sketch bytes x
// signed bytes of S q_rot rounded per query row to 16 bits), interleaved
// with the logit k-steps; the integer sums are exact.
//
// Precision: with at most 4 query rows (HL layout) the 8 MMA columns hold the
// rows' bf16 hi halves (columns 0-3) and lo halves (columns 4-7), so two
// products (A_hi B, A_lo B) give all four hi/lo cross terms and a lane adds
// its column n and n + 4 (lane c4 and c4 ^ 2) at the end. With 8 rows the
// columns are all taken and three products (hi.hi + hi.lo + lo.hi) are
// used. Either way the logits keep about 16 mantissa bits, well inside the
// logit tolerance. P.V uses the same layouts with P split into hi + lo.
//
// Memory pipeline: the CTA's key range is cut into rounds of CPR chunks of
// 16 keys, one chunk per consumer warp of a team (the consumer warps form
// NWARP / CPR teams that take the rounds in turn). A producer warp stages whole rounds
// into a ring of shared-memory stages with a few large tensor copies (TMA:
// the round's V as two 128-byte-swizzled boxes, its gammas, one code box per
// chunk), completion counted on the stage's full barrier; the consumer
// warps release a stage on its empty barrier. The load/store unit then only
// serves shared-memory reads, and no consumer ever waits on a copy issue.
// ---------------------------------------------------------------------------
#ifndef OCTO_DECODE_F32X2
#define OCTO_DECODE_F32X2 1  // packed fp32 pairs for the split-norm products and residuals
#endif
#ifndef OCTO_DECODE_SR_MIN_B
#define OCTO_DECODE_SR_MIN_B 4  // bit budgets from which the norm is looked up apart from the direction
#endif
// Rounds in flight at most (shared-memory stages; fewer when they do not fit).
#ifdef OCTO_DECODE_TC_STAGES
constexpr int tc_stages(int, int) { return OCTO_DECODE_TC_STAGES; }
#else
constexpr int tc_stages(int d, int) { return d <= 64 ? 4 : 6; }
#endif

// Consumer warps per CTA, and 16-key chunks per round. A warp's chunk is a
// long dependent sequence (code and table reads, MMAs, softmax, P.V), so
// more warps hide more of it; the round size sets the stage size, and with
// it how many rounds fit in flight. When there are more warps than chunks,
// the warps form teams that take the rounds in turn (team t: rounds t,
// t + teams, ...), so warps can be added without growing the stages.
// Measured best: for d = 128, 10 warps in two teams over 5-chunk rounds
// (6 stages; against 8 warps over 8-chunk rounds, 4 stages: 2 % faster at
// b = 4 and 3), for d = 64, 12 warps over 12-chunk rounds.
// OCTO_DECODE_TC_WARPS / OCTO_DECODE_TC_CHUNKS override the choice.
#ifdef OCTO_DECODE_TC_WARPS
constexpr int tc_warps(int, int) { return OCTO_DECODE_TC_WARPS; }
#else
constexpr int tc_warps(int d, int) { return d <= 64 ? 12 : 10; }
#endif
#ifdef OCTO_DECODE_TC_CHUNKS
constexpr int tc_chunks(int, int) { return OCTO_DECODE_TC_CHUNKS; }
#else
constexpr int tc_chunks(int d, int) { return d <= 64 ? 12 : 5; }
#endif

// Floats per rotated query row in the tensor-core kernel's scratch: whole
// k-steps of 4 triplets (12 floats), at least d + 4.
constexpr int tc_qrow(int d) { return 12 * (((d + 2) / 3 + 3) / 4) > d + 4 ? 12 * (((d + 2) / 3 + 3) / 4) : d + 4; }

// Keys of one round (the tensor maps' boxes are built for this size).
constexpr int tc_round_keys(int d, int b) { return 16 * tc_chunks(d, b); }

// Tensor maps of one decode call (built on the host; token extents are
// kv_len, so rows past the end arrive as zeros).
struct TmaDesc {
  CUtensorMap v;      // bf16 [heads][kv_len][D], box 64 x round, 128-byte swizzle
  CUtensorMap codes;  // u32 [heads][W][kv_len], box 16 keys x W
  CUtensorMap gamma;  // f32 [heads][kv_len], box round
  CUtensorMap qbits;  // u32 [heads][D/32][kv_len], box round x D/32 (OCTOPUS-QJL)
  CUtensorMap qnorm;  // f32 [heads][kv_len], box round (OCTOPUS-QJL)
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int D, int B, int G, bool QJL>
struct TcCfg {
  static constexpr int T = (D + 2) / 3;
  static constexpr int BD = B + 1, BR = B - 1;
  static constexpr int C = 2 * BD + BR;
  static constexpr int W = (T * C + 31) / 32;
  static constexpr int NDIR = 1 << BD, NRHO = 1 << BR;
  // Decoded-triplet table. For b <= 3 it covers the positive-level quadrant
  // (m_xi, m_eta, i_rho) with rho_hat * n_hat pre-split into bf16 hi + lo.
  // For b >= OCTO_DECODE_SR_MIN_B ("split rho") that table would have 2048
  // entries, too many to replicate in shared memory, so the direction and
  // the norm are looked up apart: n_hat of the quadrant (m_xi, m_eta) as
  // fp32, and a small table of signed norm pairs (s_x rho_hat, s_y rho_hat)
  // indexed by (s_xi, s_eta, i_rho); the product and the hi + lo split are
  // formed in registers (the same fp32 product, so the same fragments).
  static constexpr bool SR = B >= OCTO_DECODE_SR_MIN_B;
  // A code of at most 8 bits (b = 2) indexes a full table of every signed
  // code directly (128 entries, 16 KB with 8 replicas): no quadrant index,
  // no sign masks.
  static constexpr bool FULL = !SR && C <= 8;
  static constexpr int NE = SR ? (1 << (2 * B)) : (FULL ? (1 << C) : (1 << (3 * B - 1)));
  // replicas: 8 give every lane of a quarter-warp its own bank group (no
  // conflicts); a full 2048-entry b = 4 table keeps 2 to stay in shared memory
  static constexpr int REP = NE <= 256 ? 8 : 2;
  static constexpr int NSR = SR ? (1 << (B + 1)) : 0;  // signed norm pairs (s_x, s_y, i_rho)
  static constexpr int REP_SR = 16;                    // one 8-byte slot per lane of a half-warp
  static constexpr int NKS = (T + 3) / 4;    // logit k-steps (4 triplets each)
  static constexpr bool HL = G <= 4;         // hi and lo halves side by side in the MMA columns
  static constexpr int NB = HL ? 2 : 4;      // query B-fragment registers per k-step
  static constexpr int KW = 16;              // keys per consumer chunk (one m-tile)
  static constexpr int QW = D / 32;          // sketch words per key
  static constexpr int QKS = D / 32;         // sketch k-steps (32 coordinates each, 8-bit operands)
  static constexpr int NWARP = tc_warps(D, B);         // consumer warps
  static constexpr int CPR = tc_chunks(D, B);          // chunks per round
  static constexpr int NTEAM = NWARP / CPR;            // teams taking the rounds in turn
  static_assert(NWARP % CPR == 0, "whole teams");
  static constexpr int THREADS = 32 * (NWARP + 1);     // + the producer warp
  static constexpr int NS_MAX = tc_stages(D, B);
  static constexpr int RK = tc_round_keys(D, B);  // keys per round
  static constexpr int MT = D / 16, NCH = D / 64;
  // one stage: V (NCH swizzled boxes of RK rows x 128 bytes), per-warp code
  // boxes [W][16], gammas, (sketch words [QW][RK], norms); parts 128-byte aligned
  static constexpr int VHALF = RK * 128;
  static constexpr int CW = (4 * W * KW + 127) / 128 * 128;
  static constexpr int ST_V = 0;
  static constexpr int ST_C = ST_V + NCH * VHALF;
  static constexpr int ST_G = ST_C + CPR * CW;
  static constexpr int ST_Q = ST_G + (4 * RK + 127) / 128 * 128;
  static constexpr int ST_N = ST_Q + (QJL ? 4 * QW * RK : 0);
  static constexpr int ST_END = ST_N + (QJL ? (4 * RK + 127) / 128 * 128 : 0);
  static constexpr int STAGE = (ST_END + 1023) / 1024 * 1024;
  static constexpr int PS = KW + 8;          // P row stride (floats)
  static constexpr size_t TABLE = sizeof(uint4) * NE * REP + sizeof(float2) * NSR * REP_SR;
  static constexpr size_t QROW = tc_qrow(D);  // padded rotated query row
  static constexpr size_t SCRATCH = (sizeof(float) * G * (QROW + (QJL ? D : 0)) + 15) / 16 * 16;
  // OCTOPUS-QJL: the query scratch arrives from decode_prep_kernel's output
  // with the first round (one bulk copy of the whole image)
  static constexpr uint32_t PREP_BYTES = QJL ? static_cast<uint32_t>(sizeof(float) * G * (QROW + D)) : 0u;
  static_assert(PREP_BYTES % 16 == 0, "bulk copy size");
  static constexpr size_t PBUF = (sizeof(float) * G * PS + 15) / 16 * 16;  // per consumer warp
  // offsets from a 1024-byte aligned base
  static constexpr size_t BUDGET = 227 * 1024 - 2048;
  // shared memory without the stages (+ alignment slack)
  static constexpr size_t REST = NWARP * PBUF + TABLE + SCRATCH + 1024;
  // as many stages as fit, up to NS_MAX
  static constexpr int fit_stages(int n) { return n <= 2 || REST + size_t(n) * STAGE <= BUDGET ? n : fit_stages(n - 1); }
  static constexpr int NS = fit_stages(NS_MAX);
  static constexpr size_t SREG = 0;                                  // [NS] stages
  static constexpr size_t PREG = SREG + size_t(NS) * STAGE;          // [NWARP] P
  static constexpr size_t TREG = PREG + NWARP * PBUF;                // table
  static constexpr size_t QREG = TREG + TABLE;                       // query scratch
  static constexpr size_t SMEM = QREG + SCRATCH + 1024;              // + alignment slack
  static constexpr bool FITS = SMEM <= BUDGET && NWARP >= G;  // (one warp per query row in the prologue)
  static constexpr uint32_t TX_FIXED = (QJL ? 4u * QW * RK + 4u * RK : 0u) + 4u * RK;  // gammas (+ sketch, norms)
  static constexpr uint32_t TX_CHUNK = 4u * W * KW;                                     // one code box
  static_assert(G <= 8 && D <= 128 && NCH >= 1, "tensor-core logits shape");
  static_assert(CPR >= 4 && RK <= 256 && NS >= 2, "chunks per round, box rows, stages");
  static_assert(VHALF % 1024 == 0 && ST_C % 128 == 0 && ST_G % 128 == 0 && ST_Q % 128 == 0 && ST_N % 128 == 0,
                "alignment of the stage parts");
  static_assert(size_t(NS) * STAGE >= sizeof(float) * NWARP * G * (D + 2), "the warp merge reuses the stages");
};

// Table row of a triplet code m_x | m_y << B | s_x << 2B | s_y << (2B+1) |
// i_rho << (2B+2): the magnitudes and the norm index, signs dropped.
template <int B>
__device__ __forceinline__ uint32_t quadrant_index(uint32_t code) {
  return (code & ((1u << (2 * B)) - 1u)) | ((code >> (2 * B + 2)) << (2 * B));
}
// The code's direction signs at the sign bits of the bf16 pair (x, y):
// s_x -> bit 15, s_y -> bit 31. One multiply forms code << (15 - 2B) plus
// code << (30 - 2B); for a code of at most 13 bits (b <= 4) the two copies
// do not overlap, so the sum is their OR and nothing else lands on bit 15
// or bit 31.
template <int B>
__device__ __forceinline__ uint32_t quadrant_signs(uint32_t code) {
  static_assert(B <= 4, "non-overlapping shifted copies");
  return (code * ((1u << (15 - 2 * B)) + (1u << (30 - 2 * B)))) & 0x80008000u;
}

// Four 8x8 b16 matrices from shared memory, transposed (ldmatrix): lanes
// 8i .. 8i+7 give the row addresses of matrix i, register i receives it.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                              const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

// D += A B for one m16n8k32 tile, A unsigned and B signed 8-bit operands,
// 32-bit integer accumulation (exact).
__device__ __forceinline__ void mma_u8s8_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int D, int B, int G, bool QJL>
__global__ void __launch_bounds__(TcCfg<D, B, G, QJL>::THREADS, 1)
    decode_tc_kernel(DecodeArgs a, const __grid_constant__ TmaDesc tm) {
  using Cfg = TcCfg<D, B, G, QJL>;
  static_assert(Cfg::FITS, "shared memory budget");
  constexpr int T = Cfg::T, C = Cfg::C, NDIR = Cfg::NDIR;
  constexpr int NE = Cfg::NE, REP = Cfg::REP, NWARP = Cfg::NWARP, NKS = Cfg::NKS;
  constexpr int KW = Cfg::KW, NS = Cfg::NS, RK = Cfg::RK;
  constexpr int PS = Cfg::PS, MT = Cfg::MT, NCH = Cfg::NCH, QKS = Cfg::QKS, NB = Cfg::NB;
  constexpr bool HL = Cfg::HL;
  constexpr int QROW = static_cast<int>(Cfg::QROW);
  constexpr uint32_t HALF = 1u << B;

  extern __shared__ __align__(128) unsigned char smem_raw[];
  // 1024-byte aligned base: the swizzled V boxes follow the address bits
  unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint4* table = reinterpret_cast<uint4*>(base + Cfg::TREG);        // [NE][REP]
  float* scratch = reinterpret_cast<float*>(base + Cfg::QREG);      // [G][QROW] (+ [G][D])
  __shared__ __align__(8) uint64_t full[NS], empty[NS];
  __shared__ float s_rho_c[8];
  __shared__ float s_dir_c[32];
  __shared__ int s_last;
  __shared__ int s_abort;
  __shared__ float s_qscale[8];  // OCTOPUS-QJL: per query row scale of the integer sketch projections
  __shared__ float s_qsum[8];    // ... and the sum of those integers

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool producer = warp == NWARP;
  const int g8 = lane >> 2, c4 = lane & 3;
  const int split = blockIdx.x;
  const int bh = blockIdx.y;  // b * Hkv + h_kv
  const int bidx = bh / a.Hkv, hkv = bh - bidx * a.Hkv;
  const int64_t trow = bh % a.table_heads;
  const bool with_v = a.V != nullptr;

  const bool lo_head = bh < a.heads_lo;
  const int n_sl = lo_head ? a.n_splits_lo : a.n_splits;  // this head's slices
  const int64_t kps = lo_head ? a.keys_per_split_lo : a.keys_per_split;
  if (split >= n_sl) return;  // a grid slot this head does not use (nothing touched yet)
  const int64_t k_begin = static_cast<int64_t>(split) * kps;
  const int64_t k_end = min(a.kv_len, k_begin + kps);
  // rounds of RK keys; consumer warp w (team w / CPR, chunk cw = w % CPR)
  // takes keys [16 cw, 16 cw + 16) of every NTEAM-th round
  const int n_rounds = k_end > k_begin ? static_cast<int>((k_end - k_begin + RK - 1) / RK) : 0;
  auto stage_base = [&](int s) { return base + Cfg::SREG + static_cast<size_t>(s) * Cfg::STAGE; };
  float* pw = reinterpret_cast<float*>(base + Cfg::PREG + (producer ? 0 : warp) * Cfg::PBUF);  // [G][PS]

  // Round r into stage r % NS (producer lane 0): arm the full barrier with
  // the byte count of the boxes (boxes past kv_len arrive zero-filled and
  // count in full), then copy the V boxes, the gammas (sketch words, norms)
  // and one code box per chunk that starts inside the range.
  auto issue_round = [&](int r) {
    const int64_t r0 = k_begin + static_cast<int64_t>(r) * RK;
    const int nch = static_cast<int>((min(k_end - r0, static_cast<int64_t>(RK)) + KW - 1) / KW);
    const int s = r % NS;
    unsigned char* st = stage_base(s);
    uint64_t* bar = &full[s];
    const int x = static_cast<int>(r0);
    const bool prep = QJL && r == 0;  // the first round also brings the query scratch image
    mbar_expect_tx(bar, Cfg::TX_FIXED + static_cast<uint32_t>(nch) * Cfg::TX_CHUNK +
                            (with_v ? static_cast<uint32_t>(NCH * Cfg::VHALF) : 0u) + (prep ? Cfg::PREP_BYTES : 0u));
    if (prep) bulk_g2s(scratch, a.prep + bh * a.prep_stride, Cfg::PREP_BYTES, bar);
    if (with_v) {
#pragma unroll
      for (int hh = 0; hh < NCH; ++hh) tma_load_3d(st + Cfg::ST_V + hh * Cfg::VHALF, &tm.v, 64 * hh, x, bh, bar);
    }
    tma_load_2d(st + Cfg::ST_G, &tm.gamma, x, bh, bar);
    if constexpr (QJL) {
      tma_load_3d(st + Cfg::ST_Q, &tm.qbits, x, 0, bh, bar);
      tma_load_2d(st + Cfg::ST_N, &tm.qnorm, x, bh, bar);
    }
    for (int c = 0; c < nch; ++c) tma_load_3d(st + Cfg::ST_C + c * Cfg::CW, &tm.codes, x + c * KW, 0, bh, bar);
  };

  // The small global reads (codebooks, one sign-flipped query row per warp)
  // are issued first, ahead of the bulk copies in the memory queues.
  constexpr int E = D / 32;
  float qraw[E];
  const float dir_v = tid < NDIR ? __ldg(a.dir_c + tid) : 0.0f;
  const float rho_v = tid < Cfg::NRHO ? __ldg(a.rho_c + tid) : 0.0f;
  if (!QJL && warp < G && warp < a.Gq) {
    const int gi = warp / a.Lq, lq = warp - gi * a.Lq;
    const int64_t qoff = ((static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq) * D + lane * E;
    const float* sg = a.signs + trow * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float x = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[qoff + e])
                               : static_cast<const float*>(a.q)[qoff + e];
      qraw[e] = x * __ldg(sg + e);
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) qraw[e] = 0.0f;
  }
  if (producer && lane == 0) {
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Cfg::CPR);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int r = 0; r < NS && r < n_rounds; ++r) issue_round(r);
  }
  if (tid == 0) s_abort = 0;
  if (tid < NDIR) s_dir_c[tid] = dir_v;
  if (tid < Cfg::NRHO) s_rho_c[tid] = rho_v;
  __syncthreads();

  // ------------------------------------------------ prologue (overlaps the first copies)
  // decoded-triplet table of the positive quadrant (cells HALF + m_xi,
  // HALF + m_eta), pre-split into bf16 hi + lo fragment halves
  for (int e = tid; e < NE; e += Cfg::THREADS) {
    const int ix = static_cast<int>(HALF + (e & (HALF - 1))), iy = static_cast<int>(HALF + ((e >> B) & (HALF - 1)));
    float3 n = oct_inverse(s_dir_c[ix], s_dir_c[iy]);
    uint4 v;
    if constexpr (Cfg::SR) {
      v = make_uint4(__float_as_uint(n.x), __float_as_uint(n.y), __float_as_uint(n.z), 0u);
    } else {
      // quadrant entries: the norm index sits above the magnitudes; full
      // entries: above the two direction signs, which flip x and y (the
      // codebook and the inverse map are odd in each coordinate)
      const float r = s_rho_c[Cfg::FULL ? (e >> (2 * B + 2)) : (e >> (2 * B))];
      if constexpr (Cfg::FULL) {
        if ((e >> (2 * B)) & 1) n.x = -n.x;
        if ((e >> (2 * B + 1)) & 1) n.y = -n.y;
      }
      n.x *= r; n.y *= r; n.z *= r;
      uint32_t xyh, xyl, zh, zl;
      split_bf16x2(n.x, n.y, xyh, xyl);
      split_bf16x2(n.z, 0.0f, zh, zl);
      v = make_uint4(xyh, zh, xyl, zl);
    }
#pragma unroll
    for (int k = 0; k < REP; ++k) table[e * REP + ((k + lane) & (REP - 1))] = v;
  }
  if constexpr (Cfg::SR) {
    // signed norm pairs: entry s_x | s_y << 1 | i_rho << 2 holds (s_x ? -rho : rho, s_y ? -rho : rho)
    float2* srt = reinterpret_cast<float2*>(table + NE * REP);
    for (int e = tid; e < Cfg::NSR * Cfg::REP_SR; e += Cfg::THREADS) {
      const int idx = e / Cfg::REP_SR;
      const float r = s_rho_c[idx >> 2];
      srt[e] = make_float2((idx & 1) ? -r : r, (idx & 2) ? -r : r);
    }
  }
  if constexpr (QJL) {
    // the query scratch image (rotated rows, p = S q_rot) lands with the
    // first round; on a timeout the main loop times out on the same round
    const bool ok = n_rounds == 0 || mbar_wait_bounded(&full[0], 0);
    if (!ok && lane == 0) atomicOr(a.status, OCTO_DEVICE_TIMEOUT);
  } else {
    // rotate the query rows: warp r handles row r
    if (warp < G) {
      fwht_warp<E>(qraw, lane);
      const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
      float* qrow = scratch + warp * QROW;
#pragma unroll
      for (int e = 0; e < E; ++e) qrow[lane * E + e] = qraw[e] * inv_sqrt_d;
      for (int c = D + lane; c < QROW; c += 32) qrow[c] = 0.0f;  // zero pad to whole k-steps
    }
  }
  __syncthreads();

  // B fragments of the rotated queries: triplet 4s + c4 as (x, y | z, 0) of
  // MMA column g8, i.e. query row g8 & 3, lo half for g8 >= 4 (HL), or row
  // g8 with separate hi and lo registers (8 rows)
  const int brow = HL ? (g8 & 3) : g8;
  const bool blo = HL && g8 >= 4;
  uint32_t bq[NKS][NB];
#pragma unroll
  for (int s = 0; s < NKS; ++s) {
    const int t = 4 * s + c4;
    float x = 0.0f, y = 0.0f, z = 0.0f;
    if (brow < G) {
      const float* qrow = scratch + brow * QROW;
      x = qrow[3 * t]; y = qrow[3 * t + 1]; z = qrow[3 * t + 2];
    }
    uint32_t xyh, xyl, zh, zl;
    split_bf16x2(x, y, xyh, xyl);
    split_bf16x2(z, 0.0f, zh, zl);
    if constexpr (HL) {
      bq[s][0] = blo ? xyl : xyh;
      bq[s][1] = blo ? zl : zh;
    } else {
      bq[s][0] = xyh; bq[s][1] = zh; bq[s][NB - 2] = xyl; bq[s][NB - 1] = zl;
    }
  }
  // Sketch B fragments: p_r = S q_rot_r as 16-bit integers v = round(p /
  // scale_r), scale_r = max_m |p_rm| / 32639, held as signed bytes hi = floor((v
  // + 128) / 256) and lo = v - 256 hi (so v = 256 hi + lo, |hi| <= 127). The A
  // operand is the sketch bits themselves as 0/1 bytes, and
  // sum_m v_m (2 b_m - 1) = 2 sum_m v_m b_m - sum_m v_m, the last a constant of
  // the row: exact integer arithmetic throughout. The k order is a relabelling
  // of the coordinates chosen so that a lane's A fragment is its sketch word
  // shifted and masked: in k-step ks (word ks), lane c4 takes bits c4 + 8i
  // (k = 4c4 + i) and c4 + 4 + 8i (k = 4c4 + 16 + i), i < 4; over the four
  // lanes: all 32 bits.
  uint32_t bp[QJL ? QKS : 1][NB];
  float qscale0 = 0.0f, qscale1 = 0.0f;  // scales of this lane's query columns q0, q1 (below)
  float qsum0 = 0.0f, qsum1 = 0.0f;      // their sum_m v_m
  if constexpr (QJL) {
    const float* pq = scratch + G * QROW;  // [G][D]
    if (warp < G) {  // row warp: max |p| -> scale, then sum_m v_m
      float mx = 0.0f;
      for (int m = lane; m < D; m += 32) mx = fmaxf(mx, fabsf(pq[warp * D + m]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float sc = mx / 32639.0f, inv = sc > 0.0f ? 1.0f / sc : 0.0f;
      int vs = 0;
      for (int m = lane; m < D; m += 32) vs += max(-32639, min(32639, __float2int_rn(pq[warp * D + m] * inv)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) vs += __shfl_xor_sync(0xffffffffu, vs, o);
      if (lane == 0) { s_qscale[warp] = sc; s_qsum[warp] = static_cast<float>(vs); }
    }
    __syncthreads();
    auto qbytes = [&](int r, int m0, bool lo_bytes) -> uint32_t {  // 4 bytes of coordinates m0 + 8i
      uint32_t w = 0;
      if (r < G) {
        const float sc = s_qscale[r], inv = sc > 0.0f ? 1.0f / sc : 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int v = max(-32639, min(32639, __float2int_rn(pq[r * D + m0 + 8 * i] * inv)));
          const int hi = (v + 128) >> 8, lo = v - 256 * hi;
          w |= (static_cast<uint32_t>(lo_bytes ? lo : hi) & 0xFFu) << (8 * i);
        }
      }
      return w;
    };
#pragma unroll
    for (int ks = 0; ks < QKS; ++ks) {
      const int m0 = 32 * ks + c4;
      if constexpr (HL) {
        bp[ks][0] = qbytes(brow, m0, blo);
        bp[ks][1] = qbytes(brow, m0 + 4, blo);
      } else {
        bp[ks][0] = qbytes(brow, m0, false); bp[ks][1] = qbytes(brow, m0 + 4, false);
        bp[ks][NB - 2] = qbytes(brow, m0, true); bp[ks][NB - 1] = qbytes(brow, m0 + 4, true);
      }
    }
  }
  // where this lane's triplet code of each k-step sits in a key's bit stream
  // (word << 8 | shift). A padding triplet (t >= T) reads code 0's position:
  // its query coordinates are zero, so whatever entry it finds adds nothing.
  // With split norm tables the code is taken from bit p - 7 of the stream, so
  // that it arrives shifted left by 7 (the byte offset of a 128-byte table
  // row); rows are then counted from -1 (+1 in cpos) and the first code of
  // the stream comes from the pair (row -1, row 0) shifted by 25 - the seven
  // low bits read from row -1 (other shared data) fall below the masks.
  constexpr bool PRESHIFT = Cfg::SR || Cfg::FULL;
  constexpr int PRE = PRESHIFT ? 7 : 0;
  uint32_t cpos[NKS];
#pragma unroll
  for (int s = 0; s < NKS; ++s) {
    const int t = 4 * s + c4;
    const int p = (t < T ? t * C : 0) - PRE + (PRESHIFT ? 32 : 0);
    cpos[s] = (static_cast<uint32_t>(p >> 5) << 8) | static_cast<uint32_t>(p & 31);
  }
  const int rep_off = lane & (REP - 1);
  const uint32_t rep16 = static_cast<uint32_t>(rep_off) * 16u;                      // byte offset of this lane's replica
  const uint32_t sr8 = static_cast<uint32_t>(lane & (Cfg::REP_SR - 1)) * 8u;       // ... in the signed norm table

  // ------------------------------------------------ main loop
  // This lane's query columns: HL lanes c4 and c4 ^ 2 hold the same two rows
  // (hi and lo columns before the pairwise add), 8-row lanes rows 2c4, 2c4+1.
  const int q0 = HL ? 2 * (c4 & 1) : 2 * c4, q1 = q0 + 1;
  if constexpr (QJL) {
    qscale0 = q0 < G ? s_qscale[q0] : 0.0f;
    qscale1 = q1 < G ? s_qscale[q1] : 0.0f;
    qsum0 = q0 < G ? s_qsum[q0] : 0.0f;
    qsum1 = q1 < G ? s_qsum[q1] : 0.0f;
  }
  const bool owner = !HL || c4 < 2;  // writes this lane's columns (the HL mirror lanes do not)
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
  float acc_o[MT][4];
#pragma unroll
  for (int t = 0; t < MT; ++t) acc_o[t][0] = acc_o[t][1] = acc_o[t][2] = acc_o[t][3] = 0.0f;
  bool aborted = false;

  if (producer) {
    // Stage round r once the consumers have released its stage (their round
    // r - NS). Every wait is bounded; on expiry the kernel records the status
    // and stops issuing. Before the block may exit, the copies of the last
    // rounds issued have landed (again bounded).
    if (lane == 0) {
      int issued = n_rounds < NS ? n_rounds : NS;
      for (int r = NS; r < n_rounds; ++r) {
        if (!mbar_wait_bounded(&empty[r % NS], ((r / NS) - 1) & 1)) {
          aborted = true;
          break;
        }
        issue_round(r);
        issued = r + 1;
      }
      for (int r = issued > NS ? issued - NS : 0; r < issued; ++r)
        if (!mbar_wait_bounded(&full[r % NS], (r / NS) & 1)) aborted = true;
    }
  } else {
    const int cw = warp % Cfg::CPR;
    for (int r = warp / Cfg::CPR; r < n_rounds; r += Cfg::NTEAM) {
      const int s = r % NS;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (r / NS) & 1))) {
        aborted = true;  // warp-uniform
        break;
      }
      const unsigned char* st = stage_base(s);
      const int64_t s0 = k_begin + static_cast<int64_t>(r) * RK + cw * KW;
      if (s0 < k_end) {  // warp-uniform: this warp's chunk of the round has keys
      // Logits of the chunk in C-fragment layout. Rows are permuted so that a
      // lane owns 2 consecutive keys: row g8 is key 2 g8, row g8 + 8 is key
      // 2 g8 + 1; one 8-byte load gives a code word (or gamma, or sketch word)
      // of both. lgv = (key 2g8, q0), (same, q1), (key 2g8+1, q0), (same, q1).
      float lgv[4];
      {
        constexpr int NC = HL ? 2 : 3;  // independent accumulator chains
        float acc[NC][4];
  #pragma unroll
        for (int c = 0; c < NC; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;
        const uint32_t* bk = reinterpret_cast<const uint32_t*>(st + Cfg::ST_C + cw * Cfg::CW) + 2 * g8 -
                             (PRESHIFT ? KW : 0);
        // OCTOPUS-QJL: the sketch contraction runs interleaved with the logit
        // k-steps (independent work between dependent MMAs), in two
        // accumulator chains (even and odd sketch k-steps)
        // integer accumulators: the hi-byte and lo-byte products (the HL
        // layout keeps both in one, as separate columns)
        int accq[HL ? 1 : 2][4] = {};
        const uint32_t* qk = QJL ? reinterpret_cast<const uint32_t*>(st + Cfg::ST_Q) + cw * KW + 2 * g8 : nullptr;
        auto qjl_step = [&](int ks) {
          // bits c4 + 8i of word ks to byte i (a0, a1), bits c4 + 4 + 8i likewise (a2, a3)
          const uint2 w2 = *reinterpret_cast<const uint2*>(qk + ks * RK);
          const uint32_t a0 = (w2.x >> c4) & 0x01010101u, a1 = (w2.y >> c4) & 0x01010101u;
          const uint32_t a2 = (w2.x >> (c4 + 4)) & 0x01010101u, a3 = (w2.y >> (c4 + 4)) & 0x01010101u;
          mma_u8s8_16832(accq[0], a0, a1, a2, a3, bp[ks][0], bp[ks][1]);
          if constexpr (!HL) mma_u8s8_16832(accq[HL ? 0 : 1], a0, a1, a2, a3, bp[ks][NB - 2], bp[ks][NB - 1]);
        };
  #pragma unroll
        for (int s = 0; s < NKS; ++s) {
          if constexpr (QJL) {
            if (s < QKS) qjl_step(s);
          }
          // the code may straddle words wi and wi + 1; for the last word the
          // next row (the following block of the stage) supplies bits that the mask drops
          const int wi = static_cast<int>(cpos[s] >> 8), sh = static_cast<int>(cpos[s] & 31u);
          const uint2 lo = *reinterpret_cast<const uint2*>(bk + wi * KW);
          const uint2 hi = *reinterpret_cast<const uint2*>(bk + (wi + 1) * KW);
          const uint32_t cm = (1u << C) - 1u;
          uint4 eA, eB;
          if constexpr (Cfg::SR) {
            // n_hat of the quadrant (fp32) times the signed norm pair, split into
            // bf16 hi + lo. Byte offsets straight from the unmasked code:
            // direction (m_xi, m_eta) = bits [0, 2B) at 16 REP bytes an entry;
            // (s_x, s_y, i_rho) = bits [2B, 3B + 1) at 8 REP_SR bytes.
            static_assert(REP * 16 == 128 && Cfg::REP_SR * 8 == 128, "entry strides of the split tables");
            // c7 = code << 7 (low seven bits: neighbouring data)
            const uint32_t c7A = __funnelshift_r(lo.x, hi.x, sh), c7B = __funnelshift_r(lo.y, hi.y, sh);
            constexpr uint32_t DMB = ((1u << (2 * B)) - 1u) << 7, SMB = ((1u << (B + 1)) - 1u) << 7;
            const unsigned char* tb = reinterpret_cast<const unsigned char*>(table);
            const unsigned char* sb = tb + 16 * NE * REP;
            const uint4 nA = *reinterpret_cast<const uint4*>(tb + ((c7A & DMB) | rep16));
            const uint4 nB = *reinterpret_cast<const uint4*>(tb + ((c7B & DMB) | rep16));
            const float2 rA = *reinterpret_cast<const float2*>(sb + (((c7A >> (2 * B)) & SMB) | sr8));
            const float2 rB = *reinterpret_cast<const float2*>(sb + (((c7B >> (2 * B)) & SMB) | sr8));
            // x, y take the signed norms, z takes |rho|
#if OCTO_DECODE_F32X2
            const float2 xyA = mul_f32x2(make_float2(__uint_as_float(nA.x), __uint_as_float(nA.y)), rA);
            const float2 xyB = mul_f32x2(make_float2(__uint_as_float(nB.x), __uint_as_float(nB.y)), rB);
            split_bf16x2_v(xyA, eA.x, eA.z);
            split_bf16x2_v(xyB, eB.x, eB.z);
#else
            const float xA = __uint_as_float(nA.x) * rA.x, yA = __uint_as_float(nA.y) * rA.y;
            const float xB = __uint_as_float(nB.x) * rB.x, yB = __uint_as_float(nB.y) * rB.y;
            split_bf16x2(xA, yA, eA.x, eA.z);
            split_bf16x2(xB, yB, eB.x, eB.z);
#endif
            const float zA = __uint_as_float(nA.z) * fabsf(rA.x);
            const float zB = __uint_as_float(nB.z) * fabsf(rB.x);
            split_bf16_z0(zA, eA.y, eA.w);
            split_bf16_z0(zB, eB.y, eB.w);
          } else if constexpr (Cfg::FULL) {
            // the pre-shifted code is the entry's byte offset (128 bytes an entry)
            static_assert(REP * 16 == 128, "entry stride of the full table");
            constexpr uint32_t FMB = ((1u << C) - 1u) << 7;
            const uint32_t c7A = __funnelshift_r(lo.x, hi.x, sh), c7B = __funnelshift_r(lo.y, hi.y, sh);
            const unsigned char* tb = reinterpret_cast<const unsigned char*>(table);
            eA = *reinterpret_cast<const uint4*>(tb + ((c7A & FMB) | rep16));
            eB = *reinterpret_cast<const uint4*>(tb + ((c7B & FMB) | rep16));
          } else {
            const uint32_t cA = __funnelshift_r(lo.x, hi.x, sh) & cm, cB = __funnelshift_r(lo.y, hi.y, sh) & cm;
            eA = table[quadrant_index<B>(cA) * REP + rep_off];
            eB = table[quadrant_index<B>(cB) * REP + rep_off];
            // the direction signs flip x and y of the hi and lo halves
            const uint32_t sA = quadrant_signs<B>(cA), sB = quadrant_signs<B>(cB);
            eA.x ^= sA; eA.z ^= sA;
            eB.x ^= sB; eB.z ^= sB;
          }
          if constexpr (HL) {
            mma_bf16_16816(acc[0], eA.x, eB.x, eA.y, eB.y, bq[s][0], bq[s][1]);
            mma_bf16_16816(acc[1], eA.z, eB.z, eA.w, eB.w, bq[s][0], bq[s][1]);
          } else {
            mma_bf16_16816(acc[0], eA.x, eB.x, eA.y, eB.y, bq[s][0], bq[s][1]);
            mma_bf16_16816(acc[1], eA.x, eB.x, eA.y, eB.y, bq[s][NB - 2], bq[s][NB - 1]);
            mma_bf16_16816(acc[NC - 1], eA.z, eB.z, eA.w, eB.w, bq[s][0], bq[s][1]);
          }
        }
        float v[4];
  #pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[i] = acc[0][i] + acc[1][i];
          if constexpr (!HL) v[i] += acc[NC - 1][i];
        }
        if constexpr (QJL) {
  #pragma unroll
          for (int ks = NKS; ks < QKS; ++ks) qjl_step(ks);  // sketch k-steps beyond the logit ones
          const float kq = 1.2533141373155003f / static_cast<float>(D);  // sqrt(pi/2)/m, m = d
          const uint2 nu = *reinterpret_cast<const uint2*>(
              reinterpret_cast<const uint32_t*>(st + Cfg::ST_N) + cw * KW + 2 * g8);
          const float fA = kq * __uint_as_float(nu.x), fB = kq * __uint_as_float(nu.y);
          // sum_m v_m (2 b_m - 1) = 2 (256 hi-product + lo-product) - sum_m v_m,
          // times scale_r; in the HL layout lanes c4 < 2 hold the hi products and
          // c4 >= 2 the lo ones, added by the column shuffle below (the row
          // constant goes with the hi lanes)
          float sq[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float qs = (i & 1) ? qsum1 : qsum0;
            if constexpr (HL)
              sq[i] = c4 < 2 ? fmaf(512.0f, static_cast<float>(accq[0][i]), -qs) : 2.0f * static_cast<float>(accq[0][i]);
            else
              sq[i] = fmaf(512.0f, static_cast<float>(accq[0][i]), fmaf(2.0f, static_cast<float>(accq[HL ? 0 : 1][i]), -qs));
          }
          v[0] = fmaf(fA * qscale0, sq[0], v[0]); v[1] = fmaf(fA * qscale1, sq[1], v[1]);
          v[2] = fmaf(fB * qscale0, sq[2], v[2]); v[3] = fmaf(fB * qscale1, sq[3], v[3]);
        }
        if constexpr (HL) {
  #pragma unroll
          for (int i = 0; i < 4; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], 2);  // hi column + lo column
        }
        const uint2 g2 = *reinterpret_cast<const uint2*>(
            reinterpret_cast<const uint32_t*>(st + Cfg::ST_G) + cw * KW + 2 * g8);
        const float gA = __uint_as_float(g2.x), gB = __uint_as_float(g2.y);
        lgv[0] = v[0] * gA; lgv[1] = v[1] * gA;
        lgv[2] = v[2] * gB; lgv[3] = v[3] * gB;
      }

      const int64_t kown = s0 + 2 * g8;  // lgv[2h + qq] is key kown + h
      if (a.logits != nullptr && owner) {
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t key = kown + h;
          if (key >= k_end) continue;
  #pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            const int r = q0 + qq;
            if (r < a.Gq) {
              const int gi = r / a.Lq, lq = r - gi * a.Lq;
              const int64_t row = (static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq;
              a.logits[row * a.kv_len + key] = lgv[2 * h + qq];
            }
          }
        }
      }
      if (with_v) {
        // online softmax over the chunk, base 2, per query column; keys live on the g8 lanes
        const bool vA = kown < k_end, vB = kown + 1 < k_end;
        lgv[0] = vA ? lgv[0] * a.scale_log2 : -INFINITY;
        lgv[1] = vA ? lgv[1] * a.scale_log2 : -INFINITY;
        lgv[2] = vB ? lgv[2] * a.scale_log2 : -INFINITY;
        lgv[3] = vB ? lgv[3] * a.scale_log2 : -INFINITY;
        // The reference maximum m of a column only has to bound its logits
        // loosely (softmax does not depend on it): it is raised to the
        // chunk's maximum, with a rescale of l and O, only when some logit
        // exceeds it by more than kSlack (so every p = 2^(s - m) <= 2^kSlack).
        // Most chunks then skip the cross-lane reduction. The first chunk
        // always raises it (m = -inf), and it has a valid key on lanes g8 = 0.
        constexpr float kSlack = 8.0f;
        float mx0 = fmaxf(lgv[0], lgv[2]), mx1 = fmaxf(lgv[1], lgv[3]);
        if (__any_sync(0xffffffffu, mx0 > m0 + kSlack || mx1 > m1 + kSlack)) {
  #pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
          }
          const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
          const float al0 = fast_exp2(m0 - n0), al1 = fast_exp2(m1 - n1);  // m = -inf -> 0
          m0 = n0; m1 = n1;
          l0 *= al0; l1 *= al1;
  #pragma unroll
          for (int t = 0; t < MT; ++t) {
            acc_o[t][0] *= al0; acc_o[t][1] *= al1; acc_o[t][2] *= al0; acc_o[t][3] *= al1;
          }
        }
        lgv[0] = fast_exp2(lgv[0] - m0); lgv[2] = fast_exp2(lgv[2] - m0);
        lgv[1] = fast_exp2(lgv[1] - m1); lgv[3] = fast_exp2(lgv[3] - m1);
        l0 += lgv[0] + lgv[2];
        l1 += lgv[1] + lgv[3];
        // P rows (query-major) for the P.V B fragments: this lane's 2 consecutive keys
        if (owner) {
          if (q0 < G) *reinterpret_cast<float2*>(pw + q0 * PS + 2 * g8) = make_float2(lgv[0], lgv[2]);
          if (q1 < G) *reinterpret_cast<float2*>(pw + q1 * PS + 2 * g8) = make_float2(lgv[1], lgv[3]);
        }
        __syncwarp();

        // P.V over the chunk (O^T = V^T P^T: d as M, keys as K)
        uint32_t b0 = 0, b1 = 0, b2 = 0, b3 = 0;  // (hi | lo) of keys 2c4, 2c4+1 and 2c4+8, 2c4+9
        if (brow < G) {
          const float* prow = pw + brow * PS + 2 * c4;
          const float2 p01 = *reinterpret_cast<const float2*>(prow);
          const float2 p89 = *reinterpret_cast<const float2*>(prow + 8);
          uint32_t h01, l01, h89, l89;
          split_bf16x2(p01.x, p01.y, h01, l01);
          split_bf16x2(p89.x, p89.y, h89, l89);
          if constexpr (HL) {
            b0 = blo ? l01 : h01; b1 = blo ? l89 : h89;
          } else {
            b0 = h01; b1 = h89; b2 = l01; b3 = l89;
          }
        }
        // A fragments of V^T by transposed matrix loads from the swizzled
        // box: d-tile t (16 dims) x the chunk's 16 keys. Lane L addresses key
        // (L & 7) + 8 (L >> 4) at 16-byte unit 2t + ((L >> 3) & 1) of the
        // row, which the swizzle keeps at unit ^ (key & 7) (this warp's rows
        // start at a multiple of 8); units 8.. are the second 64-dim box.
        const int vkey = (lane & 7) + ((lane >> 4) << 3);
        const unsigned char* vrow = st + Cfg::ST_V + (cw * KW + vkey) * 128;
  #pragma unroll
        for (int t = 0; t < MT; ++t) {
          const int unit = 2 * t + ((lane >> 3) & 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4_trans(a0, a1, a2, a3, vrow + (unit >> 3) * Cfg::VHALF + (((unit & 7) ^ (vkey & 7)) << 4));
          mma_bf16_16816(acc_o[t], a0, a1, a2, a3, b0, b1);
          if constexpr (!HL) mma_bf16_16816(acc_o[t], a0, a1, a2, a3, b2, b3);
        }
      }
      }
      // this warp is done with the stage: release it to the producer
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  if (aborted && lane == 0) {
    atomicOr(a.status, OCTO_DEVICE_TIMEOUT);
    s_abort = 1;
  }
  __syncthreads();  // every stage is free: no copy is in flight after the last round
  if (s_abort || !with_v) return;

  // ------------------------------------------------ epilogue: merge warps (in the stage memory)
  if constexpr (HL) {  // hi column + lo column of every output
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc_o[t][i] += __shfl_xor_sync(0xffffffffu, acc_o[t][i], 2);
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  auto wbase = [&](int w) { return reinterpret_cast<float*>(base + Cfg::SREG) + w * G * (D + 2); };
  if (!producer && owner) {
    float* wm = wbase(warp);  // [G] m, [G] l, [G][D] O
    if (g8 == 0) {
      if (q0 < G) { wm[q0] = m0; wm[G + q0] = l0; }
      if (q1 < G) { wm[q1] = m1; wm[G + q1] = l1; }
    }
    float* o = wm + 2 * G;
#pragma unroll
    for (int t = 0; t < MT; ++t) {  // rows g8 and g8 + 8 of d-tile t
      const int d0 = 16 * t + g8;
      if (q0 < G) { o[q0 * D + d0] = acc_o[t][0]; o[q0 * D + d0 + 8] = acc_o[t][2]; }
      if (q1 < G) { o[q1 * D + d0] = acc_o[t][1]; o[q1 * D + d0 + 8] = acc_o[t][3]; }
    }
  }
  __syncthreads();

  const int S = n_sl, SW = a.n_splits;  // this head's slices; partial slots per head
  float* pm = a.part_m + (static_cast<int64_t>(bh) * SW + split) * G;
  float* pl = a.part_l + (static_cast<int64_t>(bh) * SW + split) * G;
  float* po = a.part_o + (static_cast<int64_t>(bh) * SW + split) * G * D;
  for (int j = tid; j < G * D; j += Cfg::THREADS) {
    const int r = j / D, d = j - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) M = fmaxf(M, wbase(w)[r]);
    float o = 0.0f, l = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NWARP; ++w) {
        const float f = fast_exp2(wbase(w)[r] - M);
        o = fmaf(f, wbase(w)[2 * G + r * D + d], o);
        l = fmaf(f, wbase(w)[G + r], l);
      }
    }
    if (S == 1) {
      if (r < a.Gq) {
        const int gi = r / a.Lq, lq = r - gi * a.Lq;
        const int64_t row = (static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq;
        a.out[row * D + d] = l > 0.0f ? o / l : 0.0f;
      }
    } else {
      po[j] = o;
      if (d == 0) { pm[r] = M; pl[r] = l; }
    }
  }
  if (S == 1) return;

  // ------------------------------------------------ epilogue: merge splits (last CTA of this head)
  __syncthreads();
  if (tid == 0) {
    int ticket;
    asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(ticket) : "l"(a.counters + bh) : "memory");
    s_last = ticket == S - 1;
  }
  __syncthreads();
  if (!s_last) return;
  const float* bm = a.part_m + static_cast<int64_t>(bh) * SW * G;
  const float* bl = a.part_l + static_cast<int64_t>(bh) * SW * G;
  const float* bo = a.part_o + static_cast<int64_t>(bh) * SW * G * D;
  if (S <= 32) {
    // Up to 32 splits (the usual case), one L2 round trip: every thread
    // issues the partial-O loads of its (at most) two outputs; meanwhile
    // warp r forms row r's split weights w_s = 2^(m_s - M) / L in shared
    // memory (lane s = split s), then the outputs are the weighted sums.
    float* wsm = reinterpret_cast<float*>(base + Cfg::SREG);  // [G][32] weights (the stages are free)
    for (int j0 = 0; j0 < a.Gq * D; j0 += 2 * Cfg::THREADS) {
      float ov[2][32];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int j = j0 + tid + k * Cfg::THREADS;
        const int r = j < a.Gq * D ? j / D : 0, d = j - r * D;
#pragma unroll
        for (int s2 = 0; s2 < 32; ++s2)
          ov[k][s2] = (j < a.Gq * D && s2 < S) ? __ldcg(bo + (static_cast<int64_t>(s2) * G + r) * D + d) : 0.0f;
      }
      if (j0 == 0) {
        if (warp < a.Gq) {
          const float m = lane < S ? __ldcg(bm + lane * G + warp) : -INFINITY;
          const float l = lane < S ? __ldcg(bl + lane * G + warp) : 0.0f;
          float M = m;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
          const float f = M == -INFINITY || m == -INFINITY ? 0.0f : fast_exp2(m - M);
          float L = f * l;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
          wsm[warp * 32 + lane] = L > 0.0f ? f / L : 0.0f;
        }
        __syncthreads();
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int j = j0 + tid + k * Cfg::THREADS;
        if (j >= a.Gq * D) continue;
        const int r = j / D, d = j - r * D;
        float o = 0.0f;
#pragma unroll
        for (int s2 = 0; s2 < 32; ++s2) o = fmaf(wsm[r * 32 + s2], ov[k][s2], o);
        const int gi = r / a.Lq, lq = r - gi * a.Lq;
        const int64_t row = (static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq;
        a.out[row * D + d] = o;
      }
    }
    if (tid == 0) atomicExch(a.counters + bh, 0);  // ready for the next call
    return;
  }
  // Each thread merges its (row, column) outputs over the S split partials,
  // 32 splits per round of independent loads (one L2 round trip per round).
  for (int j = tid; j < a.Gq * D; j += Cfg::THREADS) {
    const int r = j / D, d = j - r * D;
    float M = -INFINITY, o = 0.0f, l = 0.0f;
    for (int sb = 0; sb < S; sb += 32) {
      float mv[32], lv[32], ov[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int s2 = sb + k;
        const bool ok = s2 < S;
        mv[k] = ok ? __ldcg(bm + s2 * G + r) : -INFINITY;
        lv[k] = ok ? __ldcg(bl + s2 * G + r) : 0.0f;
        ov[k] = ok ? __ldcg(bo + (static_cast<int64_t>(s2) * G + r) * D + d) : 0.0f;
      }
      float Mb = M;
#pragma unroll
      for (int k = 0; k < 32; ++k) Mb = fmaxf(Mb, mv[k]);
      if (Mb == -INFINITY) continue;
      const float sc = fast_exp2(M - Mb);  // rescale the rounds merged so far
      o *= sc;
      l *= sc;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float f = fast_exp2(mv[k] - Mb);
        o = fmaf(f, ov[k], o);
        l = fmaf(f, lv[k], l);
      }
      M = Mb;
    }
    const int gi = r / a.Lq, lq = r - gi * a.Lq;
    const int64_t row = (static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq;
    a.out[row * D + d] = l > 0.0f ? o / l : 0.0f;
  }
  if (tid == 0) atomicExch(a.counters + bh, 0);  // ready for the next call
}

// OCTOPUS-QJL query preparation for the tensor-core kernel, one block per
// KV head: the rotated query rows q_rot_r = (1/sqrt(d)) H (s_h * q_r) (zero
// rows past the group, zero pad to QROW) and p_r = S q_rot_r, written as the
// decode CTAs' query scratch image. Every CTA of the head then copies the
// image with its first round instead of reading the head's d x d sketch
// matrix itself.
template <int D, int G>
__global__ void __launch_bounds__(256) decode_prep_kernel(DecodeArgs a) {
  using Cfg = TcCfg<D, 2, G, true>;  // the scratch layout does not depend on b
  constexpr int QROW = static_cast<int>(Cfg::QROW), E = D / 32;
  static_assert(G <= 8, "one warp per query row");
  __shared__ __align__(16) float q[G][QROW];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x;
  const int bidx = bh / a.Hkv, hkv = bh - bidx * a.Hkv;
  const int64_t trow = bh % a.table_heads;
  float* out = a.prep + bh * a.prep_stride;
  // warp w takes rows m = w + 8 i of S; all of its loads are issued first
  // (S does not depend on the query), so they overlap the rotation below
  constexpr int RPW = D / 8;
  const float* S = a.qjl_S + trow * D * D;
  float sv[RPW][E];
#pragma unroll
  for (int i = 0; i < RPW; ++i)
#pragma unroll
    for (int e = 0; e < E; ++e) sv[i][e] = __ldg(S + static_cast<int64_t>(warp + 8 * i) * D + lane + 32 * e);
  if (warp < G) {
    float v[E];
    if (warp < a.Gq) {
      const int gi = warp / a.Lq, lq = warp - gi * a.Lq;
      const int64_t qoff = ((static_cast<int64_t>(bidx) * a.Hq + hkv * a.g + gi) * a.Lq + lq) * D + lane * E;
      const float* sg = a.signs + trow * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float x = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[qoff + e])
                                 : static_cast<const float*>(a.q)[qoff + e];
        v[e] = x * __ldg(sg + e);
      }
      fwht_warp<E>(v, lane);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = 0.0f;
    }
    const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
#pragma unroll
    for (int e = 0; e < E; ++e) q[warp][lane * E + e] = v[e] * inv_sqrt_d;
    for (int c = D + lane; c < QROW; c += 32) q[warp][c] = 0.0f;
  }
  __syncthreads();
  for (int j = tid; j < G * QROW; j += blockDim.x) out[j] = q[j / QROW][j % QROW];
  // p: a lane sums D/32 terms of each row, the warp reduces
  float* p = out + G * QROW;
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
#pragma unroll
    for (int r = 0; r < G; ++r) {
      float acc = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) acc = fmaf(sv[i][e], q[r][lane + 32 * e], acc);
      acc = warp_sum(acc);
      if (lane == 0) p[r * D + warp + 8 * i] = acc;
    }
  }
}

// Launch one decode instantiation for head dimension D (defined in the
// per-D translation units so that the templates compile in parallel).
cudaError_t launch_decode_d64(const DecodeArgs& a, const TmaDesc& tm, int b, int G, bool qjl, dim3 grid, cudaStream_t st);
cudaError_t launch_decode_d128(const DecodeArgs& a, const TmaDesc& tm, int b, int G, bool qjl, dim3 grid, cudaStream_t st);
cudaError_t launch_decode_d256(const DecodeArgs& a, const TmaDesc& tm, int b, int G, bool qjl, dim3 grid, cudaStream_t st);

#ifndef OCTO_DECODE_TC
#define OCTO_DECODE_TC 1  // tensor-core logits where the shape allows
#endif

// The tensor-core kernel takes d <= 128 (b <= 4),
// and only shapes whose tables and slots fit in shared memory.
template <int D, int B, int G, bool QJL>
constexpr bool tc_fits() {
  if constexpr (D <= 128 && B <= 4) return TcCfg<D, B, G, QJL>::FITS;
  else return false;
}

template <int D, int B, int G, bool QJL>
cudaError_t launch_decode_one(const DecodeArgs& a, const TmaDesc& tm, dim3 grid, cudaStream_t st) {
  if constexpr (OCTO_DECODE_TC && tc_fits<D, B, G, QJL>()) {
    using Cfg = TcCfg<D, B, G, QJL>;
    auto k = decode_tc_kernel<D, B, G, QJL>;
    static LaunchCache cache;
    int resident = 0;
    const cudaError_t e = launch_setup(k, cache, Cfg::THREADS, Cfg::SMEM, resident);
    if (e != cudaSuccess) return e;
    if constexpr (QJL) decode_prep_kernel<D, G><<<grid.y, 256, 0, st>>>(a);  // one block (8 warps) per head
    k<<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(a, tm);  // grid: (splits, heads)
  } else {
    using Cfg = DecCfg<D, B, G, QJL>;
    auto k = decode_kernel<D, B, G, QJL>;
    static LaunchCache cache;
    int resident = 0;
    const cudaError_t e = launch_setup(k, cache, Cfg::THREADS, Cfg::SMEM, resident);
    if (e != cudaSuccess) return e;
    k<<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(a);  // grid: (splits, heads)
  }
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_d(const DecodeArgs& a, const TmaDesc& tm, int b, int G, bool qjl, dim3 grid, cudaStream_t st) {
#define OCTO_G(BB)                                                                           \
  switch (G) {                                                                               \
    case 1: return qjl ? launch_decode_one<D, BB, 1, true>(a, tm, grid, st)                      \
                       : launch_decode_one<D, BB, 1, false>(a, tm, grid, st);                    \
    case 4: return qjl ? launch_decode_one<D, BB, 4, true>(a, tm, grid, st)                      \
                       : launch_decode_one<D, BB, 4, false>(a, tm, grid, st);                    \
    default: return qjl ? launch_decode_one<D, BB, 8, true>(a, tm, grid, st)                     \
                        : launch_decode_one<D, BB, 8, false>(a, tm, grid, st);                   \
  }
  switch (b) {
    case 2: OCTO_G(2)
    case 3: OCTO_G(3)
    default: OCTO_G(4)
  }
#undef OCTO_G
}

}  // namespace octo
