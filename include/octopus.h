/*
 * octopus.h - C ABI of the OCTOPUS KV-cache codec for NVIDIA B200 (sm_100a).
 *
 * OCTOPUS (the paper "OCTOPUS: Optimized KV Cache for Transformers via
 * Octahedral Parametrization Under optimal Squared error quantization",
 * abstract; method as described in the youleyou.com explainer, sections
 * "triplet decomposition", "octahedral folding", "non-uniform bit allocation",
 * "joint rounding", "optional residual correction", "engineering
 * implementation") stores each key k as its norm gamma = ||k|| (fp32) and a
 * bit-packed code of its unit direction: the direction is rotated by a
 * seeded sign-flipped Walsh-Hadamard transform, cut into coordinate
 * triplets, and each triplet's norm rho and octahedrally mapped direction
 * (xi, eta) are Lloyd-Max quantised with (b-1, b+1, b+1) bits.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Return value: OCTO_OK (0) or a negative OCTO_E* status; nothing aborts,
 *    no C++ exception crosses this boundary. octo_status_string() names it.
 *  - The caller owns every buffer. The library allocates and frees no
 *    memory and keeps no data between calls. The one exception is
 *    octo_decode_attn_static's fixed scratch array. Each kernel's launch
 *    set-up (shared-memory opt-in, blocks resident per SM, SM count) is
 *    looked up on its first call on a device and reused.
 *  - "device" pointers are CUDA global-memory addresses of the current
 *    device; "host" pointers are ordinary process memory.
 *  - Device entry points are asynchronous on the given stream; they return
 *    after the launch (OCTO_ECUDA if the launch itself failed). Arguments
 *    are validated on the host before anything is launched; an invalid
 *    argument returns OCTO_EINVAL and launches nothing.
 *  - Sizes are element counts unless stated otherwise.
 *
 * Supported shapes: head dimension d in {64, 128, 256}; bit budget
 * b in {2, 3, 4}; query rows per KV head (GQA group x query tokens) <= 8.
 *
 * Cache layout in device memory (word-planar, token-contiguous):
 *   packed   uint32 [n_heads][W][cache_cap]       W = ceil(T (3b+1) / 32)
 *   gamma    float  [n_heads][cache_cap]
 *   qjl_bits uint32 [n_heads][d/32][cache_cap]    (OCTOPUS-QJL only)
 *   qjl_norm float  [n_heads][cache_cap]          (OCTOPUS-QJL only)
 * Word w of token n's bit stream is packed[h][w][n]. Within the stream,
 * the (3b+1)-bit code of triplet i starts at bit i(3b+1), LSB first (bit p
 * of the stream is bit p mod 32 of word p / 32); a code is
 *   m_xi | m_eta << b | s_xi << 2b | s_eta << (2b+1) | i_rho << 2(b+1),
 * where a direction cell index i in [0, 2^(b+1)) of the odd-symmetric
 * codebook is stored as a sign s (1 for the lower half, i < 2^b) and the
 * rank m of |level| among the positive levels (m = i - 2^b above the
 * middle, 2^b - 1 - i below).
 */
#ifndef OCTOPUS_B200_H
#define OCTOPUS_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define OCTO_API __attribute__((visibility("default")))
#else
#define OCTO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* CUDA stream handle (cudaStream_t); 0 is the legacy default stream. */
typedef void* octo_stream_t;

enum octo_status {
  OCTO_OK = 0,
  OCTO_EINVAL = -1,       /* bad argument: null pointer, size, stride, alignment, range */
  OCTO_EUNSUPPORTED = -2, /* valid but not built: d, b or query rows outside the supported set */
  OCTO_ECUDA = -3,        /* a CUDA launch or runtime call failed */
  OCTO_EWORKSPACE = -4    /* workspace smaller than octo_decode_attn_workspace() */
};

enum octo_rounding {
  OCTO_ROUND_SCALAR = 0, /* each of xi, eta, rho to its nearest centroid */
  OCTO_ROUND_JOINT = 1   /* 3x3 joint search ("joint rounding" section); the default */
};

enum octo_dtype { OCTO_F32 = 0, OCTO_BF16 = 1 };

/* Sizes that follow from (d, b). Filled by octo_layout_init. */
typedef struct octo_layout {
  int32_t d;          /* key / head dimension */
  int32_t b;          /* bit budget per coordinate */
  int32_t T;          /* triplets per key, ceil(d/3); the last one is zero-padded if 3 does not divide d */
  int32_t b_dir;      /* bits of xi and of eta: b+1 */
  int32_t b_rho;      /* bits of rho: b-1 */
  int32_t code_bits;  /* bits per triplet: 3b+1 */
  int32_t words;      /* W, 32-bit words per key */
  int32_t n_dir;      /* direction codebook levels, 2^(b+1) */
  int32_t n_rho;      /* norm codebook levels, 2^(b-1) */
  int32_t qjl;        /* 1: keep the OCTOPUS-QJL residual sign sketch (d bits + fp32 norm) */
  int32_t qjl_words;  /* d/32 when qjl, else 0 */
  int32_t rounding;   /* enum octo_rounding */
} octo_layout;

/* Device pointers to the data-independent tables (built by the host
 * functions below, copied to the device by the caller). A cache head h
 * uses table row (h mod n_heads): with caches laid out [batch][kv_head],
 * n_heads = number of KV heads shares one rotation across the batch. */
typedef struct octo_tables {
  const float* dir_c;  /* [n_dir]     direction centroids, increasing */
  const float* dir_t;  /* [n_dir-1]   direction thresholds (cell k = #thresholds <= x) */
  const float* rho_c;  /* [n_rho]     norm centroids, increasing */
  const float* rho_t;  /* [n_rho-1]   norm thresholds */
  const float* signs;  /* [n_heads][d] +1/-1 diagonal of the sign-flipped WHT */
  const float* qjl_S;  /* [n_heads][d][d] row-major Gaussian projection, 16-byte aligned; NULL unless layout.qjl */
  int64_t n_heads;     /* rows in signs / qjl_S, >= 1 */
} octo_tables;

/* Fills *L for head dimension d, bit budget b, QJL flag and rounding mode
 * (explainer, "non-uniform bit allocation": b+1 bits for each direction
 * coordinate, b-1 for the triplet norm). Returns OCTO_EUNSUPPORTED for d or
 * b outside the supported set, OCTO_EINVAL for a NULL L or a bad flag. */
OCTO_API int octo_layout_init(octo_layout* L, int d, int b, int qjl, int rounding);

/* Fills *L for another split of the bit budget (explainer, "non-uniform bit
 * allocation": each direction coordinate gets b + delta bits and the triplet
 * norm b - delta; the OCTOPUS allocation is delta = +1, which
 * octo_layout_init uses). code_bits = 3b + delta. Supported: b in {2, 3, 4}
 * with 2 <= b + delta <= 5 and 1 <= b - delta <= 5 for octo_codebook_build;
 * octo_encode and octo_dequant run delta = +1 for every d and, at d = 128
 * without the sketch, also b = 3 with delta in {-1, 0, +2} and b = 4 with
 * delta in {-1, 0} (the sweep the explainer reports); octo_decode_attn runs
 * delta = +1 only. Other combinations return OCTO_EUNSUPPORTED from the call
 * that cannot run them; qjl with delta != +1 returns OCTO_EUNSUPPORTED here.
 * Errors as octo_layout_init. */
OCTO_API int octo_layout_init_delta(octo_layout* L, int d, int b, int delta, int qjl, int rounding);

/* Host. Lloyd-Max codebooks for layout L (explainer, "triplet
 * decomposition": Lloyd-Max quantisers designed for the marginal law; the
 * abstract: "implementation-matched marginals", data-oblivious). The
 * direction codebook is designed for the marginal of the octahedral map of
 * a uniform direction on the sphere (shared by xi and eta); the norm
 * codebook for the law of the norm of three coordinates of a uniform unit
 * vector in R^d. Outputs are caller-allocated host arrays of n_dir,
 * n_dir-1, n_rho, n_rho-1 floats. Thresholds are the midpoints of adjacent
 * centroids. Deterministic; takes about a second for b = 4. */
OCTO_API int octo_codebook_build(const octo_layout* L, float* dir_c, float* dir_t, float* rho_c, float* rho_t);

/* Host. Rotation signs for n_heads heads of dimension d into the
 * caller-allocated host array signs[n_heads][d] (explainer, "rotation":
 * sign-flipped Walsh-Hadamard transform; abstract: deterministic given a
 * seed). signs[h][j] = -1 if the top bit of SplitMix64 output number
 * h*d + j + 1 (generator seeded with `seed`) is set, else +1. */
OCTO_API int octo_rotation_build(uint64_t seed, int d, int64_t n_heads, float* signs);

/* Host. OCTOPUS-QJL projections S[n_heads][d][d] (caller-allocated host
 * array; explainer, "optional residual correction"). Entry
 * e = (h*d + i)*d + j is the float32 rounding of the Box-Muller normal
 * sqrt(-2 ln u1) cos(2 pi u2), u1 = ((z1 >> 11) + 1) 2^-53,
 * u2 = (z2 >> 11) 2^-53, z1, z2 = SplitMix64 outputs 2e+1 and 2e+2. */
OCTO_API int octo_qjl_build(uint64_t seed, int d, int64_t n_heads, float* S);

/* Device. Encodes n_tokens keys of each of n_heads heads into the cache at
 * token positions [token_offset, token_offset + n_tokens) (explainer,
 * "triplet decomposition" steps 1-4 and "joint rounding"; with layout.qjl
 * also the residual sketch of "optional residual correction").
 *   keys        device, element (h, n, j) at keys[h*head_stride + n*token_stride + j];
 *               key_dtype OCTO_F32 or OCTO_BF16; j is contiguous. Each lane
 *               of a warp loads d/32 consecutive elements at once, so the
 *               base address and both strides (in bytes) must be multiples
 *               of min(16, (d/32) * element size).
 *   cache_cap   tokens per head in the cache arrays (see layout above).
 *   packed, gamma               device, required.
 *   qjl_bits, qjl_norm          device, required iff layout.qjl, else ignored.
 * Errors: OCTO_EINVAL if a pointer is NULL, n_heads < 0, n_tokens < 0,
 * token_offset < 0, token_offset + n_tokens > cache_cap, or a key is
 * misaligned. n_tokens == 0 or n_heads == 0 launches nothing. */
OCTO_API int octo_encode(const octo_layout* L, const octo_tables* tables,
                const void* keys, int key_dtype,
                int64_t n_heads, int64_t n_tokens, int64_t head_stride, int64_t token_stride,
                int64_t cache_cap, int64_t token_offset,
                uint32_t* packed, float* gamma, uint32_t* qjl_bits, float* qjl_norm,
                octo_stream_t stream);

/* Bytes of device workspace octo_decode_attn needs for these sizes (at
 * least 256: the workspace also carries a status word). Returns 0 for
 * unsupported arguments. */
OCTO_API size_t octo_decode_attn_workspace(const octo_layout* L, int B, int Hq, int Hkv, int Lq, int64_t kv_len);

/* Device. One fused decode-attention step over a compressed cache
 * (explainer, "engineering implementation"; abstract: keys are
 * reconstructed on the fly and never materialised). The queries are
 * rotated once by the same transform as the keys, so the raw logit of key n
 * is gamma_n * sum_i rho_hat_i (q_rot_i . n_hat_i) (+ the QJL term
 * gamma_n * nu_n * sqrt(pi/2)/d * <S q_rot, 2 bits_n - 1> when layout.qjl);
 * then softmax(scale * logits) and the product with bf16 V, all on chip.
 *   q        device, [B][Hq][Lq][d], q_dtype OCTO_F32 or OCTO_BF16, contiguous.
 *   Hq = g*Hkv; query head hq reads KV head hq / g. Cache head index is
 *   b*Hkv + h_kv in packed / gamma / qjl_* / V.
 *   packed, gamma, qjl_bits, qjl_norm: the cache (layout above), capacity
 *   cache_cap, the first kv_len tokens are attended. The code rows are
 *   staged into shared memory by 16-byte bulk copies, so cache_cap must be
 *   a multiple of 4 and these four base addresses 16-byte aligned.
 *   V        device bf16 [B*Hkv][cache_cap][d] (16-byte aligned), or NULL
 *            for logits only.
 *   scale    softmax temperature (1/sqrt(d) for standard attention).
 *   out      device fp32 [B][Hq][Lq][d]; required iff V != NULL.
 *   logits   device fp32 [B][Hq][Lq][kv_len] raw (unscaled) logits, or NULL.
 *   workspace device, >= octo_decode_attn_workspace() bytes, 256-byte
 *            aligned, always required. Bytes [0, 4) are a status word: the
 *            kernel ORs in 1 if one of its bounded on-chip waits expired
 *            (the outputs of that call are then invalid). Bytes [256, 256 +
 *            4*B*Hkv) are arrival counters. Status and counters must be zero
 *            before the first call (zero the whole workspace once); every
 *            completed call leaves the counters zero again. The rest is
 *            the call's scratch (per-slice partial results; with
 *            layout.qjl and d <= 128 also the rotated queries and S q_rot of
 *            every KV head). Calls that share a workspace must not overlap
 *            on the GPU.
 * The call launches one kernel on `stream`, two with layout.qjl and
 * d <= 128 (a per-KV-head query preparation into the workspace, then the
 * decode, which reads it).
 * kv_len == 0 gives out = 0. Errors: OCTO_EINVAL (NULL required pointer,
 * bad sizes, kv_len > cache_cap, both V and logits NULL, misalignment),
 * OCTO_EUNSUPPORTED (g*Lq > 8 or B*Hkv > 65535), OCTO_EWORKSPACE. */
OCTO_API int octo_decode_attn(const octo_layout* L, const octo_tables* tables,
                     const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq,
                     int64_t kv_len, int64_t cache_cap,
                     const uint32_t* packed, const float* gamma,
                     const uint32_t* qjl_bits, const float* qjl_norm,
                     const void* V, float scale, float* out, float* logits,
                     void* workspace, size_t ws_bytes, octo_stream_t stream);

/* Device. octo_decode_attn without a caller-provided workspace, for callers
 * that cannot allocate device memory themselves: for example a plugin whose
 * host framework owns every device allocation, or a caller whose allocator
 * cannot be reached from the code that issues the decode step. It allocates
 * nothing: the split-merge scratch is a fixed array of
 * OCTO_STATIC_SCRATCH_BYTES (8 MiB) in the library's own device memory,
 * reserved on every GPU that loads the library until the process exits.
 * (Not part of the method: the paper has no counterpart; this is a
 * deployment convenience.)
 * Arguments and results are those of octo_decode_attn, minus the workspace.
 *   - Returns OCTO_EWORKSPACE when the sizes need more scratch than
 *     OCTO_STATIC_SCRATCH_BYTES (octo_decode_attn_workspace() tells).
 *   - The first call on a device (with that device current) looks up the
 *     array's device address; make that first call outside any stream
 *     capture.
 *   - Arguments are checked exactly as octo_decode_attn checks them (same
 *     status codes, same order) before anything touches the GPU; a
 *     rejected call launches nothing and leaves the array alone.
 *   - Each accepted call zeroes the array's status word and arrival
 *     counters on `stream` before the decode kernel. All calls on a device
 *     share the array, which keeps the last call's contents: calls that
 *     overlap on the GPU (other streams, or other threads) race on it and
 *     must not be issued.
 *   - The kernel's timeout flag (bit 0 of the status word, see
 *     octo_decode_attn) lives in the array; read it with
 *     octo_decode_attn_static_status. */
#define OCTO_STATIC_SCRATCH_BYTES (8u << 20)
OCTO_API int octo_decode_attn_static(const octo_layout* L, const octo_tables* tables,
                                     const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq,
                                     int64_t kv_len, int64_t cache_cap,
                                     const uint32_t* packed, const float* gamma,
                                     const uint32_t* qjl_bits, const float* qjl_norm,
                                     const void* V, float scale, float* out, float* logits,
                                     octo_stream_t stream);

/* Host. The status word that the last octo_decode_attn_static call on the
 * current device left in the library's scratch array (bit 0 set: one of
 * the kernel's bounded on-chip waits expired, and that call's outputs are
 * invalid). Waits for the work queued on `stream` (the stream of that
 * call) to finish, then copies the word into *status. Not part of the
 * method; it serves octo_decode_attn_static's callers, who have no
 * workspace to read the word from. Errors: OCTO_EINVAL (status NULL),
 * OCTO_ECUDA. */
OCTO_API int octo_decode_attn_static_status(int* status, octo_stream_t stream);

/* Device. Fills the whole scratch array of octo_decode_attn_static on the
 * current device with the byte value `byte` & 0xff, on `stream`. A
 * diagnostic: it lets a test leave nonzero status and counter bytes behind,
 * as an interrupted call would, and check that the next call still clears
 * what must start at zero. Normal use never needs it. Same race rules as
 * octo_decode_attn_static. */
OCTO_API int octo_decode_attn_static_fill(int byte, octo_stream_t stream);

/* Device. Reconstructs keys from the cache: k_hat = gamma * R^T u_hat
 * (explainer, "triplet decomposition" steps 1-4 undone, for the codec's
 * compress-and-reconstruct use). u_hat concatenates rho_hat_i * n_hat_i over
 * the T triplets (inverse octahedral map of section "octahedral folding"),
 * padding dropped; R = (1/sqrt(d)) H diag(s_h) is the encoder's rotation, so
 * k_hat_j = gamma * s_h[j] * (H u_hat)_j / sqrt(d). The QJL sketch, if the
 * layout keeps one, is not read: it estimates inner products, it does not
 * correct keys.
 *   packed, gamma  device cache (layout above), cache_cap tokens per head;
 *                  tokens [token_offset, token_offset + n_tokens) of each of
 *                  the first n_heads cache heads are read. Cache head h uses
 *                  sign row h mod tables->n_heads.
 *   out            device [n_heads][n_tokens][d], row-major, out_dtype
 *                  OCTO_F32 or OCTO_BF16 (round to nearest even); 16-byte
 *                  aligned. Computed in fp32.
 * Errors: OCTO_EINVAL (NULL pointer, negative sizes, token_offset +
 * n_tokens > cache_cap, misaligned out, bad out_dtype), OCTO_EUNSUPPORTED
 * (d or b outside the supported set). n_heads == 0 or n_tokens == 0
 * launches nothing. */
OCTO_API int octo_dequant(const octo_layout* L, const octo_tables* tables,
                          int64_t n_heads, int64_t n_tokens, int64_t cache_cap, int64_t token_offset,
                          const uint32_t* packed, const float* gamma, void* out, int out_dtype,
                          octo_stream_t stream);

/* Static string for a status code. */
OCTO_API const char* octo_status_string(int status);

/* ABI version of this header (major*100 + minor). */
OCTO_API int octo_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OCTOPUS_B200_H */
