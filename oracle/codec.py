"""Oracle: OCTOPUS key encoding and decoding, step by step (test infrastructure only).

Follows [EXPL] "triplet decomposition" (pipeline steps 1-4), "octahedral
folding" (forward and inverse map), "non-uniform bit allocation" ((b+1, b-1)
bits) and "joint rounding" (3x3 neighbourhood, rho chosen from s = n_hat . t).
All arithmetic is float64; indices are int64.

Index layout conventions (readings where the pages leave the layout open):
* key k (length d) -> gamma = ||k||, u = k / gamma (gamma = 0 gives u = 0);
* rotated direction u_rot = (1/sqrt(d)) H (s * u), H the Sylvester-ordered
  Walsh-Hadamard matrix, s the per-head sign vector;
* u_rot zero-padded at the end to 3T, T = ceil(d/3); triplet i is
  coordinates 3i, 3i+1, 3i+2;
* per-triplet code = i_xi | i_eta << (b+1) | i_rho << 2(b+1), 3b+1 bits;
* code of triplet i sits at bit i*(3b+1) of the key's bit stream, LSB first:
  stream bit k is bit (k mod 32) of 32-bit word floor(k/32); a key has
  W = ceil(T (3b+1) / 32) words.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

SCALAR = 0
JOINT = 1


@dataclass(frozen=True)
class Layout:
    """Sizes that follow from (d, b, delta) ([EXPL] "non-uniform bit allocation":
    each direction coordinate gets b + delta bits, the triplet norm b - delta;
    OCTOPUS uses delta = +1)."""
    d: int
    b: int
    delta: int = 1

    @property
    def T(self) -> int:
        return -(-self.d // 3)

    @property
    def b_dir(self) -> int:
        return self.b + self.delta

    @property
    def b_rho(self) -> int:
        return self.b - self.delta

    @property
    def code_bits(self) -> int:
        return 2 * self.b_dir + self.b_rho

    @property
    def words(self) -> int:
        return -(-self.T * self.code_bits // 32)

    @property
    def n_dir(self) -> int:
        return 1 << self.b_dir

    @property
    def n_rho(self) -> int:
        return 1 << self.b_rho


# --------------------------------------------------------------------------
# Rotation ([EXPL] "rotation": sign-flipped Walsh-Hadamard transform).
# --------------------------------------------------------------------------
def hadamard(d: int) -> np.ndarray:
    """Sylvester Walsh-Hadamard matrix, H[i, j] = (-1)^popcount(i & j)."""
    i = np.arange(d)
    pc = np.zeros((d, d), dtype=np.int64)
    m = i[:, None] & i[None, :]
    while np.any(m):
        pc += m & 1
        m = m >> 1
    return np.where(pc % 2 == 0, 1.0, -1.0)


def rotation_matrix(signs: np.ndarray) -> np.ndarray:
    """R = (1/sqrt(d)) H diag(s) for one head's sign vector s."""
    d = signs.shape[-1]
    return hadamard(d) * signs[None, :] / math.sqrt(d)


def rotate(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """x_rot = R x for rows of x ([..., d])."""
    return np.asarray(x, dtype=np.float64) @ rotation_matrix(signs).T


# --------------------------------------------------------------------------
# Octahedral map ([EXPL] "octahedral folding").
# --------------------------------------------------------------------------
def _sgn(x):
    return np.where(x >= 0, 1.0, -1.0)


def oct_forward(n: np.ndarray):
    """(xi, eta) in [-1, 1]^2 for 3-vectors n ([..., 3]).

    Divide by l = |x|+|y|+|z|; upper hemisphere (z >= 0) keeps (px, py);
    the lower one folds its four triangles onto the square's corners:
    ((1-|py|) sgn px, (1-|px|) sgn py). sgn(0) = +1; the zero vector maps
    to (0, 0).
    """
    n = np.asarray(n, dtype=np.float64)
    l1 = np.sum(np.abs(n), axis=-1)
    safe = np.where(l1 > 0, l1, 1.0)
    px = np.where(l1 > 0, n[..., 0] / safe, 0.0)
    py = np.where(l1 > 0, n[..., 1] / safe, 0.0)
    pz = np.where(l1 > 0, n[..., 2] / safe, 1.0)
    up = pz >= 0
    xi = np.where(up, px, (1.0 - np.abs(py)) * _sgn(px))
    eta = np.where(up, py, (1.0 - np.abs(px)) * _sgn(py))
    return xi, eta


def oct_inverse(xi, eta) -> np.ndarray:
    """Unit 3-vector for (xi, eta): r = 1-|xi|-|eta|; unfold if r < 0; normalise."""
    xi = np.asarray(xi, dtype=np.float64)
    eta = np.asarray(eta, dtype=np.float64)
    r = 1.0 - np.abs(xi) - np.abs(eta)
    x = np.where(r >= 0, xi, (1.0 - np.abs(eta)) * _sgn(xi))
    y = np.where(r >= 0, eta, (1.0 - np.abs(xi)) * _sgn(eta))
    v = np.stack([x, y, r], axis=-1)
    return v / np.linalg.norm(v, axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# Triplets ([EXPL] "triplet decomposition", step 3).
# --------------------------------------------------------------------------
def triplets(u_rot: np.ndarray) -> np.ndarray:
    """[..., d] -> [..., T, 3], zero-padded at the end."""
    d = u_rot.shape[-1]
    T = -(-d // 3)
    pad = 3 * T - d
    z = np.concatenate([u_rot, np.zeros(u_rot.shape[:-1] + (pad,))], axis=-1)
    return z.reshape(u_rot.shape[:-1] + (T, 3))


# --------------------------------------------------------------------------
# Quantisation ([EXPL] "triplet decomposition" step 4, "joint rounding").
# --------------------------------------------------------------------------
def scalar_index(x, thresholds) -> np.ndarray:
    """Cell index = number of thresholds <= x (a value on a threshold goes up)."""
    return np.searchsorted(np.asarray(thresholds), np.asarray(x), side="right").astype(np.int64)


def joint_round(t, i_xi0, i_eta0, dir_c, rho_c, rho_t):
    """Joint rounding of triplets t ([..., 3]) around the scalar indices.

    [EXPL] "joint rounding": for a fixed direction candidate n_hat the best
    norm level is the one nearest s = n_hat . t (not nearest rho); only the
    3x3 neighbourhood of the scalar (i_xi, i_eta) needs to be searched.
    Each candidate's error is ||t - rho_hat n_hat||^2 = rho^2 - 2 rho_hat s
    + rho_hat^2. Order (reading): the centre candidate first, then
    (d_xi, d_eta) row-major from -1 to +1; a candidate replaces the best only
    if its error is strictly smaller; out-of-range neighbours are skipped.

    Returns (i_xi, i_eta, i_rho, err) with err the chosen squared error.
    """
    t = np.asarray(t, dtype=np.float64)
    L = len(dir_c)
    rho2 = np.sum(t * t, axis=-1)

    def cand(ix, iy):
        nh = oct_inverse(dir_c[ix], dir_c[iy])
        s = np.sum(nh * t, axis=-1)
        ir = scalar_index(s, rho_t)
        rh = rho_c[ir]
        return rho2 - 2.0 * rh * s + rh * rh, ir

    bx, by = np.asarray(i_xi0).copy(), np.asarray(i_eta0).copy()
    berr, br = cand(bx, by)
    for dx in (-1, 0, 1):
        for dy in (-1, 0, 1):
            if dx == 0 and dy == 0:
                continue
            ix = i_xi0 + dx
            iy = i_eta0 + dy
            ok = (ix >= 0) & (ix < L) & (iy >= 0) & (iy < L)
            e, r = cand(np.clip(ix, 0, L - 1), np.clip(iy, 0, L - 1))
            better = ok & (e < berr)
            bx = np.where(better, ix, bx)
            by = np.where(better, iy, by)
            br = np.where(better, r, br)
            berr = np.where(better, e, berr)
    return bx, by, br, berr


def exhaustive_round(t, dir_c, rho_c):
    """Best code over ALL (i_xi, i_eta, i_rho): the joint rounding's target."""
    t = np.asarray(t, dtype=np.float64)
    L, R = len(dir_c), len(rho_c)
    best = np.full(t.shape[:-1], np.inf)
    bx = np.zeros(t.shape[:-1], dtype=np.int64)
    by = np.zeros_like(bx)
    br = np.zeros_like(bx)
    for ix in range(L):
        for iy in range(L):
            nh = oct_inverse(dir_c[ix], dir_c[iy])
            for ir in range(R):
                e = np.sum((t - rho_c[ir] * nh) ** 2, axis=-1)
                better = e < best
                best = np.where(better, e, best)
                bx = np.where(better, ix, bx)
                by = np.where(better, iy, by)
                br = np.where(better, ir, br)
    return bx, by, br, best


# --------------------------------------------------------------------------
# Bit packing (compact bit stream; layout is a reading).
# --------------------------------------------------------------------------
def direction_field(i_xi, i_eta, b: int):
    """Ordered direction cells -> the 2(b+1)-bit direction field of a code.

    Reading: the direction codebook is odd-symmetric (c_k = -c_{L-1-k}, L =
    2^(b+1)), so each cell index i is stored as a sign and a magnitude rank:
    s = 1 for the lower half (i < 2^b, negative levels), m = rank of |c_i|
    among the positive levels (m = i - 2^b above the middle, 2^b - 1 - i
    below). Field = m_xi | m_eta << b | s_xi << 2b | s_eta << (2b + 1).
    """
    half = 1 << b
    fields = []
    for i in (np.asarray(i_xi, dtype=np.int64), np.asarray(i_eta, dtype=np.int64)):
        s = (i < half).astype(np.int64)
        m = np.where(i >= half, i - half, half - 1 - i)
        fields.append((s, m))
    (sx, mx), (sy, my) = fields
    return (mx | (my << b) | (sx << (2 * b)) | (sy << (2 * b + 1))).astype(np.uint64)


def direction_cells(field, b: int):
    """Inverse of direction_field: the ordered (i_xi, i_eta) cell indices."""
    f = np.asarray(field, dtype=np.int64)
    half = 1 << b
    mx, my = f & (half - 1), (f >> b) & (half - 1)
    sx, sy = (f >> (2 * b)) & 1, (f >> (2 * b + 1)) & 1
    i_xi = np.where(sx == 1, half - 1 - mx, half + mx)
    i_eta = np.where(sy == 1, half - 1 - my, half + my)
    return i_xi.astype(np.int64), i_eta.astype(np.int64)


def pack(i_xi, i_eta, i_rho, lay: Layout) -> np.ndarray:
    """[..., T] ordered cell indices -> [..., W] uint32 words (LSB-first stream).

    Triplet code (c = 2 b_dir + b_rho bits; 3b+1 for the OCTOPUS split) =
    direction field (2 b_dir bits, see direction_field with b_dir - 1
    magnitude bits) | i_rho << 2 b_dir. The code of triplet i occupies
    stream bits [i c, i c + c); stream bit p is bit p mod 32 of
    word p // 32, so a code that crosses a word boundary puts its low bits
    at the top of one word and its high bits at the bottom of the next.
    """
    code = direction_field(i_xi, i_eta, lay.b_dir - 1) | (np.asarray(i_rho, dtype=np.uint64) << np.uint64(2 * lay.b_dir))
    lead = code.shape[:-1]
    words = np.zeros(lead + (lay.words,), dtype=np.uint64)
    c = lay.code_bits
    for i in range(lay.T):
        p = i * c
        w, o = divmod(p, 32)
        words[..., w] |= (code[..., i] << np.uint64(o)) & np.uint64(0xFFFFFFFF)
        if o + c > 32:
            words[..., w + 1] |= code[..., i] >> np.uint64(32 - o)
    return words.astype(np.uint32)


def unpack(words: np.ndarray, lay: Layout):
    """[..., W] uint32 -> (i_xi, i_eta, i_rho), each [..., T] int64 (inverse of pack)."""
    w = np.asarray(words, dtype=np.uint64)
    lead = w.shape[:-1]
    c = lay.code_bits
    mask = np.uint64((1 << c) - 1)
    code = np.zeros(lead + (lay.T,), dtype=np.uint64)
    for i in range(lay.T):
        p = i * c
        wi, o = divmod(p, 32)
        v = w[..., wi] >> np.uint64(o)
        if o + c > 32:
            v = v | (w[..., wi + 1] << np.uint64(32 - o))
        code[..., i] = v & mask
    m_field = np.uint64((1 << (2 * lay.b_dir)) - 1)
    m_rho = np.uint64((1 << lay.b_rho) - 1)
    i_xi, i_eta = direction_cells(code & m_field, lay.b_dir - 1)
    i_rho = ((code >> np.uint64(2 * lay.b_dir)) & m_rho).astype(np.int64)
    return i_xi, i_eta, i_rho


# --------------------------------------------------------------------------
# Encode / decode of whole keys.
# --------------------------------------------------------------------------
@dataclass
class Encoded:
    gamma: np.ndarray      # [..., ] key norms
    i_xi: np.ndarray       # [..., T]
    i_eta: np.ndarray      # [..., T]
    i_rho: np.ndarray      # [..., T]
    words: np.ndarray      # [..., W] uint32
    # diagnostics for boundary classification
    xi: np.ndarray         # [..., T] continuous xi
    eta: np.ndarray        # [..., T] continuous eta
    rho: np.ndarray        # [..., T] triplet norms
    t: np.ndarray          # [..., T, 3] rotated, padded triplets
    u_rot: np.ndarray      # [..., d] rotated unit direction
    err: np.ndarray        # [..., T] chosen squared error per triplet


def encode(keys: np.ndarray, signs: np.ndarray, tables, lay: Layout, rounding: int = JOINT) -> Encoded:
    """Encode keys [..., d] of ONE head (signs [d]) with tables (dir_c, dir_t, rho_c, rho_t).

    [EXPL] "triplet decomposition": (1) gamma = ||k|| kept in fp32, u = k /
    gamma; (2) sign-flipped WHT rotation; (3) triplets, zero pad, rho_i and
    n_i; (4) octahedral map of n_i and Lloyd-Max indexing of xi, eta, rho;
    then joint rounding ([EXPL] "joint rounding") unless rounding = SCALAR.
    """
    dir_c, dir_t, rho_c, rho_t = (np.asarray(a, dtype=np.float64) for a in tables)
    k = np.asarray(keys, dtype=np.float64)
    gamma = np.linalg.norm(k, axis=-1)
    u = np.where(gamma[..., None] > 0, k / np.where(gamma > 0, gamma, 1.0)[..., None], 0.0)
    u_rot = rotate(u, signs)
    t = triplets(u_rot)
    rho = np.linalg.norm(t, axis=-1)
    xi, eta = oct_forward(t)
    i_xi = scalar_index(xi, dir_t)
    i_eta = scalar_index(eta, dir_t)
    if rounding == SCALAR:
        i_rho = scalar_index(rho, rho_t)
        nh = oct_inverse(dir_c[i_xi], dir_c[i_eta])
        err = np.sum((t - rho_c[i_rho][..., None] * nh) ** 2, axis=-1)
    else:
        i_xi, i_eta, i_rho, err = joint_round(t, i_xi, i_eta, dir_c, rho_c, rho_t)
    words = pack(i_xi, i_eta, i_rho, lay)
    return Encoded(gamma, i_xi, i_eta, i_rho, words, xi, eta, rho, t, u_rot, err)


def decode_rotated(i_xi, i_eta, i_rho, tables, lay: Layout) -> np.ndarray:
    """u_rot_hat [..., d]: concat_i rho_hat_i n_hat_i, padding dropped."""
    dir_c, _, rho_c, _ = (np.asarray(a, dtype=np.float64) for a in tables)
    nh = oct_inverse(dir_c[np.asarray(i_xi)], dir_c[np.asarray(i_eta)])
    v = rho_c[np.asarray(i_rho)][..., None] * nh
    v = v.reshape(v.shape[:-2] + (3 * lay.T,))
    return v[..., :lay.d]


def decode_keys(gamma, i_xi, i_eta, i_rho, signs, tables, lay: Layout) -> np.ndarray:
    """Materialised keys k_hat = gamma * R^T u_rot_hat ([..., d])."""
    ur = decode_rotated(i_xi, i_eta, i_rho, tables, lay)
    R = rotation_matrix(signs)
    return np.asarray(gamma, dtype=np.float64)[..., None] * (ur @ R)


# --------------------------------------------------------------------------
# OCTOPUS-QJL residual sketch ([EXPL] "optional residual correction",
# [SUMM] "OCTOPUS-QJL").
# --------------------------------------------------------------------------
def qjl_encode(u_rot: np.ndarray, u_rot_hat: np.ndarray, S: np.ndarray):
    """Sign sketch of the rotated residual e = u_rot - u_rot_hat.

    Returns (bits [..., d] in {0,1} with bit = [ (S e)_j >= 0 ], nu = ||e||,
    projections S e for boundary diagnostics). m = d sketch rows (reading).
    """
    e = np.asarray(u_rot, dtype=np.float64) - np.asarray(u_rot_hat, dtype=np.float64)
    nu = np.linalg.norm(e, axis=-1)
    proj = e @ np.asarray(S, dtype=np.float64).T
    bits = (proj >= 0).astype(np.int64)
    return bits, nu, proj


def qjl_pack(bits: np.ndarray) -> np.ndarray:
    """[..., d] bits -> [..., d/32] uint32, bit j of the sketch at bit j%32 of word j//32."""
    b = np.asarray(bits, dtype=np.uint64)
    lead = b.shape[:-1]
    b = b.reshape(lead + (b.shape[-1] // 32, 32))
    return np.sum(b << np.arange(32, dtype=np.uint64), axis=-1).astype(np.uint32)


def qjl_unpack(words: np.ndarray, d: int) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint64)
    bits = (w[..., :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    return bits.reshape(w.shape[:-1] + (d,)).astype(np.int64)


def qjl_correction(q_rot: np.ndarray, bits: np.ndarray, nu: np.ndarray, S: np.ndarray) -> np.ndarray:
    """Estimate of q_rot . e from the sketch: nu sqrt(pi/2)/m <S q_rot, 2 bits - 1>.

    [EXPL] "optional residual correction": the 1-bit residual signs make the
    inner-product estimate unbiased in expectation (QJL estimator with a
    Gaussian projection of m rows). q_rot [..., d]; bits [N, d]; returns
    [..., N].
    """
    m = S.shape[0]
    p = np.asarray(q_rot, dtype=np.float64) @ np.asarray(S, dtype=np.float64).T   # [..., m]
    sg = 2.0 * np.asarray(bits, dtype=np.float64) - 1.0                         # [N, m]
    return (p @ sg.T) * np.asarray(nu, dtype=np.float64) * math.sqrt(math.pi / 2.0) / m
