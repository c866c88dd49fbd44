"""Oracle: the codec's data-independent tables (test infrastructure only).

* rotation signs and the QJL projection, drawn from SplitMix64;
* the analytic marginals the Lloyd-Max codebooks are designed against;
* the Lloyd-Max iteration itself.

The codebooks depend only on the key dimension d and the bit budget b
([SUMM] "bit allocation": the allocation depends only on d, so codebooks are
generated ahead of time; [ABS]: "data-oblivious, online, and deterministic
given a seed").
"""

from __future__ import annotations

import functools
import math

import numpy as np

M64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15


# --------------------------------------------------------------------------
# SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
# generators", OOPSLA 2014; 64-bit finaliser constants as published by
# S. Vigna). Counter form: output number n (n >= 1) of the generator seeded
# with ``seed`` is mix(seed + n * GOLDEN mod 2^64).
# --------------------------------------------------------------------------
def splitmix64(seed: int, n: np.ndarray) -> np.ndarray:
    """The ``n``-th outputs (uint64 array, n >= 1) of SplitMix64 seeded with ``seed``."""
    n = np.asarray(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & M64) + n * np.uint64(GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def rotation_signs(seed: int, d: int, n_heads: int) -> np.ndarray:
    """[n_heads][d] float64 of +-1: the diagonal D_s of the sign-flipped WHT.

    [EXPL] "rotation": the rotation is a sign-flipped Walsh-Hadamard
    transform; [ABS]: deterministic given a seed. Reading: sign j of head h
    is -1 when the top bit of SplitMix64 output number h*d + j + 1 is set.
    """
    idx = np.arange(n_heads * d, dtype=np.uint64) + np.uint64(1)
    top = splitmix64(seed, idx) >> np.uint64(63)
    return np.where(top == 1, -1.0, 1.0).reshape(n_heads, d)


def qjl_matrix(seed: int, d: int, n_heads: int) -> np.ndarray:
    """[n_heads][d][d] float32-valued Gaussian projection S (returned as float64).

    [EXPL] "optional residual correction": the residual is projected again
    with an independent random transform and only its signs are kept. Reading
    (the pages disagree on the transform; the LLM-shaped QJL workload names a
    seeded Gaussian projection): entry e = (h*d + i)*d + j takes two uniforms
    from SplitMix64 outputs 2e+1 and 2e+2, u1 = ((z1 >> 11) + 1) * 2^-53 in
    (0, 1], u2 = (z2 >> 11) * 2^-53 in [0, 1), and the Box-Muller normal
    sqrt(-2 ln u1) * cos(2 pi u2), rounded to float32.
    """
    n = n_heads * d * d
    e = np.arange(n, dtype=np.uint64)
    z1 = splitmix64(seed, np.uint64(2) * e + np.uint64(1))
    z2 = splitmix64(seed, np.uint64(2) * e + np.uint64(2))
    u1 = ((z1 >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (z2 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    g = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return g.astype(np.float32).astype(np.float64).reshape(n_heads, d, d)


# --------------------------------------------------------------------------
# Quadrature: composite Gauss-Legendre between breakpoints.
# --------------------------------------------------------------------------
@functools.lru_cache(maxsize=None)
def _gl(n: int):
    x, w = np.polynomial.legendre.leggauss(n)
    return x, w


def integrate(f, breaks, n: int = 32, max_width: float = 0.125) -> float:
    """Integral of vectorised ``f`` over [breaks[0], breaks[-1]].

    Panels are split at every breakpoint and then into equal pieces no wider
    than ``max_width``; each piece gets an ``n``-point Gauss-Legendre rule.
    """
    x0, w0 = _gl(n)
    br = np.unique(np.asarray(breaks, dtype=np.float64))
    xs, ws = [], []
    for a, b in zip(br[:-1], br[1:]):
        if b <= a:
            continue
        m = max(1, int(math.ceil((b - a) / max_width)))
        edges = np.linspace(a, b, m + 1)
        for lo, hi in zip(edges[:-1], edges[1:]):
            h = 0.5 * (hi - lo)
            xs.append(lo + h * (x0 + 1.0))
            ws.append(h * w0)
    if not xs:
        return 0.0
    x = np.concatenate(xs)
    w = np.concatenate(ws)
    return float(np.dot(w, f(x)))


# --------------------------------------------------------------------------
# Analytic marginals.
# --------------------------------------------------------------------------
def octahedral_vector(xi, eta):
    """Unnormalised inverse octahedral map v(xi, eta) (see codec.oct_inverse)."""
    xi = np.asarray(xi, dtype=np.float64)
    eta = np.asarray(eta, dtype=np.float64)
    r = 1.0 - np.abs(xi) - np.abs(eta)
    sx = np.where(xi >= 0, 1.0, -1.0)
    sy = np.where(eta >= 0, 1.0, -1.0)
    x = np.where(r >= 0, xi, (1.0 - np.abs(eta)) * sx)
    y = np.where(r >= 0, eta, (1.0 - np.abs(xi)) * sy)
    return x, y, r


def direction_joint_density(xi, eta):
    """Density on [-1,1]^2 of (xi, eta) = octahedral map of a uniform S^2 direction.

    [EXPL] "octahedral folding": the square is the unfolded octahedron
    |x|+|y|+|z| = 1. A face of that octahedron has area element sqrt(3) dxi
    deta over the square (the fold has unit Jacobian), and the solid angle
    subtended by a surface element at point v is (v . N) dA / |v|^3 with
    v . N = 1/sqrt(3). So the density of a uniform direction (solid angle
    / 4 pi) is 1 / (4 pi |v(xi, eta)|^3).
    """
    x, y, z = octahedral_vector(xi, eta)
    nv = np.sqrt(x * x + y * y + z * z)
    return 1.0 / (4.0 * math.pi * nv ** 3)


def direction_marginal(xi) -> np.ndarray:
    """Marginal density of xi (and, by symmetry, of eta) on [-1, 1].

    [ABS] "Lloyd-Max quantized against implementation-matched marginals";
    [SUMM] "method overview": one-dimensional Lloyd-Max on the two mapped
    coordinates. Reading: the exact marginal of the map of a uniform S^2
    direction, i.e. the integral over eta of direction_joint_density, with
    quadrature panels split where the integrand has kinks (eta = 0 and
    |xi| + |eta| = 1).
    """
    shape = np.shape(xi)
    x = np.asarray(xi, dtype=np.float64).reshape(-1, 1, 1)
    x0, w0 = _gl(48)
    a = 1.0 - np.abs(x)
    lo = np.concatenate([np.full_like(a, -1.0), -a, np.zeros_like(a), a], axis=1)
    hi = np.concatenate([-a, np.zeros_like(a), a, np.ones_like(a)], axis=1)
    h = 0.5 * (hi - lo)                       # [n, 4, 1]
    y = lo + h * (x0[None, None, :] + 1.0)    # [n, 4, 48]
    f = direction_joint_density(np.broadcast_to(x, y.shape), y)
    out = np.sum(h[..., 0] * (f @ w0), axis=1)
    return out.reshape(shape)


def rho_density(rho, d: int) -> np.ndarray:
    """Density of a triplet norm rho of a uniform unit vector in R^d.

    [EXPL] "triplet decomposition" (Lemma 3.1: rho concentrates near
    sqrt(3/d)). For u uniform on S^{d-1}, rho^2 = u1^2+u2^2+u3^2 is
    Beta(3/2, (d-3)/2), so rho has density
    2 rho^2 (1 - rho^2)^((d-5)/2) / B(3/2, (d-3)/2) on [0, 1].
    """
    rho = np.asarray(rho, dtype=np.float64)
    a, b = 1.5, 0.5 * (d - 3)
    lbeta = math.lgamma(a) + math.lgamma(b) - math.lgamma(a + b)
    one = np.clip(1.0 - rho * rho, 0.0, None)
    return 2.0 * rho * rho * one ** (0.5 * (d - 5)) * math.exp(-lbeta)


# --------------------------------------------------------------------------
# Lloyd-Max.
# --------------------------------------------------------------------------
def lloyd_max(pdf, lo: float, hi: float, levels: int, kinks=(), tol: float = 1e-13,
              max_iter: int = 200000, init=None, n_nodes: int = 32,
              max_width: float = 0.125):
    """Lloyd-Max scalar quantiser of ``levels`` levels for density ``pdf`` on [lo, hi].

    [EXPL] "triplet decomposition": the Lloyd-Max quantiser cuts the line into
    cells chosen from the probability law. The two optimality conditions
    are iterated in turn: every threshold is the midpoint of its two
    neighbouring centroids, every centroid is the conditional mean of its
    cell. Stops when no centroid moves by more than ``tol``.

    Returns (centroids[levels], thresholds[levels-1], iterations).
    """
    kinks = [k for k in kinks if lo < k < hi]

    def cell_moments(a, b):
        br = [a] + [k for k in kinks if a < k < b] + [b]
        m0 = integrate(pdf, br, n_nodes, max_width)
        m1 = integrate(lambda x: x * pdf(x), br, n_nodes, max_width)
        return m0, m1

    if init is None:
        # start from equal-probability cells (quantiles of a fine CDF table)
        grid = np.linspace(lo, hi, 4001)
        dens = pdf(grid)
        cdf = np.concatenate([[0.0], np.cumsum(0.5 * (dens[1:] + dens[:-1]) * np.diff(grid))])
        cdf /= cdf[-1]
        t = np.interp(np.arange(1, levels) / levels, cdf, grid)
    else:
        t = np.asarray(init, dtype=np.float64)
    c = np.zeros(levels)
    edges = np.concatenate([[lo], t, [hi]])
    for k in range(levels):
        m0, m1 = cell_moments(edges[k], edges[k + 1])
        c[k] = m1 / m0 if m0 > 0 else 0.5 * (edges[k] + edges[k + 1])
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[lo], t, [hi]])
        cn = np.empty(levels)
        for k in range(levels):
            m0, m1 = cell_moments(edges[k], edges[k + 1])
            cn[k] = m1 / m0 if m0 > 0 else 0.5 * (edges[k] + edges[k + 1])
        delta = float(np.max(np.abs(cn - c)))
        c = cn
        if delta < tol:
            break
    t = 0.5 * (c[:-1] + c[1:])
    return c, t, it


@functools.lru_cache(maxsize=None)
def direction_codebook_levels(levels: int, tol: float = 1e-13):
    """Lloyd-Max codebook of ``levels`` levels for direction_marginal, symmetrised."""
    c, t, _ = lloyd_max(direction_marginal, -1.0, 1.0, levels, kinks=(0.0,),
                        tol=tol, n_nodes=24, max_width=0.25)
    c = 0.5 * (c - c[::-1])
    return c, 0.5 * (c[:-1] + c[1:])


@functools.lru_cache(maxsize=None)
def rho_codebook_levels(d: int, levels: int, tol: float = 1e-14):
    """Lloyd-Max codebook of ``levels`` levels for rho_density(., d)."""
    c, t, _ = lloyd_max(lambda r: rho_density(r, d), 0.0, 1.0, levels, tol=tol,
                        n_nodes=32, max_width=1.0 / 64)
    return c, t


def direction_codebook(b: int):
    """Codebook for xi and eta: 2^(b+1) levels on [-1, 1].

    [EXPL] "non-uniform bit allocation": the direction coordinates get b+1
    bits. [SUMM] "method overview": xi and eta share one 1-D Lloyd-Max
    quantiser (the marginal is the same for both by symmetry). The
    marginal is symmetric, so the result is symmetrised (c_k = -c_{L-1-k}).
    """
    return direction_codebook_levels(1 << (b + 1))


def rho_codebook(d: int, b: int):
    """Codebook for the triplet norm: 2^(b-1) levels on [0, 1].

    [EXPL] "non-uniform bit allocation": rho gets b-1 bits; its marginal
    is rho_density for the key dimension d (the same for every triplet,
    including a zero-padded last one, since the codebooks depend only on d
    and b).
    """
    return rho_codebook_levels(d, 1 << (b - 1))


def codebooks(d: int, b: int):
    """(dir_c, dir_t, rho_c, rho_t) float64 for key dimension d and budget b."""
    dc, dt = direction_codebook(b)
    rc, rt = rho_codebook(d, b)
    return dc.copy(), dt.copy(), rc.copy(), rt.copy()


def as_f32(*arrs):
    """Round tables to float32 values (still float64 arrays)."""
    return tuple(np.asarray(a, dtype=np.float32).astype(np.float64) for a in arrs)
