"""Pins for the oracle's tables: generator, rotation, marginals, Lloyd-Max.

Each test checks the oracle against something other than itself: a published
test vector, a closed form, a textbook table, an exact identity or a Monte
Carlo estimate.
"""

import json
import math
import os

import numpy as np
import pytest
from scipy import integrate as sint
from scipy import stats

from oracle import codec, tables
from rotation_preconditioned_quantization_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- SplitMix64
def test_splitmix64_published_vector():
    g = _gold("textbook.json")
    out = tables.splitmix64(g["splitmix64_seed"], np.arange(1, 6))
    assert [int(v) for v in out] == [int(s) for s in g["splitmix64_first5"]]


def test_signs_are_pm1_and_seeded():
    s = tables.rotation_signs(7, 128, 4)
    assert s.shape == (4, 128)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert np.array_equal(s, tables.rotation_signs(7, 128, 4))
    assert not np.array_equal(s, tables.rotation_signs(8, 128, 4))
    # heads draw consecutive, disjoint stretches of one SplitMix64 stream:
    # row h is outputs h*d + 1 .. h*d + d, so a table of fewer heads is a
    # prefix of a table of more, and row h is not row 0 again
    assert np.array_equal(s[:2], tables.rotation_signs(7, 128, 2))
    for h in range(4):
        top = tables.splitmix64(7, np.arange(h * 128 + 1, h * 128 + 129)) >> np.uint64(63)
        assert np.array_equal(s[h] == -1.0, top == 1)
    assert not any(np.array_equal(s[0], s[h]) for h in range(1, 4))
    assert abs(np.mean(tables.rotation_signs(1, 256, 64))) < 0.02


def test_qjl_matrix_is_standard_normal():
    S = tables.qjl_matrix(3, 64, 4)
    assert S.shape == (4, 64, 64)
    assert np.array_equal(S, S.astype(np.float32).astype(np.float64))
    x = S.ravel()
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02
    assert stats.kstest(x, "norm").pvalue > 1e-3


# ---------------------------------------------------------------- rotation
def test_hadamard_small_by_hand():
    H4 = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], float)
    assert np.array_equal(codec.hadamard(4), H4)


@pytest.mark.parametrize("d", [2, 8, 64, 128, 256])
def test_hadamard_sylvester_recursion_and_orthogonality(d):
    H = codec.hadamard(d)
    h = np.array([[1.0]])
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    assert np.array_equal(H, h)
    Hi = H.astype(np.int64)
    assert np.array_equal(Hi @ Hi.T, d * np.eye(d, dtype=np.int64))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rotation_is_orthogonal_and_norm_preserving(d):
    s = tables.rotation_signs(5, d, 1)[0]
    R = codec.rotation_matrix(s)
    assert np.max(np.abs(R @ R.T - np.eye(d))) < 1e-14
    H = codec.hadamard(d) / math.sqrt(d)
    assert np.max(np.abs(H @ H - np.eye(d))) < 1e-14
    x = inputs.normal(1, (100, d), np.float64)
    assert np.max(np.abs(np.linalg.norm(codec.rotate(x, s), axis=1) - np.linalg.norm(x, axis=1))) < 1e-12


# ---------------------------------------------------------------- marginals
def _marginal_closed_form(x):
    """Closed form of the xi-marginal from the antiderivative of (a e^2 + b e + c)^(-3/2).

    For x >= 0 (the marginal is even): upper face |eta| <= 1-x has
    |v|^2 = 2e^2 - 2(1-x)e + x^2 + (1-x)^2, the unfolded lower part
    1-x <= eta <= 1 has |v|^2 = 2e^2 - 2(2-x)e + 1 + 2(1-x)^2, and
    int dE/(aE^2+bE+c)^(3/2) = 2(2aE+b)/((4ac-b^2) sqrt(aE^2+bE+c)).
    """
    x = abs(x)

    def F(e, a, b, c):
        return 2.0 * (2 * a * e + b) / ((4 * a * c - b * b) * math.sqrt(a * e * e + b * e + c))

    a1, b1, c1 = 2.0, -2.0 * (1 - x), x * x + (1 - x) ** 2
    a2, b2, c2 = 2.0, -2.0 * (2 - x), 1.0 + 2.0 * (1 - x) ** 2
    up = F(1 - x, a1, b1, c1) - F(0.0, a1, b1, c1)
    lo = F(1.0, a2, b2, c2) - F(1 - x, a2, b2, c2)
    return 2.0 * (up + lo) / (4.0 * math.pi)


def test_direction_marginal_matches_closed_form():
    xs = np.linspace(-1, 1, 41)
    num = tables.direction_marginal(xs)
    ref = np.array([_marginal_closed_form(x) for x in xs])
    assert np.max(np.abs(num - ref)) < 1e-13


def test_direction_density_mass():
    tot = tables.integrate(tables.direction_marginal, [-1, 0, 1], 32, 0.25)
    assert abs(tot - 1.0) < 1e-13
    # the diamond |xi|+|eta| <= 1 is the upper hemisphere: mass 1/2
    val, _ = sint.dblquad(lambda e, x: tables.direction_joint_density(x, e),
                          0, 1, lambda x: 0.0, lambda x: 1 - x, epsabs=1e-13, epsrel=1e-13)
    assert abs(4 * val - 0.5) < 1e-10


def test_direction_density_monte_carlo():
    v = inputs.normal(11, (400000, 3), np.float64)
    xi, eta = codec.oct_forward(v)
    hist, edges = np.histogram(xi, bins=20, range=(-1, 1))
    p_mc = hist / len(xi)
    p = np.array([tables.integrate(tables.direction_marginal, [a, b], 24, 0.25)
                  for a, b in zip(edges[:-1], edges[1:])])
    # multinomial standard error ~ sqrt(p/n) ~ 5e-4
    assert np.max(np.abs(p - p_mc)) < 3e-3
    # joint density on a few boxes
    H2, ex, ey = np.histogram2d(xi, eta, bins=4, range=[[-1, 1], [-1, 1]])
    for i in range(4):
        for j in range(4):
            val, _ = sint.dblquad(lambda e, x: tables.direction_joint_density(x, e),
                                  ex[i], ex[i + 1], ey[j], ey[j + 1], epsabs=1e-9)
            assert abs(val - H2[i, j] / len(xi)) < 3e-3


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rho_density_moments(d):
    f = lambda r: tables.rho_density(r, d)
    assert abs(tables.integrate(f, [0, 1], 32, 1 / 64) - 1.0) < 1e-12
    # E[rho^2] = 3/d exactly for a uniform direction
    m2 = tables.integrate(lambda r: r * r * f(r), [0, 1], 32, 1 / 64)
    assert abs(m2 - 3.0 / d) < 1e-13


@pytest.mark.parametrize("d", [64, 128, 256])
def test_lemma_3_1_concentration(d):
    """Triplet norms of rotated Gaussian keys: sum rho^2 = 1, E rho^2 = 3/d, law = rho_density."""
    k = inputs.gaussian_keys(3, 1, 4000, d)[0].astype(np.float64)
    s = tables.rotation_signs(0, d, 1)[0]
    u = k / np.linalg.norm(k, axis=1, keepdims=True)
    t = codec.triplets(codec.rotate(u, s))
    rho = np.linalg.norm(t, axis=-1)
    assert np.max(np.abs(np.sum(rho ** 2, axis=1) - 1.0)) < 1e-12
    full = rho[:, : d // 3]                     # triplets without padding
    assert abs(np.mean(full ** 2) - 3.0 / d) < 0.02 * 3.0 / d
    grid = np.linspace(0, 1, 2001)
    cdf = np.concatenate([[0.0], np.cumsum([tables.integrate(lambda r: tables.rho_density(r, d), [a, b], 16, 1)
                                            for a, b in zip(grid[:-1], grid[1:])])])
    ks = stats.kstest(full[:, 0], lambda x: np.interp(x, grid, cdf))
    assert ks.pvalue > 1e-3


def test_lemma_3_1_variance_scales_as_1_over_d():
    """d Var(rho) is O(1): it tends to Var(chi_3) = 3 - 8/pi, and sqrt(d) E rho to E chi_3."""
    dv = []
    for d in (64, 128, 256):
        m1 = tables.integrate(lambda r: r * tables.rho_density(r, d), [0, 1], 32, 1 / 64)
        dv.append(d * (3.0 / d - m1 * m1))
        assert abs(math.sqrt(d) * m1 - 2.0 * math.sqrt(2.0 / math.pi)) < 0.02
    assert dv[0] < dv[1] < dv[2] < 3.0 - 8.0 / math.pi
    assert max(dv) / min(dv) < 1.05


# ---------------------------------------------------------------- Lloyd-Max
def test_lloyd_max_uniform_density():
    c, t, _ = tables.lloyd_max(lambda x: np.ones_like(x), 0.0, 1.0, 8, tol=1e-14)
    assert np.max(np.abs(c - (np.arange(8) + 0.5) / 8)) < 1e-12
    assert np.max(np.abs(t - np.arange(1, 8) / 8)) < 1e-12


def test_lloyd_max_gaussian_textbook():
    g = _gold("textbook.json")
    pdf = lambda x: np.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
    c1, _, _ = tables.lloyd_max(pdf, -12.0, 12.0, 2, kinks=(0.0,), tol=1e-14, max_width=0.5)
    assert np.max(np.abs(c1 - np.array(g["gauss_1bit_levels"]))) < 1e-4
    assert abs(c1[1] - math.sqrt(2 / math.pi)) < 1e-12
    c2, t2, _ = tables.lloyd_max(pdf, -12.0, 12.0, 4, kinks=(0.0,), tol=1e-14, max_width=0.5)
    assert np.max(np.abs(c2 - np.array(g["gauss_2bit_levels"]))) < 1e-3
    assert np.max(np.abs(t2 - np.array(g["gauss_2bit_thresholds"]))) < 1e-3


@pytest.mark.parametrize("b", [2, 3, 4])
def test_direction_codebook_optimality(b):
    c, t = tables.direction_codebook(b)
    assert len(c) == 1 << (b + 1)
    assert np.all(np.diff(c) > 0) and np.array_equal(c, -c[::-1])
    assert np.max(np.abs(t - 0.5 * (c[:-1] + c[1:]))) == 0.0
    edges = np.concatenate([[-1.0], t, [1.0]])
    for k in range(len(c)):
        a, e = edges[k], edges[k + 1]
        pts = [0.0] if a < 0 < e else None
        m0, _ = sint.quad(lambda x: _marginal_closed_form(x), a, e, points=pts, epsabs=1e-14, epsrel=1e-13)
        m1, _ = sint.quad(lambda x: x * _marginal_closed_form(x), a, e, points=pts, epsabs=1e-14, epsrel=1e-13)
        assert abs(m1 / m0 - c[k]) < 1e-10


@pytest.mark.parametrize("d,b", [(64, 2), (128, 3), (128, 4), (256, 4)])
def test_rho_codebook_optimality(d, b):
    c, t = tables.rho_codebook(d, b)
    assert len(c) == 1 << (b - 1)
    edges = np.concatenate([[0.0], t, [1.0]])
    pdf = lambda r: float(tables.rho_density(r, d))
    for k in range(len(c)):
        m0, _ = sint.quad(pdf, edges[k], edges[k + 1], epsabs=1e-15, epsrel=1e-13, limit=200)
        m1, _ = sint.quad(lambda r: r * pdf(r), edges[k], edges[k + 1], epsabs=1e-15, epsrel=1e-13, limit=200)
        assert abs(m1 / m0 - c[k]) < 1e-10
    assert np.max(np.abs(t - 0.5 * (c[:-1] + c[1:]))) < 1e-15
