"""Pins for the oracle's codec: octahedral map, indexing, joint rounding,
packing, codec quality against the pages' printed numbers, logits, attention
and the QJL sketch."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention, baselines, codec, tables
from rotation_preconditioned_quantization_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _unit(seed, n):
    v = inputs.normal(seed, (n, 3), np.float64)
    return v / np.linalg.norm(v, axis=1, keepdims=True)


# ---------------------------------------------------------------- octahedral
def test_octahedral_round_trip():
    n = _unit(1, 1_000_000)
    xi, eta = codec.oct_forward(n)
    assert np.all(np.abs(xi) <= 1) and np.all(np.abs(eta) <= 1)
    back = codec.oct_inverse(xi, eta)
    assert np.max(np.abs(back - n)) < 1e-12
    # upper hemisphere <-> inside the diamond
    inside = np.abs(xi) + np.abs(eta) <= 1 + 1e-15
    assert np.array_equal(inside, n[:, 2] >= 0) or np.mean(inside != (n[:, 2] >= 0)) < 1e-5


def test_octahedral_special_points():
    pts = np.array([[0, 0, 1], [0, 0, -1], [1, 0, 0], [-1, 0, 0], [0, 1, 0], [0, -1, 0],
                    [1, 1, -1e-300], [0.0, 0.0, 0.0]], float)
    xi, eta = codec.oct_forward(pts)
    want = np.array([[0, 0], [1, 1], [1, 0], [-1, 0], [0, 1], [0, -1], [0, 0], [0, 0]], float)
    got = np.stack([xi, eta], axis=1)
    assert np.allclose(got[:6], want[:6], atol=0)
    # a point just below the equator on the x=y diagonal: p = (1/2, 1/2, -tiny) takes the
    # lower branch, ((1 - 1/2) sgn p_x, (1 - 1/2) sgn p_y) = (1/2, 1/2), the same point
    # the upper branch gives on the equator (the fold is continuous there)
    assert np.array_equal(got[6], [0.5, 0.5])
    assert np.array_equal(got[7], [0.0, 0.0])
    # corners of the square are the south pole, centre the north pole
    assert np.allclose(codec.oct_inverse(np.array([1.0, -1, 1, -1]), np.array([1.0, 1, -1, -1])),
                       np.tile([0, 0, -1.0], (4, 1)), atol=1e-15)
    assert np.allclose(codec.oct_inverse(0.0, 0.0), [0, 0, 1.0])


def test_octahedral_by_hand():
    # n = (1, 2, 2)/3 : l1 = 5/3 -> p = (0.2, 0.4, 0.4), upper: (0.2, 0.4)
    xi, eta = codec.oct_forward(np.array([1.0, 2.0, 2.0]) / 3)
    assert abs(xi - 0.2) < 1e-15 and abs(eta - 0.4) < 1e-15
    # n = (1, -2, -2)/3 : p = (0.2, -0.4, -0.4), lower: ((1-0.4)*1, (1-0.2)*(-1)) = (0.6, -0.8)
    xi, eta = codec.oct_forward(np.array([1.0, -2.0, -2.0]) / 3)
    assert abs(xi - 0.6) < 1e-15 and abs(eta + 0.8) < 1e-15
    # inverse of (0.6, -0.8): r = -0.4 -> v = ((1-0.8), -(1-0.6), -0.4) = (0.2, -0.4, -0.4)
    v = codec.oct_inverse(0.6, -0.8)
    assert np.allclose(v, np.array([1.0, -2.0, -2.0]) / 3, atol=1e-15)


# ---------------------------------------------------------------- indexing
@pytest.mark.parametrize("b", [2, 3, 4])
def test_scalar_index_is_nearest_centroid(b):
    c, t = tables.direction_codebook(b)
    x = inputs.rng(b).uniform(-1, 1, 100000)
    idx = codec.scalar_index(x, t)
    brute = np.argmin(np.abs(x[:, None] - c[None, :]), axis=1)
    assert np.array_equal(idx, brute)
    # a value exactly on a threshold goes to the upper cell
    assert np.array_equal(codec.scalar_index(t, t), np.arange(1, len(c)))


def _rot_triplets(seed, n, d=128):
    k = inputs.gaussian_keys(seed, 1, n, d)[0].astype(np.float64)
    s = tables.rotation_signs(seed, d, 1)[0]
    u = k / np.linalg.norm(k, axis=1, keepdims=True)
    return codec.triplets(codec.rotate(u, s))[:, : d // 3].reshape(-1, 3)


@pytest.mark.parametrize("b", [2, 3, 4])
def test_joint_rounding_equals_exhaustive(b):
    """[EXPL] "joint rounding": the 3x3 search matched exhaustive search on 10 000 triplets."""
    g = _gold("synthetic_quality.json")["joint_3x3_equals_exhaustive"]
    d = 128
    dc, dt, rc, rt = tables.codebooks(d, b)
    t = _rot_triplets(40 + b, 240)[: g["triplets"]]
    t = np.concatenate([t, _rot_triplets(90 + b, 240)])[: g["triplets"]]
    assert len(t) == g["triplets"]
    xi, eta = codec.oct_forward(t)
    _, _, _, ej = codec.joint_round(t, codec.scalar_index(xi, dt), codec.scalar_index(eta, dt), dc, rc, rt)
    _, _, _, ee = codec.exhaustive_round(t, dc, rc)
    assert np.max(ej - ee) < 1e-15


def test_joint_rounding_tiny_brute_force():
    """Hand-checkable case: 2 direction levels... via a full enumeration on random triplets."""
    dc = np.array([-0.5, 0.5])
    rc = np.array([0.1, 0.3])
    rt = np.array([0.2])
    t = inputs.normal(5, (500, 3), np.float64) * 0.2
    xi, eta = codec.oct_forward(t)
    ix, iy, ir, e = codec.joint_round(t, codec.scalar_index(xi, [0.0]), codec.scalar_index(eta, [0.0]), dc, rc, rt)
    bx, by, br, be = codec.exhaustive_round(t, dc, rc)
    assert np.max(np.abs(e - be)) < 1e-15
    # the error formula is ||t - rho_hat n_hat||^2
    nh = codec.oct_inverse(dc[ix], dc[iy])
    assert np.max(np.abs(np.sum((t - rc[ir][:, None] * nh) ** 2, axis=1) - e)) < 1e-15


def test_joint_rho_is_nearest_to_projection():
    """For a fixed direction the best rho level is the one nearest s = n_hat . t."""
    d, b = 128, 3
    dc, dt, rc, rt = tables.codebooks(d, b)
    t = _rot_triplets(3, 50)
    xi, eta = codec.oct_forward(t)
    ix, iy = codec.scalar_index(xi, dt), codec.scalar_index(eta, dt)
    nh = codec.oct_inverse(dc[ix], dc[iy])
    errs = np.stack([np.sum((t - r * nh) ** 2, axis=1) for r in rc], axis=1)
    s = np.sum(nh * t, axis=1)
    assert np.array_equal(np.argmin(errs, axis=1), np.argmin(np.abs(s[:, None] - rc[None, :]), axis=1))


# ---------------------------------------------------------------- packing
def test_pack_by_hand():
    # b=2 (c = 7 bits, half = 4): cells (xi 5, eta 3, rho 1) -> m_xi 1, s_xi 0, m_eta 0, s_eta 1:
    # 1 | 0 << 2 | 0 << 4 | 1 << 5 | 1 << 6 = 97; (7, 0, 1) -> 3 | 3 << 2 | 0 | 1 << 5 | 1 << 6 = 111
    lay = codec.Layout(6, 2)
    w = codec.pack(np.array([[5, 7]]), np.array([[3, 0]]), np.array([[1, 1]]), lay)
    assert lay.words == 1 and int(w[0, 0]) == 97 + (111 << 7)
    # b=4 (c = 13 bits, half = 16): (28, 5, 5) -> 12 | 10 << 4 | 1 << 9 | 5 << 10 = 0x16AC,
    # (16, 15, 0) -> 0 | 0 | 1 << 9 = 0x200, (0, 31, 7) -> 15 | 15 << 4 | 1 << 8 | 7 << 10 = 0x1DFF;
    # the third code crosses into word 1
    lay = codec.Layout(9, 4)
    w = codec.pack(np.array([[28, 16, 0]]), np.array([[5, 15, 31]]), np.array([[5, 0, 7]]), lay)
    assert lay.words == 2
    assert int(w[0, 0]) == (0x16AC | (0x200 << 13) | ((0x1DFF & 63) << 26))
    assert int(w[0, 1]) == 0x1DFF >> 6


def _code_by_hand(ix, iy, ir, b):
    half = 1 << b
    sx, sy = int(ix < half), int(iy < half)
    mx = ix - half if ix >= half else half - 1 - ix
    my = iy - half if iy >= half else half - 1 - iy
    return mx | my << b | sx << 2 * b | sy << (2 * b + 1) | ir << (2 * b + 2)


@pytest.mark.parametrize("d,b", [(64, 2), (128, 3), (128, 4), (256, 2), (256, 4)])
def test_pack_round_trip_and_sizes(d, b):
    lay = codec.Layout(d, b)
    assert lay.code_bits == 3 * b + 1
    assert lay.words == math.ceil(lay.T * (3 * b + 1) / 32)
    ix = inputs.random_codes(1, (7, lay.T), lay.n_dir)
    iy = inputs.random_codes(2, (7, lay.T), lay.n_dir)
    ir = inputs.random_codes(3, (7, lay.T), lay.n_rho)
    w = codec.pack(ix, iy, ir, lay)
    # bit-by-bit reference of the stream
    for r in range(7):
        stream = 0
        for i in range(lay.T):
            stream |= _code_by_hand(int(ix[r, i]), int(iy[r, i]), int(ir[r, i]), b) << (i * lay.code_bits)
        assert [int(x) for x in w[r]] == [(stream >> (32 * j)) & 0xFFFFFFFF for j in range(lay.words)]
    a, bb, c = codec.unpack(w, lay)
    assert np.array_equal(a, ix) and np.array_equal(bb, iy) and np.array_equal(c, ir)


def test_direction_field_pairs_opposite_cells():
    # cells i and L-1-i (levels c and -c) share the magnitude and differ only in the sign bit
    for b in (2, 3, 4):
        L = 1 << (b + 1)
        i = np.arange(L)
        f = codec.direction_field(i, np.zeros_like(i), b).astype(np.int64)
        g = codec.direction_field(L - 1 - i, np.zeros_like(i), b).astype(np.int64)
        sign = 1 << (2 * b)
        assert np.array_equal(f ^ g, np.full(L, sign))
        assert np.array_equal(np.sort(f & ((1 << b) - 1)), np.repeat(np.arange(1 << b), 2))


# ---------------------------------------------------------------- quality
def _mse(d, b, mode, reps=4, n=1024, dir_bits=None, rho_bits=None):
    if dir_bits is None:
        dc, dt, rc, rt = tables.codebooks(d, b)
    else:
        # the sweep's MSE (second order in centroid errors) needs codebooks to ~1e-7, not to the 1e-13 of the shipped tables
        dc, dt = tables.direction_codebook_levels(1 << dir_bits, 1e-7)
        rc, rt = tables.rho_codebook_levels(d, 1 << rho_bits, 1e-7)
    lay = codec.Layout(d, b)
    out = []
    for rep in range(reps):
        k = inputs.gaussian_keys(1000 + rep, 1, n, d)[0].astype(np.float64)
        s = tables.rotation_signs(rep, d, 1)[0]
        u = k / np.linalg.norm(k, axis=1, keepdims=True)
        t = codec.triplets(codec.rotate(u, s))
        xi, eta = codec.oct_forward(t)
        ix, iy = codec.scalar_index(xi, dt), codec.scalar_index(eta, dt)
        if mode == codec.SCALAR:
            ir = codec.scalar_index(np.linalg.norm(t, axis=-1), rt)
        else:
            ix, iy, ir, _ = codec.joint_round(t, ix, iy, dc, rc, rt)
        nh = codec.oct_inverse(dc[ix], dc[iy])
        ur = (rc[ir][..., None] * nh).reshape(n, -1)[:, :d]
        uh = ur @ codec.rotation_matrix(s)
        out.append(np.mean(np.sum((u - uh) ** 2, axis=1)))
    return float(np.mean(out))


@pytest.mark.parametrize("b", [2, 4])
def test_mse_matches_printed_values(b):
    g = _gold("synthetic_quality.json")["mse"]
    printed = g[f"octopus_b{b}"]
    scalar = _mse(128, b, codec.SCALAR)
    joint = _mse(128, b, codec.JOINT)
    assert abs(scalar - printed) < 0.03 * printed
    assert abs(joint - printed) < 0.10 * printed
    assert joint < scalar


def test_per_coordinate_baseline_matches_printed_value():
    g = _gold("synthetic_quality.json")["mse"]
    k = inputs.gaussian_keys(1000, 1, 1024, 128)[0].astype(np.float64)
    u = k / np.linalg.norm(k, axis=1, keepdims=True)
    m = baselines.per_coordinate_mse(u, tables.rotation_signs(0, 128, 1)[0], 4)
    assert abs(m - g["turboquant_mse_b4"]) < 0.03 * g["turboquant_mse_b4"]


@pytest.mark.parametrize("b", [2, 3, 4])
def test_octopus_beats_per_coordinate_lloyd_max(b):
    k = inputs.gaussian_keys(1000, 1, 1024, 128)[0].astype(np.float64)
    u = k / np.linalg.norm(k, axis=1, keepdims=True)
    base = baselines.per_coordinate_mse(u, tables.rotation_signs(0, 128, 1)[0], b)
    assert _mse(128, b, codec.JOINT, reps=1) < base


@pytest.mark.parametrize("b", [3, 4])
def test_bit_allocation_sweep(b):
    """[EXPL] "non-uniform bit allocation": delta=+1 is best; +2 is 44-73% worse than 0; -1 >200% worse."""
    g = _gold("synthetic_quality.json")["delta_sweep"]
    m = {dl: _mse(128, b, codec.JOINT, reps=1, dir_bits=b + dl, rho_bits=b - dl) for dl in (-1, 0, 1, 2)}
    assert min(m, key=m.get) == g["best_delta"]
    gain = 100 * (1 - m[1] / m[0])
    lo, hi = g["gain_delta_plus1_vs_0_percent"]
    assert lo - 10 <= gain <= hi + 10
    assert 100 * (m[-1] / m[0] - 1) > g["loss_delta_minus1_vs_0_percent_min"]
    lo, hi = g["loss_delta_plus2_vs_0_percent"]
    assert lo - 10 <= 100 * (m[2] / m[0] - 1) <= hi + 10


@pytest.mark.parametrize("d,b", [(64, 2), (128, 3), (256, 4)])
def test_joint_rounding_picks_the_candidate_of_largest_s(d, b):
    """With every norm centroid positive, the error rho^2 + min_l (c_l^2 - 2 c_l s) falls strictly
    as s = n_hat . t grows, so the 3x3 search's least-error candidate is the valid neighbour with the
    largest s (the encoder kernel searches by s and picks the norm level once)."""
    lay = codec.Layout(d, b)
    dc, dt, rc, rt = (np.asarray(x, dtype=np.float64) for x in tables.codebooks(d, b))
    assert np.all(rc > 0)
    k = inputs.gaussian_keys(31, 1, 200, d)[0].astype(np.float64)
    t = codec.triplets(codec.rotate(k / np.linalg.norm(k, axis=1, keepdims=True), tables.rotation_signs(3, d, 1)[0]))
    xi, eta = codec.oct_forward(t)
    ix0, iy0 = codec.scalar_index(xi, dt), codec.scalar_index(eta, dt)
    bx, by, br, _ = codec.joint_round(t, ix0, iy0, dc, rc, rt)
    L = len(dc)
    best_s = np.full(ix0.shape, -np.inf)
    sx, sy = ix0.copy(), iy0.copy()
    for dx, dy in [(0, 0)] + [(a, c) for a in (-1, 0, 1) for c in (-1, 0, 1) if (a, c) != (0, 0)]:
        ux, uy = ix0 + dx, iy0 + dy
        ok = (ux >= 0) & (ux < L) & (uy >= 0) & (uy < L)
        s = np.sum(codec.oct_inverse(dc[np.clip(ux, 0, L - 1)], dc[np.clip(uy, 0, L - 1)]) * t, axis=-1)
        take = ok & (s > best_s)
        sx, sy, best_s = np.where(take, ux, sx), np.where(take, uy, sy), np.where(take, s, best_s)
    assert np.array_equal(sx, bx) and np.array_equal(sy, by)
    assert np.array_equal(codec.scalar_index(best_s, rt), br)


def test_zero_key():
    d, b = 128, 3
    lay = codec.Layout(d, b)
    tb = tables.codebooks(d, b)
    e = codec.encode(np.zeros((2, d)), tables.rotation_signs(0, d, 1)[0], tb, lay)
    assert np.array_equal(e.gamma, [0.0, 0.0])
    L = lay.n_dir
    assert np.all(e.i_xi == L // 2) and np.all(e.i_eta == L // 2) and np.all(e.i_rho == 0)


def test_encode_matches_stepwise_definition():
    d, b = 128, 3
    lay = codec.Layout(d, b)
    tb = tables.codebooks(d, b)
    s = tables.rotation_signs(2, d, 1)[0]
    k = inputs.llm_keys(4, 1, 300, d)[0].astype(np.float64)
    e = codec.encode(k, s, tb, lay, codec.SCALAR)
    # independent restatement with explicit loops on a few keys
    H = np.array([[(-1) ** bin(i & j).count("1") for j in range(d)] for i in range(d)], float)
    for r in range(0, 300, 37):
        g = math.sqrt(sum(x * x for x in k[r]))
        assert abs(g - e.gamma[r]) < 1e-12 * g
        ur = H @ (s * k[r] / g) / math.sqrt(d)
        ur = list(ur) + [0.0] * (3 * lay.T - d)
        for i in range(lay.T):
            t = ur[3 * i: 3 * i + 3]
            l1 = sum(abs(x) for x in t)
            p = [x / l1 for x in t]
            if p[2] >= 0:
                xi, eta = p[0], p[1]
            else:
                xi = (1 - abs(p[1])) * (1 if p[0] >= 0 else -1)
                eta = (1 - abs(p[0])) * (1 if p[1] >= 0 else -1)
            assert e.i_xi[r, i] == int(np.argmin(np.abs(tb[0] - xi)))
            assert e.i_eta[r, i] == int(np.argmin(np.abs(tb[0] - eta)))
            rho = math.sqrt(sum(x * x for x in t))
            assert e.i_rho[r, i] == int(np.argmin(np.abs(tb[2] - rho)))


# ---------------------------------------------------------------- logits / attention
def test_logits_materialised_equals_rotated_query_route():
    d, b = 128, 3
    lay = codec.Layout(d, b)
    tb = tables.codebooks(d, b)
    s = tables.rotation_signs(9, d, 1)[0]
    k = inputs.llm_keys(1, 1, 500, d)[0]
    q = inputs.normal(2, (4, d), np.float64)
    e = codec.encode(k, s, tb, lay)
    lg = attention.logits(q, e.gamma, e.i_xi, e.i_eta, e.i_rho, s, tb, lay)
    ur = codec.decode_rotated(e.i_xi, e.i_eta, e.i_rho, tb, lay)
    lg2 = (codec.rotate(q, s) @ ur.T) * e.gamma[None, :]
    assert np.max(np.abs(lg - lg2)) < 1e-12 * np.max(np.abs(lg))


def test_attention_identity_codec_equals_sdpa():
    G, N, d = 4, 300, 64
    q = inputs.normal(1, (G, d), np.float64)
    K = inputs.normal(2, (N, d), np.float64)
    V = inputs.to_bf16(inputs.normal(3, (N, d))).astype(np.float64)
    out = attention.softmax_attention(q @ K.T, V, 1.0 / math.sqrt(d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0].numpy()
    assert np.max(np.abs(out - ref)) < 1e-13


def test_attention_of_decoded_keys_equals_sdpa_on_materialised_keys():
    d, b = 64, 2
    lay = codec.Layout(d, b)
    tb = tables.codebooks(d, b)
    s = tables.rotation_signs(1, d, 1)[0]
    k = inputs.gaussian_keys(5, 1, 200, d)[0]
    V = inputs.to_bf16(inputs.normal(6, (200, d))).astype(np.float64)
    q = inputs.normal(7, (8, d), np.float64)
    e = codec.encode(k, s, tb, lay)
    out, _ = attention.decode_attention(q, e.gamma, e.i_xi, e.i_eta, e.i_rho, V, s, tb, lay)
    kh = codec.decode_keys(e.gamma, e.i_xi, e.i_eta, e.i_rho, s, tb, lay)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(kh)[None], torch.from_numpy(V)[None])[0].numpy()
    assert np.max(np.abs(out - ref)) < 1e-13


# ---------------------------------------------------------------- key reconstruction
@pytest.mark.parametrize("d,b", [(64, 2), (128, 3), (256, 4)])
def test_decode_keys_matches_library_hadamard(d, b):
    """k_hat = gamma R^T u_hat with R = (1/sqrt(d)) H diag(s): rebuilt here from
    scipy's Sylvester Hadamard matrix (independent of the oracle's own H and
    of the orientation of its rotation matrix)."""
    import scipy.linalg

    lay = codec.Layout(d, b)
    tb = tables.codebooks(d, b)
    s = tables.rotation_signs(4, d, 1)[0]
    k = inputs.llm_keys(3, 1, 64, d)[0].astype(np.float64)
    e = codec.encode(k, s, tb, lay)
    ur = codec.decode_rotated(e.i_xi, e.i_eta, e.i_rho, tb, lay)
    H = scipy.linalg.hadamard(d).astype(np.float64)
    ref = e.gamma[:, None] * (ur @ H) * s[None, :] / math.sqrt(d)
    kh = codec.decode_keys(e.gamma, e.i_xi, e.i_eta, e.i_rho, s, tb, lay)
    assert np.max(np.abs(kh - ref)) < 1e-12 * np.max(np.abs(ref))
    # and the reconstruction is close to the key (relative MSE of the b-bit codec)
    rel = np.sum((kh - k) ** 2, axis=1) / np.sum(k ** 2, axis=1)
    assert np.mean(rel) < {2: 0.12, 3: 0.035, 4: 0.01}[b]


def test_decode_keys_norm_is_gamma_times_the_norm_of_the_decoded_triplets():
    """R is orthogonal and every n_hat is a unit vector, so ||k_hat||^2 =
    gamma^2 sum_i rho_hat_i^2 over the triplets that survive the padding
    (only the last one can lose coordinates)."""
    for d, b in ((64, 2), (128, 4), (256, 3)):
        lay = codec.Layout(d, b)
        tb = tables.codebooks(d, b)
        dc, _, rc, _ = (np.asarray(x, dtype=np.float64) for x in tb)
        s = tables.rotation_signs(6, d, 1)[0]
        rng = np.random.default_rng(d + b)
        n = 50
        i_xi = rng.integers(0, lay.n_dir, (n, lay.T)); i_eta = rng.integers(0, lay.n_dir, (n, lay.T))
        i_rho = rng.integers(0, lay.n_rho, (n, lay.T))
        gamma = rng.uniform(0.5, 3.0, n)
        kh = codec.decode_keys(gamma, i_xi, i_eta, i_rho, s, tb, lay)
        keep = 3 * lay.T - d                      # coordinates of the last triplet that are dropped
        last = codec.oct_inverse(dc[i_xi[:, -1]], dc[i_eta[:, -1]])[:, : 3 - keep]
        sq = np.sum(rc[i_rho[:, :-1]] ** 2, axis=1) + rc[i_rho[:, -1]] ** 2 * np.sum(last ** 2, axis=1)
        assert np.allclose(np.sum(kh ** 2, axis=1), gamma ** 2 * sq, rtol=1e-12)


# ---------------------------------------------------------------- QJL
def test_qjl_estimator_is_unbiased_over_seeds():
    """[EXPL] "optional residual correction": the sketch makes the inner-product estimate unbiased."""
    d, b = 64, 2
    lay = codec.Layout(d, b)
    tb = tables.codebooks(d, b)
    s = tables.rotation_signs(0, d, 1)[0]
    k = inputs.gaussian_keys(8, 1, 4, d)[0].astype(np.float64)
    q = inputs.normal(9, (1, d), np.float64)
    e = codec.encode(k, s, tb, lay)
    ur_hat = codec.decode_rotated(e.i_xi, e.i_eta, e.i_rho, tb, lay)
    q_rot = codec.rotate(q, s)
    exact = (q @ k.T)[0]
    base = e.gamma * (q_rot @ ur_hat.T)[0]
    ests = []
    for seed in range(2000):
        S = tables.qjl_matrix(10_000 + seed, d, 1)[0]
        bits, nu, _ = codec.qjl_encode(e.u_rot, ur_hat, S)
        ests.append(base + e.gamma * codec.qjl_correction(q_rot, bits, nu, S)[0])
    ests = np.array(ests)
    mean = ests.mean(axis=0)
    se = ests.std(axis=0) / math.sqrt(len(ests))
    assert np.all(np.abs(mean - exact) < 4 * se + 1e-12)
    # the base estimate is biased by more than the corrected one's noise for some key
    assert np.max(np.abs(base - exact)) > np.max(4 * se)
    # error shrinks like 1/sqrt(seeds)
    half = np.abs(ests[:500].mean(axis=0) - exact)
    assert np.all(half < 4 * ests.std(axis=0) / math.sqrt(500) + 1e-12)


def test_qjl_pack_round_trip():
    bits = inputs.random_codes(4, (5, 128), 2)
    w = codec.qjl_pack(bits)
    assert w.shape == (5, 4)
    assert np.array_equal(codec.qjl_unpack(w, 128), bits)
    assert int(w[0, 0]) == sum(int(bits[0, j]) << j for j in range(32))


def test_qjl_sketch_by_hand_with_a_permutation_projection():
    """[EXPL] "optional residual correction" / [SUMM] "OCTOPUS-QJL": bit j is
    the sign of row j of S applied to the residual, a zero projection counts
    as a 1, and the correction is nu sqrt(pi/2)/m <S q, 2 bits - 1>. S is a
    permutation that is not symmetric, so S e and S^T e differ."""
    S = np.zeros((4, 4))
    for j, t in enumerate((1, 3, 0, 2)):   # row j picks coordinate t
        S[j, t] = 1.0
    u_rot = np.array([[0.5, -0.25, 0.0, 0.125]])
    u_hat = np.array([[0.25, 0.0, 0.0, 0.125]])
    bits, nu, proj = codec.qjl_encode(u_rot, u_hat, S)
    # e = (0.25, -0.25, 0, 0); S e = (e1, e3, e0, e2) = (-0.25, 0, 0.25, 0)
    assert np.array_equal(proj, [[-0.25, 0.0, 0.25, 0.0]])
    assert np.array_equal(bits, [[0, 1, 1, 1]])
    assert nu[0] == pytest.approx(math.sqrt(0.125), rel=1e-15)
    q_rot = np.array([[1.0, 2.0, 3.0, 4.0]])
    # S q = (2, 4, 1, 3); signs (-1, +1, +1, +1): -2 + 4 + 1 + 3 = 6
    got = codec.qjl_correction(q_rot, bits, nu, S)
    assert got.shape == (1, 1)
    assert got[0, 0] == pytest.approx(6.0 * math.sqrt(0.125) * math.sqrt(math.pi / 2.0) / 4.0, rel=1e-15)


def test_qjl_estimator_variance_matches_closed_form():
    """For one Gaussian row s, Y = nu sqrt(pi/2) (s.q) sign(s.e) has E[Y] = q.e
    and E[Y^2] = (pi/2) nu^2 |q|^2, so the mean over m independent rows has
    variance ((pi/2) nu^2 |q|^2 - (q.e)^2) / m. A wrong scale, a dropped nu
    or a mismatched m moves the sample variance off this value."""
    d, b = 64, 2
    lay = codec.Layout(d, b)
    tb = tables.codebooks(d, b)
    s = tables.rotation_signs(1, d, 1)[0]
    k = inputs.gaussian_keys(21, 1, 3, d)[0].astype(np.float64)
    q = inputs.normal(22, (1, d), np.float64)
    e = codec.encode(k, s, tb, lay)
    ur_hat = codec.decode_rotated(e.i_xi, e.i_eta, e.i_rho, tb, lay)
    q_rot = codec.rotate(q, s)
    n_seeds = 3000
    corr = np.empty((n_seeds, k.shape[0]))
    for i in range(n_seeds):
        S = tables.qjl_matrix(50_000 + i, d, 1)[0]
        bits, nu, _ = codec.qjl_encode(e.u_rot, ur_hat, S)
        corr[i] = codec.qjl_correction(q_rot, bits, nu, S)[0]
    res = e.u_rot - ur_hat
    nu = np.linalg.norm(res, axis=1)
    qe = (q_rot @ res.T)[0]
    var = ((math.pi / 2.0) * nu ** 2 * np.sum(q_rot ** 2) - qe ** 2) / d
    # the sample variance of 3000 draws is within ~3 % (1 sigma) of the true one
    assert np.all(np.abs(corr.var(axis=0) / var - 1.0) < 0.15)
    assert np.all(np.abs(corr.mean(axis=0) - qe) < 4.0 * np.sqrt(var / n_seeds))


@pytest.mark.parametrize("b,delta", [(3, -1), (3, 0), (3, 2), (4, -1), (4, 0)])
def test_pack_round_trip_for_the_sweep_splits(b, delta):
    """Codes of another split of the bit budget (b + delta direction bits, b - delta norm bits)
    pack into c = 3b + delta bits a triplet and unpack to the same cells."""
    lay = codec.Layout(128, b, delta)
    g = inputs.rng(100 + 10 * b + delta)
    ix = g.integers(0, lay.n_dir, size=(50, lay.T))
    iy = g.integers(0, lay.n_dir, size=(50, lay.T))
    ir = g.integers(0, lay.n_rho, size=(50, lay.T))
    w = codec.pack(ix, iy, ir, lay)
    assert w.shape == (50, lay.words) and lay.code_bits == 3 * b + delta
    bx, by, br = codec.unpack(w, lay)
    assert np.array_equal(bx, ix) and np.array_equal(by, iy) and np.array_equal(br, ir)


def test_pack_by_hand_for_an_even_split():
    """b = 3, delta = 0: 3 bits per direction coordinate (magnitude 2 bits + sign), 3 for the norm,
    9 bits a triplet. Triplet 0: xi cell 5 (upper half, m = 1), eta cell 2 (lower, m = 4-1-2 = 1),
    rho 6 -> 1 | 1 << 2 | 0 << 4 | 1 << 5 | 6 << 6 = 0b110_100_101 = 421.
    Triplet 1 (cells 0, 7, rho 1): m = 3, s = 1; m = 3, s = 0 -> 3 | 3 << 2 | 1 << 4 | 0 << 5 | 1 << 6 = 95,
    at bit 9: word 0 = 421 | 95 << 9."""
    lay = codec.Layout(128, 3, 0)
    ix = np.zeros((1, lay.T), np.int64); iy = np.zeros((1, lay.T), np.int64); ir = np.zeros((1, lay.T), np.int64)
    ix[0, :2], iy[0, :2], ir[0, :2] = [5, 0], [2, 7], [6, 1]
    # the remaining triplets: cells (4, 4), rho 0 -> m = 0, s = 0: code 0
    ix[0, 2:], iy[0, 2:] = 4, 4
    w = codec.pack(ix, iy, ir, lay)
    assert int(w[0, 0]) == 421 | (95 << 9)
    assert int(w[0].astype(np.int64).sum()) == 421 | (95 << 9)
