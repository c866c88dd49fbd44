"""GPU parity of octo_encode against the oracle (called through the C ABI).

Both sides receive identical inputs: the same keys and the oracle's tables
rounded to float32. Codes must match bit-exactly except for mismatches at a
decision boundary (see tests/parity.py), which are counted and reported.
"""

import numpy as np
import pytest
import torch

from oracle import codec, tables
from rotation_preconditioned_quantization_b200 import api, inputs

from . import parity

pytestmark = pytest.mark.gpu

MAX_BOUNDARY_FRACTION = 1e-3


def _encode_gpu(lay, dev, keys_np, dtype, cap=None, offset=0, keys_view=None):
    H, N, d = keys_np.shape
    cap = N + offset if cap is None else cap
    kt = keys_view if keys_view is not None else torch.from_numpy(keys_np).to(dtype).cuda()
    cache = api.Cache.empty(lay, H, cap)
    api.encode(lay, dev, kt, cache, offset)
    torch.cuda.synchronize()
    words = parity.from_planar(cache.packed.cpu().numpy()[:, :, offset:offset + N], N)
    gam = cache.gamma.cpu().numpy()[:, offset:offset + N]
    out = dict(words=words, gamma=gam, cache=cache)
    if lay.qjl:
        out["qbits"] = parity.from_planar(cache.qjl_bits.cpu().numpy()[:, :, offset:offset + N], N)
        out["qnorm"] = cache.qjl_norm.cpu().numpy()[:, offset:offset + N]
    return out


def _check(keys_np, d, b, rounding, dtype, seed=0, qjl=False, cap=None, offset=0, label="",
           max_boundary_fraction=MAX_BOUNDARY_FRACTION):
    H, N, _ = keys_np.shape
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(seed, d, H)
    S = tables.qjl_matrix(seed + 1, d, H) if qjl else None
    lay = api.Layout(d, b, qjl=qjl, rounding=rounding)
    dev = api.DeviceTables(*tb, signs, S)
    g = _encode_gpu(lay, dev, keys_np, dtype, cap, offset)
    olay = codec.Layout(d, b)
    tot = dict(mis=0, bnd=0, fail=0, trip=0, qmis=0, qbnd=0, qfail=0)
    for h in range(H):
        enc = codec.encode(keys_np[h].astype(np.float64), signs[h], tb, olay, rounding)
        gam_ref = enc.gamma
        np.testing.assert_allclose(g["gamma"][h], gam_ref, rtol=1e-4, atol=0)
        m, bn, f, fails = parity.classify_codes(enc, g["words"][h], tb, olay, rounding == api.ROUND_JOINT)
        assert f == 0, f"{label} head {h}: {f} non-boundary code mismatches, e.g. {fails}"
        tot["mis"] += m; tot["bnd"] += bn; tot["trip"] += N * olay.T
        if qjl:
            ur_hat = codec.decode_rotated(enc.i_xi, enc.i_eta, enc.i_rho, tb, olay)
            bits, nu, proj = codec.qjl_encode(enc.u_rot, ur_hat, S[h])
            gx, gy, gr = codec.unpack(g["words"][h], olay)
            same = np.all((gx == enc.i_xi) & (gy == enc.i_eta) & (gr == enc.i_rho), axis=1)
            gb = codec.qjl_unpack(g["qbits"][h], d)
            e = enc.u_rot - ur_hat
            qm, qb, qf = parity.classify_qjl(proj[same], S[h], e[same], gb[same], bits[same])
            assert qf == 0, f"{label} head {h}: {qf} non-boundary sketch mismatches"
            np.testing.assert_allclose(g["qnorm"][h][same], nu[same], rtol=1e-4, atol=1e-6)
            tot["qmis"] += qm; tot["qbnd"] += qb
    assert tot["bnd"] <= max_boundary_fraction * tot["trip"]
    print(f"\n[encode parity] {label} d={d} b={b} round={'J' if rounding else 'S'} {dtype}: "
          f"{tot['trip']} triplets, {tot['mis']} mismatches, all at a boundary ({tot['bnd']})"
          + (f"; sketch bits {tot['qmis']} mismatches ({tot['qbnd']} at a boundary)" if qjl else ""))
    return g, tot


def test_encode_single_head_4096_keys_b3(cuda_ok):
    """One head, d=128, 4096 fp32 N(0,1) keys, seed 0, b=3, joint rounding."""
    k = inputs.gaussian_keys(0, 1, 4096, 128)
    _check(k, 128, 3, api.ROUND_JOINT, torch.float32, seed=0, label="single-head")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [2, 3, 4])
@pytest.mark.parametrize("rounding", [api.ROUND_SCALAR, api.ROUND_JOINT])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_encode_shapes(cuda_ok, d, b, rounding, dtype):
    k = inputs.llm_keys(10 * d + b, 3, 301, d)
    if dtype == torch.bfloat16:
        k = inputs.to_bf16(k)
    _check(k, d, b, rounding, dtype, seed=d + b, label="shapes")


@pytest.mark.parametrize("d,b", [(128, 4), (64, 2), (256, 3)])
def test_encode_qjl(cuda_ok, d, b):
    k = inputs.to_bf16(inputs.llm_keys(5, 2, 257, d))
    _check(k, d, b, api.ROUND_JOINT, torch.bfloat16, seed=3, qjl=True, label="qjl")


def test_encode_appends_match_one_shot(cuda_ok):
    d, b, H, N = 128, 3, 2, 4500
    k = inputs.to_bf16(inputs.llm_keys(21, H, N, d))
    tb = parity.oracle_tables(d, b)
    lay = api.Layout(d, b)
    dev = api.DeviceTables(*tb, tables.rotation_signs(1, d, H))
    kt = torch.from_numpy(k).to(torch.bfloat16).cuda()
    one = api.Cache.empty(lay, H, N + 7)
    api.encode(lay, dev, kt, one, 7)
    app = api.Cache.empty(lay, H, N + 7)
    app.length = 7
    for n in inputs.append_lengths(3, N, 1, 4096):
        s = app.length - 7
        api.encode(lay, dev, kt[:, s:s + n], app)
    torch.cuda.synchronize()
    assert app.length == N + 7
    assert torch.equal(one.packed, app.packed) and torch.equal(one.gamma, app.gamma)
    # untouched prefix stays zero
    assert int(one.packed[:, :, :7].abs().sum()) == 0


def test_encode_strided_keys_and_offset(cuda_ok):
    d, b, H, N = 64, 3, 3, 200
    big = inputs.llm_keys(7, H, 2 * N, 2 * d)            # keys are a strided view of a bigger tensor
    view = torch.from_numpy(big).cuda()[:, ::2, d:]
    k = np.ascontiguousarray(big[:, ::2, d:])
    tb = parity.oracle_tables(d, b)
    lay = api.Layout(d, b)
    signs = tables.rotation_signs(4, d, H)
    dev = api.DeviceTables(*tb, signs)
    g = _encode_gpu(lay, dev, k, torch.float32, cap=N + 50, offset=33, keys_view=view)
    olay = codec.Layout(d, b)
    for h in range(H):
        enc = codec.encode(k[h].astype(np.float64), signs[h], tb, olay)
        m, bn, f, _ = parity.classify_codes(enc, g["words"][h], tb, olay, True)
        assert f == 0


def test_encode_special_keys(cuda_ok):
    d, b = 128, 3
    k = np.zeros((1, 6, d), np.float32)
    k[0, 1, 5] = 1.0                                   # one-hot
    k[0, 2] = 1e-10 * inputs.normal(1, d)              # tiny
    k[0, 3] = 1e10 * inputs.normal(2, d)               # huge
    k[0, 4] = -1.0                                     # constant
    k[0, 5, ::3] = 2.0                                 # sparse
    # structured keys put many values exactly on ties (equal-magnitude rotated
    # coordinates), so boundary cases are frequent here; failures must still be zero
    g, _ = _check(k, d, b, api.ROUND_JOINT, torch.float32, seed=9, label="special", max_boundary_fraction=1.0)
    assert g["gamma"][0, 0] == 0.0
    # zero key -> every triplet is the zero triplet: centre cell, lowest rho level
    lay = codec.Layout(d, b)
    ix, iy, ir = codec.unpack(g["words"][0, :1], lay)
    assert np.all(ix == lay.n_dir // 2) and np.all(iy == lay.n_dir // 2) and np.all(ir == 0)


def test_encode_llm_prefill_full_size(cuda_ok):
    """Full LLM-shaped prefill: 8 KV heads x 32768 bf16 keys, d=128, b=3, joint."""
    k = inputs.to_bf16(inputs.llm_keys(2, 8, 32768, 128))
    _check(k, 128, 3, api.ROUND_JOINT, torch.bfloat16, seed=0, label="llm-prefill-full")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [2, 3, 4])
def test_encode_sweep_appends(cuda_ok, d, b):
    """Encode sweep: 4 heads x 2^18 fp32 keys ~ N(0,1) (2^20 keys) streamed in appends of
    1-4096 tokens, seeded rotation per head. The appended cache equals a one-shot encode
    bit for bit, and 512 sampled tokens per head match the oracle (boundary cases counted)."""
    H, N = 4, 1 << 18
    k = inputs.gaussian_keys(1000 + 10 * d + b, H, N, d)
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(d * 7 + b, d, H)
    lay = api.Layout(d, b)
    dev = api.DeviceTables(*tb, signs)
    kt = torch.from_numpy(k).cuda()
    app = api.Cache.empty(lay, H, N)
    for n in inputs.append_lengths(d + b, N, 1, 4096):
        s = app.length
        api.encode(lay, dev, kt[:, s:s + n], app)
    one = api.Cache.empty(lay, H, N)
    api.encode(lay, dev, kt, one, 0)
    torch.cuda.synchronize()
    assert app.length == N
    assert torch.equal(one.packed, app.packed) and torch.equal(one.gamma, app.gamma)
    olay = codec.Layout(d, b)
    rng = np.random.default_rng(d * 10 + b)
    tot = dict(mis=0, bnd=0, trip=0)
    for h in range(H):
        idx = np.sort(rng.choice(N, 512, replace=False))
        enc = codec.encode(k[h, idx].astype(np.float64), signs[h], tb, olay)
        words = parity.from_planar(app.packed[h:h + 1].cpu().numpy(), N)[0][idx]
        gam = app.gamma[h].cpu().numpy()[idx]
        np.testing.assert_allclose(gam, enc.gamma, rtol=1e-4, atol=0)
        m, bn, f, fails = parity.classify_codes(enc, words, tb, olay, True)
        assert f == 0, f"head {h}: {f} non-boundary code mismatches, e.g. {fails}"
        tot["mis"] += m; tot["bnd"] += bn; tot["trip"] += len(idx) * olay.T
    assert tot["bnd"] <= MAX_BOUNDARY_FRACTION * tot["trip"]
    print(f"\n[encode sweep] d={d} b={b}: {H}x{N} keys appended; sampled {tot['trip']} triplets, "
          f"{tot['mis']} mismatches, all at a boundary ({tot['bnd']})")
