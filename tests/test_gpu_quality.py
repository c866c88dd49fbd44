"""GPU tests of the quality probe (the explainer's synthetic test and needle
test, run through the library's encode, key reconstruction and fused decode
kernels) against the oracle on the same inputs, and against the printed
values where the pages give them."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention, codec, tables
from rotation_preconditioned_quantization_b200 import inputs, quality

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden", "synthetic_quality.json")


def _oracle_mse(rep, b, d=128, n=1024, seed=0):
    """The oracle's MSE of the unit direction for the probe's repetition rep."""
    lay = codec.Layout(d, b)
    tb = tables.codebooks(d, b)
    k = inputs.gaussian_keys(seed + 1000 + rep, 1, n, d)[0].astype(np.float64)
    s = tables.rotation_signs(seed + rep, d, 1)[0]
    e = codec.encode(k, s, tables.as_f32(*tb), lay)
    u = k / np.linalg.norm(k, axis=1, keepdims=True)
    uh = codec.decode_keys(np.ones(n), e.i_xi, e.i_eta, e.i_rho, s, tables.as_f32(*tb), lay)
    return float(np.mean(np.sum((u - uh) ** 2, axis=1)))


@pytest.mark.parametrize("b", [2, 3, 4])
def test_synthetic_probe_matches_oracle(cuda_ok, b):
    r = quality.synthetic_probe(b, reps=2)
    for rep, m in enumerate(r["mse_per_rep"]):
        ref = _oracle_mse(rep, b)
        # the GPU encodes in fp32: a decision within rounding of a threshold may flip a code
        assert abs(m - ref) <= 2e-3 * ref, (rep, m, ref)
    assert 0.0 < r["ip_err"] and 0.9 < r["cosine"] < 1.0


def test_synthetic_probe_reproduces_printed_mse(cuda_ok):
    printed = json.load(open(GOLD))["mse"]
    for b in (2, 4):
        m = quality.synthetic_probe(b, reps=16)["mse"]
        assert abs(m - printed[f"octopus_b{b}"]) < 0.10 * printed[f"octopus_b{b}"], (b, m)


@pytest.mark.parametrize("b", [2, 4])
def test_needle_probe_matches_oracle(cuda_ok, b):
    d, n_dis, reps = 128, 2048, 2
    r = quality.needle_probe(b, reps=reps, n_distractors=n_dis)
    lay = codec.Layout(d, b)
    tb = tables.as_f32(*tables.codebooks(d, b))
    n = n_dis + 1
    for rep in range(reps):
        q = inputs.normal(7000 + rep, (d,)).astype(np.float64)
        keys = inputs.normal(9000 + rep, (1, n, d))[0].astype(np.float64)
        pos = int(inputs.rng(11000 + rep).integers(n))
        keys[pos] = q.astype(np.float32)
        s = tables.rotation_signs(rep, d, 1)[0]
        e = codec.encode(keys, s, tb, lay)
        lg = attention.logits(q[None], e.gamma, e.i_xi, e.i_eta, e.i_rho, s, tb, lay)[0] / math.sqrt(d)
        p = np.exp(lg - lg.max())
        ref = p[pos] / p.sum()
        assert abs(r["mass_per_rep"][rep] - ref) <= 1e-2 * ref, (rep, r["mass_per_rep"][rep], ref)
    assert 0.0 < r["needle_mass"] <= 1.0 and 0.0 < r["needle_mass_exact_keys"] <= 1.0


def _oracle_sweep_codebooks(d, b, delta):
    """Lloyd-Max codebooks of the split (b + delta, b - delta), rounded to fp32 (both sides get them)."""
    dc, dt = tables.direction_codebook_levels(1 << (b + delta), 1e-9)
    rc, rt = tables.rho_codebook_levels(d, 1 << (b - delta), 1e-9)
    return tables.as_f32(dc, dt, rc, rt)


def _oracle_mse_split(rep, b, delta, cb, d=128, n=1024, seed=0):
    lay = codec.Layout(d, b, delta)
    k = inputs.gaussian_keys(seed + 1000 + rep, 1, n, d)[0].astype(np.float64)
    s = tables.rotation_signs(seed + rep, d, 1)[0]
    e = codec.encode(k, s, cb, lay)
    u = k / np.linalg.norm(k, axis=1, keepdims=True)
    uh = codec.decode_keys(np.ones(n), e.i_xi, e.i_eta, e.i_rho, s, cb, lay)
    return float(np.mean(np.sum((u - uh) ** 2, axis=1)))


@pytest.mark.parametrize("b,delta", [(3, -1), (3, 0), (3, 2), (4, -1), (4, 0)])
def test_bit_allocation_split_matches_oracle(cuda_ok, b, delta):
    """Each sweep split through the encode and key reconstruction kernels, per repetition, against
    the oracle on the same keys, signs and fp32 codebooks."""
    cb = _oracle_sweep_codebooks(128, b, delta)
    r = quality.synthetic_probe(b, reps=2, delta=delta, codebooks=cb)
    for rep, m in enumerate(r["mse_per_rep"]):
        ref = _oracle_mse_split(rep, b, delta, cb)
        assert abs(m - ref) <= 2e-3 * ref, (rep, m, ref)


def test_bit_allocation_sweep_reproduces_the_printed_ranking(cuda_ok):
    """[EXPL] "non-uniform bit allocation": delta = +1 is best; against delta = 0 it gains 31-41 %,
    delta = -1 loses more than 200 % and delta = +2 loses 44-73 % (b = 3; the page's ranges, +-10 points)."""
    g = json.load(open(GOLD))["delta_sweep"]
    r = quality.bit_allocation_sweep(3, (-1, 0, 1, 2), reps=16)
    ch = r["change_vs_delta0_percent"]
    assert r["best_delta"] == g["best_delta"]
    lo, hi = g["gain_delta_plus1_vs_0_percent"]
    assert lo - 10 <= -ch["1"] <= hi + 10, ch
    assert ch["-1"] > g["loss_delta_minus1_vs_0_percent_min"], ch
    lo, hi = g["loss_delta_plus2_vs_0_percent"]
    assert lo - 10 <= ch["2"] <= hi + 10, ch
    r4 = quality.bit_allocation_sweep(4, (-1, 0, 1), reps=8)
    assert r4["best_delta"] == 1 and r4["change_vs_delta0_percent"]["-1"] > g["loss_delta_minus1_vs_0_percent_min"]
