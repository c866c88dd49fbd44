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
