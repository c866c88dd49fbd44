"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module only draws random numbers (numpy PCG64). It holds none of the
codec's arithmetic: no rotation, no triplet split, no quantisation. Both the
CUDA path and the CPU oracle receive the arrays it returns, so a parity test
compares the two on identical inputs.

Workload recipes (synthetic stand-ins for the workload classes the OCTOPUS
pages evaluate on; the pages' own models and datasets are not available):

* ``gaussian_keys``: iid N(0, 1) keys, as in the pages' synthetic probe
  (OCTOPUS explainer, "experimental results": isotropic Gaussian keys, d=128).
* ``llm_keys``: LLM-shaped keys. N(0, 1) entries, four channels chosen once
  without replacement and scaled by 10 (outlier channels), and every key scaled
  by a per-token factor drawn from lognormal(0, 0.5).
* ``normal``: plain N(0, 1) draws for queries and values.

``device_normal`` and ``device_llm_keys`` draw the same distributions with
torch's seeded generator directly in device memory, for workloads too large
to draw on the host (the benchmark's long-context cache); they follow the
same recipes but not the same numbers as their numpy counterparts.

``to_bf16`` rounds float32 to bfloat16 (round to nearest even) and returns
float32 arrays holding the bf16 values, so that numpy code sees exactly the
numbers a bf16 device buffer holds.
"""

from __future__ import annotations

import numpy as np

__all__ = ["rng", "normal", "gaussian_keys", "llm_keys", "to_bf16", "bf16_bits",
           "random_codes", "append_lengths", "device_normal", "device_llm_keys"]


def rng(seed: int) -> np.random.Generator:
    """numpy PCG64 generator for ``seed``."""
    return np.random.Generator(np.random.PCG64(seed))


def normal(seed: int, shape, dtype=np.float32) -> np.ndarray:
    """iid N(0, 1) draws of ``shape``."""
    return rng(seed).standard_normal(size=shape, dtype=np.float64).astype(dtype)


def gaussian_keys(seed: int, n_heads: int, n_tokens: int, d: int) -> np.ndarray:
    """[n_heads][n_tokens][d] float32 keys, iid N(0, 1)."""
    return normal(seed, (n_heads, n_tokens, d), np.float32)


def llm_keys(seed: int, n_heads: int, n_tokens: int, d: int,
             n_outlier: int = 4, outlier_scale: float = 10.0,
             lognormal_sigma: float = 0.5) -> np.ndarray:
    """[n_heads][n_tokens][d] float32 LLM-shaped keys (see module docstring)."""
    g = rng(seed)
    k = g.standard_normal(size=(n_heads, n_tokens, d), dtype=np.float64)
    ch = g.choice(d, size=n_outlier, replace=False)
    k[:, :, ch] *= outlier_scale
    k *= g.lognormal(mean=0.0, sigma=lognormal_sigma, size=(n_heads, n_tokens, 1))
    return k.astype(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of float32 ``x``, round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    nan = np.isnan(x)
    r = np.where(nan, 0x7FC0, r)
    return r.astype(np.uint16)


def to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 array holding ``x`` rounded to bfloat16."""
    b = bf16_bits(x).astype(np.uint32) << 16
    return b.view(np.float32).reshape(np.shape(x))


def random_codes(seed: int, shape, n_levels: int) -> np.ndarray:
    """Uniform integer draws in [0, n_levels), int64."""
    return rng(seed).integers(0, n_levels, size=shape, dtype=np.int64)


def append_lengths(seed: int, total: int, lo: int = 1, hi: int = 4096) -> list[int]:
    """Append sizes n ~ U{lo..hi} that sum to exactly ``total`` (last one cut)."""
    g = rng(seed)
    out, acc = [], 0
    while acc < total:
        n = int(g.integers(lo, hi + 1))
        n = min(n, total - acc)
        out.append(n)
        acc += n
    return out


def device_normal(seed: int, shape, device, dtype=None):
    """iid N(0, 1) draws of ``shape`` made on ``device`` (torch generator seeded
    with ``seed``), cast to ``dtype`` (default bfloat16) by torch's rounding."""
    import torch

    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16 if dtype is None else dtype)


def device_llm_keys(seed: int, n_heads: int, n_tokens: int, d: int, device, dtype=None,
                    n_outlier: int = 4, outlier_scale: float = 10.0, lognormal_sigma: float = 0.5):
    """[n_heads][n_tokens][d] LLM-shaped keys drawn on ``device`` (recipe of
    ``llm_keys``: N(0, 1) entries, ``n_outlier`` channels chosen once without
    replacement and scaled by ``outlier_scale``, every key scaled by a
    per-token lognormal(0, ``lognormal_sigma``) factor), cast to ``dtype``
    (default bfloat16). Drawn one head at a time, so the float32 temporary
    is a single head."""
    import torch

    dt = torch.bfloat16 if dtype is None else dtype
    g = torch.Generator(device=device).manual_seed(seed)
    ch = torch.from_numpy(rng(seed).choice(d, size=n_outlier, replace=False)).to(device)
    out = torch.empty((n_heads, n_tokens, d), dtype=dt, device=device)
    for h in range(n_heads):
        k = torch.randn((n_tokens, d), generator=g, device=device, dtype=torch.float32)
        k[:, ch] *= outlier_scale
        f = torch.empty((n_tokens, 1), device=device, dtype=torch.float32).log_normal_(0.0, lognormal_sigma, generator=g)
        out[h] = (k * f).to(dt)
    return out
