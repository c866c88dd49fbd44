"""Quality probe of the codec on the GPU: the explainer's synthetic test
("experimental results": d = 128 isotropic Gaussian keys, 1024 keys and 16
queries per repetition, 64 repetitions) and its needle test (one target key
among 2048 random distractors, softmax mass on the target).

Every codec step runs in the library's kernels: the keys are encoded by
``octo_encode``, reconstructed by ``octo_dequant`` and attended over by
``octo_decode_attn``; torch only draws the inputs and reduces the errors.

Readings (the pages name the metrics but not their formulas):
* MSE: mean over keys of ||u - u_hat||^2 for the unit direction u = k/||k||
  and its reconstruction u_hat = k_hat / gamma (the norm gamma is stored in
  fp32 and is not part of the error). This is the reading under which the
  pages' printed values are reproduced.
* cosine: mean over keys of cos(k, k_hat).
* inner-product error: mean over (query, key) of (<q, u> - <q, u_hat>)^2
  with q ~ N(0, I_d).
* needle: keys are 2048 distractors ~ N(0, I_d) plus the needle k* = q for a
  query q ~ N(0, I_d); the mass is the softmax weight of k* at scale 1/sqrt(d)
  (the pages do not state the temperature). It is read off the decode's
  attention output with a value row that is one-hot on the needle.

The bit-allocation sweep ("non-uniform bit allocation": direction b + delta
bits per coordinate, norm b - delta) runs the synthetic probe for each split.

Usage: ``python -m rotation_preconditioned_quantization_b200.quality``
prints one JSON line per bit budget, then one per sweep.
"""

from __future__ import annotations

import json
import math

import numpy as np
import torch

from . import api, inputs


def _tables(lay: api.Layout, seed: int, device, codebooks=None):
    dc, dt, rc, rt = api.codebook_build(lay) if codebooks is None else codebooks
    return api.DeviceTables(dc, dt, rc, rt, api.rotation_build(seed, lay.d, 1), device=device)


def synthetic_probe(b: int, reps: int = 64, n_keys: int = 1024, n_queries: int = 16, d: int = 128, seed: int = 0,
                    device="cuda", delta: int = 1, codebooks=None) -> dict:
    """MSE, cosine and inner-product error of the codec on Gaussian keys (one head per repetition,
    its own rotation seed); returns the means over the repetitions and the per-repetition MSEs.
    delta selects the split of the bit budget (b + delta direction bits, b - delta norm bits);
    codebooks (dir_c, dir_t, rho_c, rho_t) default to the library's host builder."""
    lay = api.Layout(d, b, delta=delta)
    if codebooks is None:
        codebooks = api.codebook_build(lay)  # once: they depend only on d and the split
    mses, coss, ips = [], [], []
    for rep in range(reps):
        k = torch.from_numpy(inputs.gaussian_keys(seed + 1000 + rep, 1, n_keys, d)).to(device)   # [1][n][d] fp32
        q = torch.from_numpy(inputs.normal(seed + 5000 + rep, (n_queries, d))).to(device)
        tabs = _tables(lay, seed + rep, device, codebooks)
        cache = api.Cache.empty(lay, 1, n_keys, device)
        api.encode(lay, tabs, k, cache, 0)
        kh = api.dequant(lay, tabs, cache)[0].double()
        k0 = k[0].double()
        u = k0 / k0.norm(dim=1, keepdim=True)
        uh = kh / cache.gamma[0, :n_keys].double()[:, None]
        mses.append(float(((u - uh) ** 2).sum(1).mean()))
        coss.append(float(torch.nn.functional.cosine_similarity(k0, kh, dim=1).mean()))
        qd = q.double()
        ips.append(float(((qd @ u.T - qd @ uh.T) ** 2).mean()))
    return {"b": b, "delta": delta, "d": d, "reps": reps, "keys": n_keys, "queries": n_queries,
            "mse": float(np.mean(mses)), "cosine": float(np.mean(coss)), "ip_err": float(np.mean(ips)),
            "mse_per_rep": mses}


def bit_allocation_sweep(b: int, deltas=(-1, 0, 1, 2), reps: int = 64, d: int = 128, seed: int = 0,
                         device="cuda") -> dict:
    """The explainer's bit-allocation sweep ("non-uniform bit allocation"):
    the synthetic probe's MSE with b + delta bits per direction coordinate
    and b - delta for the norm, each split with its own Lloyd-Max codebooks,
    through the encode and key reconstruction kernels. Returns the MSE per
    delta, the best delta and each delta's MSE change against delta = 0 in
    percent."""
    mse = {dl: synthetic_probe(b, reps=reps, d=d, seed=seed, device=device, delta=dl)["mse"] for dl in deltas}
    out = {"b": b, "d": d, "reps": reps, "mse": {str(k): v for k, v in mse.items()},
           "best_delta": min(mse, key=mse.get)}
    if 0 in mse:
        out["change_vs_delta0_percent"] = {str(k): 100.0 * (v / mse[0] - 1.0) for k, v in mse.items()}
    return out


def needle_probe(b: int, reps: int = 64, n_distractors: int = 2048, d: int = 128, seed: int = 0,
                 device="cuda") -> dict:
    """Softmax mass on the needle through the fused decode, and the same mass with the exact keys."""
    lay = api.Layout(d, b)
    n = n_distractors + 1
    mass, exact = [], []
    for rep in range(reps):
        q = torch.from_numpy(inputs.normal(seed + 7000 + rep, (d,))).to(device)
        keys = torch.from_numpy(inputs.normal(seed + 9000 + rep, (1, n, d))).to(device)
        pos = int(inputs.rng(seed + 11000 + rep).integers(n))
        keys[0, pos] = q
        tabs = _tables(lay, seed + rep, device)
        cache = api.Cache.empty(lay, 1, n, device)
        V = torch.zeros((1, cache.cap, d), dtype=torch.bfloat16, device=device)  # rows follow the cache capacity
        V[0, pos, 0] = 1.0
        api.encode(lay, tabs, keys, cache, 0)
        out, _ = api.decode_attn(lay, tabs, q.view(1, 1, 1, d), cache, V, 1)
        mass.append(float(out[0, 0, 0, 0]))
        lg = (keys[0].double() @ q.double()) / math.sqrt(d)
        exact.append(float(torch.softmax(lg, 0)[pos]))
    return {"b": b, "d": d, "reps": reps, "distractors": n_distractors, "scale": "1/sqrt(d)",
            "needle_mass": float(np.mean(mass)), "needle_mass_exact_keys": float(np.mean(exact)),
            "mass_per_rep": mass}


# Splits the encode and key reconstruction kernels are built for at d = 128
# (besides the OCTOPUS delta = +1 at every b).
SWEEP_DELTAS = {3: (-1, 0, 1, 2), 4: (-1, 0, 1)}


def main():
    dev = torch.device("cuda", 0)
    for b in (2, 3, 4):
        s = synthetic_probe(b, device=dev)
        nd = needle_probe(b, device=dev)
        s.pop("mse_per_rep")
        nd.pop("mass_per_rep")
        print(json.dumps({**s, **{k: v for k, v in nd.items() if k.startswith("needle") or k == "distractors"}}))
    for b, deltas in SWEEP_DELTAS.items():
        print(json.dumps({"bit_allocation_sweep": bit_allocation_sweep(b, deltas, device=dev)}))


if __name__ == "__main__":
    main()
