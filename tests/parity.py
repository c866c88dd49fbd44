"""Helpers shared by the GPU parity tests: run the oracle on the same inputs,
classify index mismatches, and convert between the oracle's per-key words and
the library's word-planar cache layout.

Parity rules (the workload statement's tolerances):
* packed indices bit-exact, except mismatches whose decision was within 1e-6
  of a boundary; those are counted and reported. A triplet mismatch counts as
  "at the boundary" if (a) one of the values the decision compares (xi, eta;
  rho for scalar rounding; s = n_hat . t for the joint rho choice) is within
  1e-6 of a threshold, or (b) under joint rounding the GPU's chosen code has
  a squared error within 1e-6 * max(rho^2, 1e-30) of the oracle's (both
  errors recomputed in float64 from the oracle's triplet). Any other
  mismatch is a failure.
* gamma within 1e-4 relative; raw logits within 1e-4 * gamma * ||q||;
  attention outputs within 2e-3 * max |o_ref| of their row.
"""

from __future__ import annotations

import numpy as np

from oracle import codec, tables

BOUNDARY = 1e-6


def oracle_tables(d, b):
    """Oracle codebooks rounded to float32 (the values both sides receive)."""
    return tables.as_f32(*tables.codebooks(d, b))


def to_planar(words: np.ndarray) -> np.ndarray:
    """[H][N][W] uint32 -> [H][W][N] (the cache layout)."""
    return np.ascontiguousarray(np.swapaxes(words, -1, -2))


def from_planar(packed: np.ndarray, n: int) -> np.ndarray:
    """[H][W][cap] (any int dtype) -> [H][n][W] uint32."""
    p = np.asarray(packed)[..., :n].astype(np.int64) & 0xFFFFFFFF
    return np.ascontiguousarray(np.swapaxes(p, -1, -2)).astype(np.uint32)


def classify_codes(enc: codec.Encoded, gpu_words: np.ndarray, tb, lay: codec.Layout, joint: bool):
    """Compare the GPU's words [N][W] with the oracle encoding of the same keys.

    Returns (n_mismatch, n_boundary, n_fail, details) over triplets.
    """
    dc, dt, rc, rt = (np.asarray(x, dtype=np.float64) for x in tb)
    gx, gy, gr = codec.unpack(gpu_words, lay)
    mis = (gx != enc.i_xi) | (gy != enc.i_eta) | (gr != enc.i_rho)
    idx = np.nonzero(mis)
    n_mis = int(mis.sum())
    if n_mis == 0:
        return 0, 0, 0, []
    t = enc.t[idx]
    xi, eta, rho = enc.xi[idx], enc.eta[idx], enc.rho[idx]
    near = lambda v, th: np.min(np.abs(v[:, None] - th[None, :]), axis=1) <= BOUNDARY if len(th) else np.zeros(len(v), bool)
    bnd = near(xi, dt) | near(eta, dt)
    nh_o = codec.oct_inverse(dc[enc.i_xi[idx]], dc[enc.i_eta[idx]])
    if joint:
        s_o = np.sum(nh_o * t, axis=-1)
        bnd |= near(s_o, rt)
        nh_g = codec.oct_inverse(dc[gx[idx]], dc[gy[idx]])
        e_g = np.sum((t - rc[gr[idx]][:, None] * nh_g) ** 2, axis=-1)
        e_o = np.sum((t - rc[enc.i_rho[idx]][:, None] * nh_o) ** 2, axis=-1)
        bnd |= np.abs(e_g - e_o) <= BOUNDARY * np.maximum(rho ** 2, 1e-30)
    else:
        bnd |= near(rho, rt)
    n_b = int(bnd.sum())
    fails = [(tuple(int(v[k]) for v in idx), int(gx[idx][k]), int(gy[idx][k]), int(gr[idx][k]),
              int(enc.i_xi[idx][k]), int(enc.i_eta[idx][k]), int(enc.i_rho[idx][k]))
             for k in np.nonzero(~bnd)[0][:10]]
    return n_mis, n_b, n_mis - n_b, fails


def classify_qjl(proj: np.ndarray, S: np.ndarray, e: np.ndarray, gpu_bits: np.ndarray, ora_bits: np.ndarray):
    """Sketch bits [N][d]: a mismatch is at the boundary when |(S e)_j| <= 1e-6 * sum_m |S_jm e_m|."""
    mis = gpu_bits != ora_bits
    scale = np.abs(e) @ np.abs(S).T
    bnd = mis & (np.abs(proj) <= BOUNDARY * np.maximum(scale, 1e-30))
    return int(mis.sum()), int(bnd.sum()), int((mis & ~bnd).sum())
