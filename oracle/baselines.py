"""Oracle: the per-coordinate rotation codec the pages compare against (test infrastructure only).

TurboQuant-MSE style ([EXPL] "rotation": after a random rotation every
coordinate follows a symmetric Beta law, and a per-coordinate optimal
scalar quantiser is built for it). Used only as the quality comparator of
the "lower MSE than a per-coordinate Lloyd-Max codec at the same bits" pin
([EXPL] "experimental results").
"""

from __future__ import annotations

import functools
import math

import numpy as np

from . import codec, tables


def coordinate_density(x, d: int) -> np.ndarray:
    """Density of one coordinate of a uniform unit vector in R^d.

    (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2) on [-1, 1]: (x+1)/2 is
    Beta((d-1)/2, (d-1)/2), the symmetric Beta law of the explainer.
    """
    x = np.asarray(x, dtype=np.float64)
    a = b = 0.5 * (d - 1)
    lbeta = math.lgamma(a) + math.lgamma(b) - math.lgamma(a + b)
    one = np.clip(1.0 - x * x, 0.0, None)
    return one ** (0.5 * (d - 3)) * math.exp(-lbeta) / 2.0 ** (d - 2)


@functools.lru_cache(maxsize=None)
def coordinate_codebook(d: int, bits: int):
    """Lloyd-Max codebook of 2^bits levels for coordinate_density."""
    c, t, _ = tables.lloyd_max(lambda x: coordinate_density(x, d), -1.0, 1.0, 1 << bits,
                               tol=1e-13, n_nodes=32, max_width=1.0 / 64)
    c = 0.5 * (c - c[::-1])
    return c, 0.5 * (c[:-1] + c[1:])


def per_coordinate_mse(u: np.ndarray, signs: np.ndarray, bits: int) -> float:
    """Mean ||u - u_hat||^2 over unit rows u when every rotated coordinate is
    Lloyd-Max quantised with ``bits`` bits and rotated back."""
    d = u.shape[-1]
    c, t = coordinate_codebook(d, bits)
    ur = codec.rotate(u, signs)
    q = c[codec.scalar_index(ur, t)]
    uh = q @ codec.rotation_matrix(signs)
    return float(np.mean(np.sum((u - uh) ** 2, axis=-1)))
