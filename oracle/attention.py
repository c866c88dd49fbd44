"""Oracle: logits and decode attention over an OCTOPUS-coded key cache (test infrastructure only).

The oracle deliberately takes the MATERIALISED route: it rebuilds every key
k_hat = gamma * R^T u_rot_hat and forms q . k_hat. The CUDA path takes the
pages' route instead ([EXPL] "engineering implementation", [ABS]: keys are
never materialised; the query is rotated once and dotted with the decoded
rotated direction). The two agree because R is orthogonal.

Attention is plain softmax(scale * q K^T) V in float64, with V the bf16
values upcast exactly.
"""

from __future__ import annotations

import math

import numpy as np

from . import codec


def logits(q: np.ndarray, gamma, i_xi, i_eta, i_rho, signs, tables, lay: codec.Layout,
           qjl=None) -> np.ndarray:
    """Raw logits q . k_hat for ONE kv head.

    q: [G, d] queries sharing this kv head; codes [N, T]; gamma [N].
    qjl: optional (bits [N, d], nu [N], S [d, d]) adding the OCTOPUS-QJL term
    gamma * nu * sqrt(pi/2)/m * <S R q, 2 bits - 1> ([EXPL] "optional residual
    correction").
    Returns [G, N].
    """
    kh = codec.decode_keys(gamma, i_xi, i_eta, i_rho, signs, tables, lay)   # [N, d]
    q = np.asarray(q, dtype=np.float64)
    out = q @ kh.T
    if qjl is not None:
        bits, nu, S = qjl
        q_rot = codec.rotate(q, signs)
        out = out + np.asarray(gamma, dtype=np.float64)[None, :] * codec.qjl_correction(q_rot, bits, nu, S)
    return out


def softmax_attention(lg: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * lg) @ V, rows of lg [G, N], V [N, d] -> [G, d]."""
    z = scale * np.asarray(lg, dtype=np.float64)
    z = z - np.max(z, axis=-1, keepdims=True)
    p = np.exp(z)
    p = p / np.sum(p, axis=-1, keepdims=True)
    return p @ np.asarray(V, dtype=np.float64)


def decode_attention(q, gamma, i_xi, i_eta, i_rho, V, signs, tables, lay: codec.Layout,
                     scale=None, qjl=None):
    """One decode-attention step for ONE kv head: returns (out [G, d], logits [G, N]).

    scale defaults to 1/sqrt(d) (reading: the usual attention temperature
    with the real head dimension).
    """
    if scale is None:
        scale = 1.0 / math.sqrt(lay.d)
    lg = logits(q, gamma, i_xi, i_eta, i_rho, signs, tables, lay, qjl)
    return softmax_attention(lg, V, scale), lg
