"""MultiScaleRetention layer pieces of the oracle, numpy fp64 -- TEST
INFRASTRUCTURE ONLY (see the package docstring).

Follows "Hybrid Architectures: RetNet and the Three Computation Paradigms"
section 9.1 (MSR(X) = (swish(X W_G) (.) Y) W_O, Y = GroupNorm_h(heads)),
section 8.4 (GroupNorm with one group per head) and the RetNet paper summary's
"Gated Multi-Scale Retention" section (W_V and W_G widen to 2d, W_O maps 2d
back to d).  Matrix products use numpy's fp64 matmul as a library step.
"""
from __future__ import annotations

import numpy as np

from . import retention_recurrent, xpos_rotate


def swish(x):
    """swish(x) = x * sigmoid(x)  (P1 section 9.1)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def group_norm_heads(y, eps: float):
    """Per-(token, head) normalisation over the head's d_v channels, biased
    variance, eps inside the square root, no affine term (P1 section 8.4:
    each head normalised by its own mean and variance).  y [..., H, dv]."""
    y = np.asarray(y, dtype=np.float64)
    mu = y.mean(axis=-1, keepdims=True)
    var = ((y - mu) ** 2).mean(axis=-1, keepdims=True)
    return (y - mu) / np.sqrt(var + eps)


def project(x, w):
    """x [..., d_in] @ w [d_in, d_out] in fp64."""
    return np.asarray(x, np.float64) @ np.asarray(w, np.float64)


def msr_forward(x, wq, wk, wv, wg, wo, gammas, H: int, k_scale: float, eps: float,
                theta_base: float = 10000.0, heads=None, return_parts: bool = False):
    """MSR(X) for X [B, N, d_model]:
        Q = rot(X W_Q), K = rot(k_scale * X W_K), V = X W_V, G = X W_G
        heads = retention(Q, K, V, gamma_h)           (recurrent definition)
        Y = GroupNorm_h(heads);  Z = swish(G) (.) Y;  out = Z W_O
    ``heads`` (optional list of head indices) restricts the retention and
    GroupNorm to those heads and skips W_O (used to sample large layers);
    then the function returns Y restricted to those heads and the gate for
    them."""
    x = np.asarray(x, np.float64)
    B, N, dm = x.shape
    dk = wq.shape[1] // H
    dv = wv.shape[1] // H
    hs = list(range(H)) if heads is None else list(heads)
    cols_k = np.concatenate([np.arange(h * dk, (h + 1) * dk) for h in hs])
    cols_v = np.concatenate([np.arange(h * dv, (h + 1) * dv) for h in hs])
    q = project(x, np.asarray(wq, np.float64)[:, cols_k]).reshape(B, N, len(hs), dk)
    k = project(x, np.asarray(wk, np.float64)[:, cols_k]).reshape(B, N, len(hs), dk) * k_scale
    v = project(x, np.asarray(wv, np.float64)[:, cols_v]).reshape(B, N, len(hs), dv)
    g = project(x, np.asarray(wg, np.float64)[:, cols_v]).reshape(B, N, len(hs), dv)
    q = xpos_rotate(q, 0, theta_base)
    k = xpos_rotate(k, 0, theta_base)
    ret, _ = retention_recurrent(q, k, v, np.asarray(gammas, np.float64)[hs])
    y = group_norm_heads(ret, eps)
    z = swish(g) * y
    if heads is not None:
        return (z, y, ret) if return_parts else z
    out = project(z.reshape(B, N, H * dv), wo)
    return (out, z, y, ret) if return_parts else out
