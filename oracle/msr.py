"""MultiScaleRetention layer and RetNet block pieces of the oracle, numpy
fp64 -- TEST INFRASTRUCTURE ONLY (see the package docstring).

Follows "Hybrid Architectures: RetNet and the Three Computation Paradigms"
section 9.1 (MSR(X) = (swish(X W_G) (.) Y) W_O, Y = GroupNorm_h(heads)),
section 8.4 (GroupNorm with one group per head) and the RetNet paper summary's
"Gated Multi-Scale Retention" section (W_V and W_G widen to 2d, W_O maps 2d
back to d); the RetNet block follows P1 section 9.2 and the summary's
"Overall RetNet Architecture" (pre-LayerNorm residual layout, FFN(x) =
gelu(x W1) W2).  Matrix products use numpy's fp64 matmul and the error
function scipy's erf, as library steps.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

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


def layer_norm(x, gain=None, bias=None, eps: float = 1e-5):
    """LayerNorm over the last axis (Ba et al. 2016, as P1 section 9.2 uses
    it): (x - mean) / sqrt(var + eps) with the biased variance, times gain
    plus bias (1 and 0 when None)."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if gain is not None:
        y = y * np.asarray(gain, np.float64)
    if bias is not None:
        y = y + np.asarray(bias, np.float64)
    return y


def gelu(x):
    """gelu(x) = x Phi(x), Phi the standard normal CDF = (1 + erf(x / sqrt 2)) / 2
    (the exact form; P1 section 9.2 names GELU)."""
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def ffn(x, w1, w2):
    """FFN(x) = gelu(x W1) W2  (P1 section 9.2)."""
    return project(gelu(project(x, w1)), w2)


def retnet_block(x, wq, wk, wv, wg, wo, w1, w2, gammas, H: int, k_scale: float, gn_eps: float = 1e-5,
                 ln_eps: float = 1e-5, ln1=(None, None), ln2=(None, None), theta_base: float = 10000.0,
                 return_y: bool = False):
    """One RetNet block, pre-LayerNorm residual layout (P1 section 9.2):
        Y   = MSR(LN(X)) + X
        out = FFN(LN(Y)) + Y
    ln1 / ln2 are (gain, bias) pairs of the two LayerNorms."""
    x = np.asarray(x, np.float64)
    y = msr_forward(layer_norm(x, ln1[0], ln1[1], ln_eps), wq, wk, wv, wg, wo, gammas, H, k_scale, gn_eps,
                    theta_base) + x
    out = ffn(layer_norm(y, ln2[0], ln2[1], ln_eps), w1, w2) + y
    return (out, y) if return_y else out
