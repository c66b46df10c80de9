"""fp64 CPU oracle for multi-scale retention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
this package imports nothing from the product library: the two share no
code.  Inputs arrive as float64 numpy arrays (the bf16- or fp32-rounded
values, widened exactly), outputs are float64.

The retention core (rotation, recurrent definition, parallel and chunkwise
cross-check forms, decode step, the gradients of the definition) is plain C
in ``retention_oracle.c``; the
MultiScaleRetention layer pieces (projections, per-head GroupNorm, swish gate,
output projection) are in ``msr.py`` on numpy fp64.  Each function cites the
passage of the pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "retention_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (IEEE fp64, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
             "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _configure(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.orc_gamma_pow.restype = ctypes.c_double
    lib.orc_gamma_pow.argtypes = [ctypes.c_double, ctypes.c_longlong]
    lib.orc_max_threads.restype = ctypes.c_int
    lib.orc_xpos_rotate.argtypes = [dp, i, i, i, i, ctypes.c_longlong, ctypes.c_double]
    lib.orc_retention_recurrent.argtypes = [dp, dp, dp, dp, i, i, i, i, i, dp, dp, dp, i]
    lib.orc_retention_parallel.argtypes = [dp, dp, dp, dp, i, i, i, i, i, dp, i]
    lib.orc_retention_chunkwise.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, dp, dp, i]
    lib.orc_decode_step.argtypes = [dp, dp, dp, dp, i, i, i, i, dp, dp, i]
    lib.orc_retention_backward.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, dp, dp, dp, i]
    lib.orc_retention_normalized.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, dp, i]
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _configure(ctypes.CDLL(_LIB))
    return _lib


def swap_library(path):
    """Load the oracle C library from ``path`` in place of the built one and
    return the previous handle (used by the mutation tests to plant a
    mistake in a copy of the oracle; pass the returned handle back to
    restore)."""
    global _lib
    prev = _load()
    _lib = path if not isinstance(path, str) else _configure(ctypes.CDLL(path))
    return prev


def _p(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def max_threads() -> int:
    return int(_load().orc_max_threads())


def gamma_pow(gamma: float, e: int) -> float:
    """gamma^e with 0^0 = 1 (the diagonal of D is 1 for every gamma)."""
    return float(_load().orc_gamma_pow(float(gamma), int(e)))


def xpos_rotate(x, pos_offset: int = 0, theta_base: float = 10000.0):
    """Return a rotated copy of x [B, N, H, d]: pair (2p, 2p+1) of position n
    turned by n * theta_base^(-2p/d)  (P1 sections 6.6 and 6.8)."""
    y = _f64(x).copy()
    B, N, H, d = y.shape
    assert d % 2 == 0
    _load().orc_xpos_rotate(_p(y), B, N, H, d, int(pos_offset), float(theta_base))
    return y


def xpos_unrotate(x, pos_offset: int = 0, theta_base: float = 10000.0):
    """Inverse of xpos_rotate (the transpose of each 2x2 rotation): pair
    (2p, 2p+1) of position n turned by -n * theta_base^(-2p/d).  The
    gradient of a rotated vector flows back through this."""
    y = _f64(x).copy()
    B, N, H, d = y.shape
    assert d % 2 == 0
    p = np.arange(d // 2)
    theta = np.power(float(theta_base), -2.0 * p / d)
    ang = (int(pos_offset) + np.arange(N))[:, None] * theta[None, :]      # [N, d/2]
    c, s = np.cos(ang)[None, :, None, :], np.sin(ang)[None, :, None, :]
    x0, x1 = y[..., 0::2].copy(), y[..., 1::2].copy()
    y[..., 0::2] = x0 * c + x1 * s
    y[..., 1::2] = -x0 * s + x1 * c
    return y


def retention_backward(q, k, v, dout, gammas, xpos: bool = False, pos_offset: int = 0,
                       theta_base: float = 10000.0, nthreads: int = 0):
    """Gradients (dq, dk, dv) of sum(out * dout) for out = retention of the
    (optionally xPos-rotated) q, k and v: the derivatives of the definition
    (P1 section 2.1, P3 Eq. 6) summed by brute force in C; with xpos the
    gradients of the rotated q, k are turned back by the inverse rotation
    (P1 sections 6.6 and 6.8)."""
    q, k, v, do, g = _f64(q), _f64(k), _f64(v), _f64(dout), _f64(gammas)
    if xpos:
        q, k = xpos_rotate(q, pos_offset, theta_base), xpos_rotate(k, pos_offset, theta_base)
    B, N, H, dk = q.shape
    dv = v.shape[3]
    assert k.shape == q.shape and v.shape[:3] == q.shape[:3] and do.shape == v.shape and g.shape == (H,)
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    _load().orc_retention_backward(_p(q), _p(k), _p(v), _p(do), _p(g), B, N, H, dk, dv, _p(dq), _p(dkk),
                                   _p(dvv), int(nthreads))
    if xpos:
        dq, dkk = xpos_unrotate(dq, pos_offset, theta_base), xpos_unrotate(dkk, pos_offset, theta_base)
    return dq, dkk, dvv


NORM_DECAY = 1  # score normalization 2: D_nm / sqrt(sum_i D_ni)
NORM_SCORE = 2  # score normalization 3: R_nm / max(|sum_i R_ni|, 1)


def retention_normalized(q, k, v, gammas, flags: int = NORM_DECAY | NORM_SCORE, xpos: bool = False,
                         pos_offset: int = 0, theta_base: float = 10000.0, nthreads: int = 0):
    """Parallel form with the score normalizations 2 and 3 (P1 section 8.5;
    P3 "Retention Score Normalization"), brute force in C over the whole
    sequence; with xpos, q and k are rotated first (P1 sections 6.6, 6.8)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(gammas)
    if xpos:
        q, k = xpos_rotate(q, pos_offset, theta_base), xpos_rotate(k, pos_offset, theta_base)
    B, N, H, dk = q.shape
    dv = v.shape[3]
    assert k.shape == q.shape and v.shape[:3] == q.shape[:3] and g.shape == (H,)
    out = np.zeros((B, N, H, dv))
    _load().orc_retention_normalized(_p(q), _p(k), _p(v), _p(g), B, N, H, dk, dv, int(flags), _p(out),
                                     int(nthreads))
    return out


def retention_recurrent(q, k, v, gammas, init_state=None, nthreads: int = 0):
    """Definition (P1 section 2.1, P3 Eq. 6).  Returns (out, final_state)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(gammas)
    B, N, H, dk = q.shape
    dv = v.shape[3]
    assert k.shape == q.shape and v.shape[:3] == q.shape[:3] and g.shape == (H,)
    out = np.zeros((B, N, H, dv))
    fs = np.zeros((B, H, dk, dv))
    st = None if init_state is None else _f64(init_state)
    if st is not None:
        assert st.shape == (B, H, dk, dv)
    _load().orc_retention_recurrent(_p(q), _p(k), _p(v), _p(g), B, N, H, dk, dv, _p(st),
                                    _p(out), _p(fs), int(nthreads))
    return out, fs


def retention_parallel(q, k, v, gammas, nthreads: int = 0):
    """Brute-force (Q K^T (.) D) V (P1 section 4.3, P3 Eq. 5)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(gammas)
    B, N, H, dk = q.shape
    dv = v.shape[3]
    out = np.zeros((B, N, H, dv))
    _load().orc_retention_parallel(_p(q), _p(k), _p(v), _p(g), B, N, H, dk, dv, _p(out),
                                   int(nthreads))
    return out


def retention_chunkwise(q, k, v, gammas, chunk: int, nthreads: int = 0):
    """Chunkwise recurrent form (P1 section 7.2, P3 Eq. 7).  Returns (out, R_final)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(gammas)
    B, N, H, dk = q.shape
    dv = v.shape[3]
    assert chunk >= 1
    out = np.zeros((B, N, H, dv))
    fs = np.zeros((B, H, dk, dv))
    _load().orc_retention_chunkwise(_p(q), _p(k), _p(v), _p(g), B, N, H, dk, dv, int(chunk),
                                    _p(out), _p(fs), int(nthreads))
    return out, fs


def decode_step(q, k, v, gammas, state, nthreads: int = 0):
    """One recurrent step on a carried state (P1 section 5.2).  q, k [B, H, dk],
    v [B, H, dv], state [B, H, dk, dv].  Returns (out [B, H, dv], new_state)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(gammas)
    st = _f64(state).copy()
    B, H, dk = q.shape
    dv = v.shape[2]
    out = np.zeros((B, H, dv))
    _load().orc_decode_step(_p(q), _p(k), _p(v), _p(g), B, H, dk, dv, _p(st), _p(out),
                            int(nthreads))
    return out, st
