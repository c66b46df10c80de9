"""Test helpers: device transfer of the seeded inputs and the error metric.

The error metric is the maximum, over (batch, head) slices, of the relative
L2 error ||gpu - oracle||_2 / ||oracle||_2 of that slice.  Tolerances: 1e-5
for fp32 inputs, 5e-3 for bf16 inputs with fp32 accumulation.
"""
import numpy as np
import torch

from retention_inputs import to_torch

TOL_F32 = 1e-5
TOL_BF16 = 5e-3


def tol_for(dtype: str) -> float:
    return TOL_F32 if dtype == "f32" else TOL_BF16


def dev(t, device="cuda"):
    return to_torch(t, device)


def host64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to(torch.float64).cpu().numpy()


def max_rel_l2(got, ref, slice_axes):
    """Max over slices (indexed by ``slice_axes``) of ||got - ref|| / ||ref||.
    Slices whose reference norm is zero use the absolute error."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite values in the GPU result"
    other = tuple(a for a in range(ref.ndim) if a not in slice_axes)
    perm = tuple(slice_axes) + other
    g = np.transpose(got, perm).reshape(int(np.prod([ref.shape[a] for a in slice_axes])), -1)
    r = np.transpose(ref, perm).reshape(g.shape)
    num = np.linalg.norm(g - r, axis=1)
    den = np.linalg.norm(r, axis=1)
    rel = np.where(den > 0, num / np.where(den > 0, den, 1.0), num)
    return float(rel.max())


def err_out(got, ref):
    """[B, N, H, dv] outputs: slices are (b, h)."""
    return max_rel_l2(got, ref, (0, 2))


def err_state(got, ref):
    """[B, H, dk, dv] states: slices are (b, h)."""
    return max_rel_l2(got, ref, (0, 1))


U_BF16 = 2.0 ** -8   # unit roundoff of bf16 (8 significant bits)


def bf16_bound_check(got_out, got_state, q_rot, k_rot, v, gammas, ref_out, ref_state, out_is_bf16):
    """Element-wise rounding bound for small shapes, where a per-slice relative
    L2 of a handful of values is ill-conditioned (e.g. one token: the output is
    the scalar q.k times v, and q.k may cancel).

    The tensor-core path rounds to bf16 the rotated q, the zeta-scaled k, the
    masked scores P and the bf16 copy of the state used for the read-out; every
    product accumulates in fp32.  To first order each output element therefore
    differs from the exact result by at most 4u times the same retention
    evaluated on absolute values,
        sum_{m<=n} gamma^(n-m) (|q_n| . |k_m|) |v_m|,
    plus u |out| when the output itself is stored in bf16, and the fp32 state
    by at most 2u times the absolute-value state.  u = 2^-8."""
    import oracle
    aq, ak, av = np.abs(q_rot), np.abs(k_rot), np.abs(v)
    abs_out, abs_state = oracle.retention_recurrent(aq, ak, av, gammas)
    bound = 4 * U_BF16 * abs_out + (U_BF16 * np.abs(ref_out) if out_is_bf16 else 0.0) + 1e-30
    excess = np.abs(np.asarray(got_out, np.float64) - ref_out) - bound
    assert excess.max() <= 0, f"output outside the bf16 rounding bound by {excess.max():.3e}"
    if got_state is not None:
        sb = 2 * U_BF16 * abs_state + 1e-30
        sx = np.abs(np.asarray(got_state, np.float64) - ref_state) - sb
        assert sx.max() <= 0, f"state outside the bf16 rounding bound by {sx.max():.3e}"
