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
