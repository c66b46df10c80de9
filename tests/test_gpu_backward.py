"""GPU parity of ret_backward_chunkwise (gradients of the chunkwise forward
with respect to q, k, v) against the fp64 oracle's derivatives of the
definition, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import gamma_schedule, make_tensor
from tests.helpers import TOL_BF16, dev, err_out, host64

pytestmark = pytest.mark.gpu

R = None


@pytest.fixture(scope="module", autouse=True)
def lib():
    global R
    import linear_recurrent_sequence_chunkwise_b200 as mod
    R = mod
    yield mod
    mod.ret_check_device_error()


def inputs(seed, B, N, H, dk, dv):
    s = dk ** -0.5
    return (make_tensor(seed, 1, (B, N, H, dk), "bf16", s), make_tensor(seed, 2, (B, N, H, dk), "bf16", s),
            make_tensor(seed, 3, (B, N, H, dv), "bf16"), make_tensor(seed, 4, (B, N, H, dv), "bf16"))


def run(q, k, v, do, g, xpos, off):
    nb = R.ret_backward_workspace_bytes(*q.shape, v.shape[3], 128, torch.bfloat16, xpos)
    assert nb > 0
    ws = torch.full((nb,), 0x7F, dtype=torch.uint8, device="cuda")     # scratch starts as garbage
    out = R.ret_backward_chunkwise(dev(q), dev(k), dev(v), dev(do), g, 128, workspace=ws, xpos=xpos, pos_offset=off)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    return [host64(t) for t in out]


@pytest.mark.parametrize("B,N,H,dk,dv,xpos,off", [
    (2, 300, 2, 128, 128, False, 0),     # ragged last chunk, no rotation
    (1, 260, 2, 256, 256, True, 7),      # rotation at an offset
    (1, 200, 1, 256, 384, True, 0),      # d_v in three 128-column slices
    (2, 513, 3, 256, 512, True, 0),      # the 6.7B head shape, two 256-column slices
])
def test_backward_matches_oracle(B, N, H, dk, dv, xpos, off):
    q, k, v, do = inputs(100 + N, B, N, H, dk, dv)
    g = gamma_schedule(H)
    got = run(q, k, v, do, g, xpos, off)
    ref = oracle.retention_backward(q.f64, k.f64, v.f64, do.f64, g, xpos=xpos, pos_offset=off)
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        assert err_out(a, r) < TOL_BF16, name


U_BF16 = 2.0 ** -8


def test_backward_single_token_within_rounding_bound():
    """One token: dv = (q'.k') dout and dq, dk = (dout.v) k', q' -- single dot
    products that can cancel, so the relative L2 is ill-conditioned.  Check
    each element against the first-order bound of the bf16 roundings on the
    path (rotated q', k', zeta-scaled keys, P): 8u times the same sums over
    absolute values (and, after the inverse rotation, over both members of
    each pair)."""
    B, N, H, dk, dv, off = 1, 1, 2, 128, 128, 3
    q, k, v, do = inputs(130, B, N, H, dk, dv)
    g = gamma_schedule(H)
    got = run(q, k, v, do, g, True, off)
    ref = oracle.retention_backward(q.f64, k.f64, v.f64, do.f64, g, xpos=True, pos_offset=off)
    qr, kr = oracle.xpos_rotate(q.f64, off), oracle.xpos_rotate(k.f64, off)
    aq, ak, av = oracle.retention_backward(np.abs(qr), np.abs(kr), np.abs(v.f64), np.abs(do.f64), g)
    for a, r, bound, rot in ((got[0], ref[0], aq, True), (got[1], ref[1], ak, True), (got[2], ref[2], av, False)):
        if rot:
            pair = bound[..., 0::2] + bound[..., 1::2]
            bound = np.repeat(pair, 2, axis=-1)
        assert np.all(np.abs(a - r) <= 8 * U_BF16 * bound + 1e-7)


@pytest.mark.parametrize("gam", [1.0, 0.75])
def test_backward_decays(gam):
    q, k, v, do = inputs(120, 1, 390, 2, 256, 128)
    g = np.array([gam, 0.99])
    got = run(q, k, v, do, g, True, 0)
    ref = oracle.retention_backward(q.f64, k.f64, v.f64, do.f64, g, xpos=True)
    for a, r in zip(got, ref):
        assert err_out(a, r) < TOL_BF16


def test_backward_long_sequence_sampled_heads():
    """16 heads of 256/512 over 2048 tokens on the GPU; heads 0 and 11
    against the oracle."""
    B, N, H, dk, dv = 1, 2048, 16, 256, 512
    q, k, v, do = inputs(121, B, N, H, dk, dv)
    g = gamma_schedule(H)
    got = run(q, k, v, do, g, True, 0)
    hs = [0, 11]
    pick = lambda t: np.ascontiguousarray(t.f64[:, :, hs])
    ref = oracle.retention_backward(pick(q), pick(k), pick(v), pick(do), np.array([g[h] for h in hs]), xpos=True)
    for a, r in zip(got, ref):
        assert err_out(np.ascontiguousarray(a[:, :, hs]), r) < TOL_BF16
