"""GPU parity of retention with the score normalizations 2 and 3 (chunkwise
forward and decode step) against the fp64 oracle's brute-force parallel form
with the normalized decay matrix and scores, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import C3, gamma_schedule, make_tensor
from tests.helpers import TOL_BF16, TOL_F32, dev, err_out, err_state, host64

pytestmark = pytest.mark.gpu

R = None
BOTH = 3


@pytest.fixture(scope="module", autouse=True)
def lib():
    global R
    import linear_recurrent_sequence_chunkwise_b200 as mod
    R = mod
    yield mod
    mod.ret_check_device_error()


def qkv(seed, B, N, H, dk, dv, scale, dtype="bf16"):
    return (make_tensor(seed, 1, (B, N, H, dk), dtype, scale), make_tensor(seed, 2, (B, N, H, dk), dtype, scale),
            make_tensor(seed, 3, (B, N, H, dv), dtype))


def workspace(B, N, H, dk, dv, xpos):
    nb = R.ret_normalized_workspace_bytes(B, N, H, dk, dv, 128, torch.bfloat16, xpos)
    assert nb > 0
    return torch.full((nb,), 0x7F, dtype=torch.uint8, device="cuda")   # scratch starts as garbage


def run(q, k, v, g, flags, xpos=False, off=0, out_dtype=torch.float32, **kw):
    B, N, H, dk = q.shape
    dv = v.shape[3]
    out = R.ret_forward_chunkwise_normalized(dev(q) if not torch.is_tensor(q) else q,
                                             dev(k) if not torch.is_tensor(k) else k,
                                             dev(v) if not torch.is_tensor(v) else v, g, 128, norm_flags=flags,
                                             workspace=workspace(B, N, H, dk, dv, xpos), out_dtype=out_dtype,
                                             xpos=xpos, pos_offset=off, **kw)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    return out


# q . k of order one, so that the score normalization divides many rows and
# leaves others (|sum| < 1) unchanged.
@pytest.mark.parametrize("B,N,H,dk,dv,xpos,flags,odt", [
    (2, 300, 2, 128, 128, False, BOTH, torch.bfloat16),     # ragged last chunk
    (1, 260, 2, 256, 256, True, BOTH, torch.float32),
    (1, 200, 3, 256, 64, True, 1, torch.bfloat16),          # decay normalization alone
    (1, 129, 2, 128, 192, False, 2, torch.float32),         # score normalization alone; one-row last chunk
    (2, 513, 2, 256, 512, True, BOTH, torch.bfloat16),      # the 6.7B head shape
    (1, 1, 2, 128, 64, True, BOTH, torch.float32),          # a single token
])
def test_normalized_matches_oracle(B, N, H, dk, dv, xpos, flags, odt):
    q, k, v = qkv(300 + N, B, N, H, dk, dv, dk ** -0.25)
    g = gamma_schedule(H)
    out = run(q, k, v, g, flags, xpos=xpos, out_dtype=odt)
    ref = oracle.retention_normalized(q.f64, k.f64, v.f64, g, flags=flags, xpos=xpos)
    assert err_out(host64(out), ref) < TOL_BF16


def test_score_normalization_is_exercised():
    """The inputs above put row sums on both sides of 1 (so both branches of
    the max run): checked on the oracle's own plain retention with v = 1."""
    q, k, _ = qkv(300 + 300, 2, 300, 2, 128, 128, 128 ** -0.25)
    s, _ = oracle.retention_recurrent(q.f64, k.f64, np.ones((2, 300, 2, 1)), gamma_schedule(2))
    assert (np.abs(s) > 1).mean() > 0.2 and (np.abs(s) < 1).mean() > 0.05


def test_normalized_without_flags_is_plain_retention():
    q, k, v = qkv(311, 1, 300, 2, 256, 128, 256 ** -0.5)
    g = gamma_schedule(2)
    out = run(q, k, v, g, 0, xpos=True)
    ref, _ = oracle.retention_recurrent(oracle.xpos_rotate(q.f64), oracle.xpos_rotate(k.f64), v.f64, g)
    assert err_out(host64(out), ref) < TOL_BF16


def test_position_offset_counts_earlier_rows():
    """pos_offset P with zero initial states is a sequence whose first P tokens
    have zero keys: they add nothing to the scores but count in the decay
    row sums, and the rotation runs at positions P + n."""
    P, N, H, dk, dv = 100, 200, 2, 128, 64
    q, k, v = qkv(312, 1, N, H, dk, dv, dk ** -0.25)
    g = gamma_schedule(H)
    out = run(q, k, v, g, BOTH, xpos=True, off=P)
    pad = lambda x: np.concatenate([np.zeros((1, P) + x.shape[2:]), x], axis=1)
    ref = oracle.retention_normalized(pad(q.f64), pad(k.f64), pad(v.f64), g, flags=BOTH, xpos=True)[:, P:]
    assert err_out(host64(out), ref) < TOL_BF16


@pytest.mark.parametrize("split", [128, 77, 1])
def test_normalized_continuation(split):
    """Two calls handing S and z on equal the oracle on the whole sequence;
    the final z is the decayed key sum (the recurrent state for v = 1)."""
    B, N, H, dk, dv = 1, 300, 2, 256, 128
    q, k, v = qkv(313, B, N, H, dk, dv, dk ** -0.25)
    g = gamma_schedule(H)
    qd, kd, vd = dev(q), dev(k), dev(v)
    S = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    z = torch.empty((B, H, dk), dtype=torch.float32, device="cuda")
    o1 = run(qd[:, :split].contiguous(), kd[:, :split].contiguous(), vd[:, :split].contiguous(), g, BOTH, xpos=True,
             final_state=S, final_z=z)
    o2 = run(qd[:, split:].contiguous(), kd[:, split:].contiguous(), vd[:, split:].contiguous(), g, BOTH, xpos=True,
             off=split, initial_state=S, final_state=S, initial_z=z, final_z=z)
    ref = oracle.retention_normalized(q.f64, k.f64, v.f64, g, flags=BOTH, xpos=True)
    got = np.concatenate([host64(o1), host64(o2)], axis=1)
    assert err_out(got, ref) < TOL_BF16
    kr = oracle.xpos_rotate(k.f64)
    _, zref = oracle.retention_recurrent(oracle.xpos_rotate(q.f64), kr, np.ones((B, N, H, 1)), g)
    assert err_state(host64(z)[..., None], zref) < TOL_BF16


@pytest.mark.parametrize("dtype,flags", [("bf16", BOTH), ("f32", BOTH), ("f32", 1), ("f32", 2)])
def test_decode_normalized_matches_oracle(dtype, flags):
    B, N, H, dk, dv = 2, 40, 2, 64, 64
    q, k, v = qkv(314, B, N, H, dk, dv, dk ** -0.25, dtype)
    g = gamma_schedule(H)
    qd, kd, vd = dev(q), dev(k), dev(v)
    S = torch.zeros((B, H, dk, dv), dtype=torch.float32, device="cuda")
    z = torch.zeros((B, H, dk), dtype=torch.float32, device="cuda")
    outs = []
    for n in range(N):
        outs.append(R.ret_decode_step_normalized(qd[:, n].contiguous(), kd[:, n].contiguous(), vd[:, n].contiguous(),
                                                 g, S, z, n, norm_flags=flags))
    torch.cuda.synchronize()
    R.ret_check_device_error()
    got = np.stack([host64(o) for o in outs], axis=1)
    ref = oracle.retention_normalized(q.f64, k.f64, v.f64, g, flags=flags)
    assert err_out(got, ref) < (TOL_BF16 if dtype == "bf16" else TOL_F32)


def test_prefill_then_decode_normalized():
    """A chunkwise prefill hands S and z to decode steps at the next positions
    (the inference protocol); every output matches the whole-sequence oracle."""
    B, N0, T, H, dk, dv = 2, 200, 12, 2, 128, 128
    q, k, v = qkv(315, B, N0 + T, H, dk, dv, dk ** -0.25)
    g = gamma_schedule(H)
    qd, kd, vd = dev(q), dev(k), dev(v)
    S = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    z = torch.empty((B, H, dk), dtype=torch.float32, device="cuda")
    pre = run(qd[:, :N0].contiguous(), kd[:, :N0].contiguous(), vd[:, :N0].contiguous(), g, BOTH,
              final_state=S, final_z=z)
    dec = [R.ret_decode_step_normalized(qd[:, n].contiguous(), kd[:, n].contiguous(), vd[:, n].contiguous(), g, S, z,
                                        n) for n in range(N0, N0 + T)]
    torch.cuda.synchronize()
    R.ret_check_device_error()
    got = np.concatenate([host64(pre), np.stack([host64(o) for o in dec], axis=1)], axis=1)
    ref = oracle.retention_normalized(q.f64, k.f64, v.f64, g, flags=BOTH)
    assert err_out(got, ref) < TOL_BF16


def test_normalized_workload_all_heads():
    """The 8k x 16-head workload (rotation on).  The normalized output is the
    plain one times f_n = c_n / max(|c_n s_n|, 1) per (token, head): the
    oracle's plain recurrence gives the plain output and, with v = 1, the row
    sums s_n; c_n^-2 is the geometric series sum_{i<=n} gamma^i."""
    w = C3
    q, k, v = w.qkv()
    qr, kr = oracle.xpos_rotate(q.f64), oracle.xpos_rotate(k.f64)
    plain, _ = oracle.retention_recurrent(qr, kr, v.f64, w.gammas)
    s, _ = oracle.retention_recurrent(qr, kr, np.ones((w.B, w.N, w.H, 1)), w.gammas)
    n = np.arange(w.N)[None, :, None, None]
    gam = w.gammas[None, None, :, None]
    c = 1.0 / np.sqrt((1 - gam ** (n + 1)) / (1 - gam))
    f = c / np.maximum(np.abs(c * s), 1.0)
    out = run(q, k, v, w.gammas, BOTH, xpos=True, out_dtype=torch.bfloat16)
    assert err_out(host64(out), f * plain) < TOL_BF16


@pytest.mark.parametrize("xpos,flags", [(True, 0), (True, BOTH), (False, BOTH)])
def test_decode_at_per_sequence_positions(xpos, flags):
    """Three sequences at positions 0, 37 and 1000 take T decode steps in one
    batch.  Each equals the oracle on its own sequence with that many leading
    zero tokens (zero keys add nothing to S or z; the positions still count
    for the rotation and the decay row sums)."""
    pos0 = [0, 37, 1000]
    B, T, H, dk, dv = len(pos0), 6, 2, 64, 64
    q, k, v = qkv(316, B, T, H, dk, dv, dk ** -0.25)
    g = gamma_schedule(H)
    qd, kd, vd = dev(q), dev(k), dev(v)
    S = torch.zeros((B, H, dk, dv), dtype=torch.float32, device="cuda")
    z = torch.zeros((B, H, dk), dtype=torch.float32, device="cuda")
    outs = []
    for t in range(T):
        pos = torch.tensor([p + t for p in pos0], dtype=torch.int64, device="cuda")
        outs.append(R.ret_decode_step_positions(qd[:, t].contiguous(), kd[:, t].contiguous(), vd[:, t].contiguous(),
                                                g, S, pos, z=z if flags else None, xpos=xpos, norm_flags=flags))
    torch.cuda.synchronize()
    R.ret_check_device_error()
    got = np.stack([host64(o) for o in outs], axis=1)    # [B, T, H, dv]
    for b, P in enumerate(pos0):
        pad = lambda x: np.concatenate([np.zeros((1, P) + x.shape[2:]), x[b:b + 1]], axis=1)
        ref = oracle.retention_normalized(pad(q.f64), pad(k.f64), pad(v.f64), g, flags=flags, xpos=xpos)[:, P:]
        assert err_out(got[b:b + 1], ref) < TOL_BF16, b
