"""GPU parity on seeded random shapes, through the C ABI: the workspace path
of the chunkwise forward (with and without a carried initial state), the
decode step and the backward, each against the fp64 oracle.  The shapes are
drawn once from a fixed seed (batch, length with ragged chunks, heads,
d_k in {64, 128, 256}, d_v a multiple of 64 (of 128 for the backward),
rotation on or off at an offset, output dtype), so that combinations the
hand-picked cases do not name are covered too."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import gamma_schedule, gamma_schedule_scaled, make_tensor
from tests.helpers import TOL_BF16, TOL_F32, bf16_bound_check, dev, err_out, err_state, host64

pytestmark = pytest.mark.gpu

R = None


@pytest.fixture(scope="module", autouse=True)
def lib():
    global R
    import linear_recurrent_sequence_chunkwise_b200 as mod
    R = mod
    yield mod
    mod.ret_check_device_error()


def _draw(seed, n):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        cases.append(dict(B=int(rng.integers(1, 4)), N=int(rng.integers(1, 700)), H=int(rng.integers(1, 5)),
                          dk=int(rng.choice([64, 128, 256])), dv=int(64 * rng.integers(1, 9)),
                          xpos=bool(rng.integers(0, 2)), off=int(rng.integers(0, 3000)),
                          f32_out=bool(rng.integers(0, 2)), scaled=bool(rng.integers(0, 2))))
    return cases


FORWARD = _draw(0xF0, 14)
BACKWARD = [dict(c, dv=128 * (1 + c["dv"] // 256), dk=max(c["dk"], 128), N=max(c["N"], 128)) for c in _draw(0xB0, 5)]
DECODE = _draw(0xD0, 6)


def _gammas(c):
    return gamma_schedule_scaled(c["H"]) if c["scaled"] else gamma_schedule(c["H"])


def _qkv(seed, c):
    B, N, H, dk, dv = c["B"], c["N"], c["H"], c["dk"], c["dv"]
    return (make_tensor(seed, 1, (B, N, H, dk), "bf16", dk ** -0.5), make_tensor(seed, 2, (B, N, H, dk), "bf16", dk ** -0.5),
            make_tensor(seed, 3, (B, N, H, dv), "bf16"))


def _check(out, fs, q, k, v, g, c):
    qr, kr = q.f64, k.f64
    if c["xpos"]:
        qr, kr = oracle.xpos_rotate(qr, c["off"]), oracle.xpos_rotate(kr, c["off"])
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    if c["N"] >= 256:
        assert err_out(host64(out), ref) < TOL_BF16
        assert err_state(host64(fs), S) < TOL_BF16
    else:   # few rows per slice: the element-wise rounding bound
        bf16_bound_check(host64(out), host64(fs), qr, kr, v.f64, g, ref, S, not c["f32_out"])


@pytest.mark.parametrize("i", range(len(FORWARD)))
def test_random_forward(i):
    c = FORWARD[i]
    q, k, v = _qkv(500 + i, c)
    g = _gammas(c)
    nb = R.ret_chunkwise_workspace_bytes(c["B"], c["N"], c["H"], c["dk"], c["dv"], 128, torch.bfloat16, c["xpos"])
    assert nb > 0, c
    ws = torch.full((nb,), 0x5A, dtype=torch.uint8, device="cuda")
    out, fs = R.ret_forward_chunkwise_ws(dev(q), dev(k), dev(v), g, 128, ws,
                                         out_dtype=torch.float32 if c["f32_out"] else torch.bfloat16,
                                         xpos=c["xpos"], pos_offset=c["off"], want_final_state=True)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    _check(out, fs, q, k, v, g, c)


@pytest.mark.parametrize("i", range(0, len(FORWARD), 2))
def test_random_forward_in_two_calls(i):
    """The same sequence split at a random token into two calls that hand
    the fp32 state on (prepare + prepared, the second from the first's
    final state at pos_offset + split)."""
    c = FORWARD[i]
    if c["N"] < 2:
        pytest.skip("one token")
    q, k, v = _qkv(500 + i, c)
    g = _gammas(c)
    split = int(np.random.default_rng(i).integers(1, c["N"]))
    qd, kd, vd = dev(q), dev(k), dev(v)
    odt = torch.float32 if c["f32_out"] else torch.bfloat16
    S = torch.empty((c["B"], c["H"], c["dk"], c["dv"]), dtype=torch.float32, device="cuda")
    outs = []
    for lo, hi, init in ((0, split, None), (split, c["N"], S)):
        part = [t[:, lo:hi].contiguous() for t in (qd, kd, vd)]
        nb = R.ret_chunkwise_prepare_workspace_bytes(c["B"], hi - lo, c["H"], c["dk"], c["dv"], 128,
                                                     torch.bfloat16, c["xpos"])
        ws = torch.full((nb,), 0x5A, dtype=torch.uint8, device="cuda")
        R.ret_chunkwise_prepare(part[0], part[1], g, 128, ws, c["dv"], xpos=c["xpos"], pos_offset=c["off"] + lo)
        outs.append(R.ret_forward_chunkwise_prepared(*part, g, 128, ws, final_state=S, initial_state=init,
                                                     out_dtype=odt, xpos=c["xpos"], pos_offset=c["off"] + lo)[0])
    torch.cuda.synchronize()
    R.ret_check_device_error()
    _check(torch.cat(outs, dim=1), S, q, k, v, g, c)


@pytest.mark.parametrize("i", range(len(BACKWARD)))
def test_random_backward(i):
    c = BACKWARD[i]
    B, N, H, dk, dv = c["B"], c["N"], c["H"], c["dk"], c["dv"]
    q, k, v = _qkv(600 + i, c)
    do = make_tensor(600 + i, 4, (B, N, H, dv), "bf16")
    g = _gammas(c)
    got = R.ret_backward_chunkwise(dev(q), dev(k), dev(v), dev(do), g, 128, xpos=c["xpos"], pos_offset=c["off"])
    torch.cuda.synchronize()
    R.ret_check_device_error()
    ref = oracle.retention_backward(q.f64, k.f64, v.f64, do.f64, g, xpos=c["xpos"], pos_offset=c["off"])
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        assert err_out(host64(a), r) < TOL_BF16, (name, c)


@pytest.mark.parametrize("i", range(len(DECODE)))
def test_random_decode(i):
    c = DECODE[i]
    B, H, dk, dv, T = c["B"], c["H"], c["dk"], c["dv"], 5
    dt = "f32" if c["f32_out"] else "bf16"
    mk = lambda st, shape: make_tensor(700 + i, st, shape, dt, dk ** -0.5 if st < 3 else 1.0)
    q, k, v = mk(1, (B, T, H, dk)), mk(2, (B, T, H, dk)), mk(3, (B, T, H, dv))
    s0 = make_tensor(700 + i, 4, (B, H, dk, dv), "f32", 0.1)
    g = _gammas(c)
    S = dev(s0).clone()
    qd, kd, vd = dev(q), dev(k), dev(v)
    outs = [R.ret_decode_step(qd[:, t].contiguous(), kd[:, t].contiguous(), vd[:, t].contiguous(), g, S)
            for t in range(T)]
    torch.cuda.synchronize()
    R.ret_check_device_error()
    ref, Sref = oracle.retention_recurrent(q.f64, k.f64, v.f64, g, init_state=s0.f64)
    got = np.stack([host64(o) for o in outs], axis=1)
    tol = TOL_F32 if dt == "f32" else TOL_BF16
    assert err_out(got, ref) < tol, c
    assert err_state(host64(S), Sref) < tol, c


@pytest.mark.parametrize("n0,dt", [(77, "bf16"), (128, "bf16"), (300, "bf16"), (41, "f32")])
def test_no_causal_leakage(n0, dt):
    """Outputs before token n0 do not depend on tokens n0 and later: new
    values from n0 on leave them bit for bit the same (the masked scores are
    exact zeros, so the later keys and values add exact zeros), on the
    tensor-core workspace path (bf16) and on the fp32 CUDA-core path."""
    B, N, H = 2, 400, 2
    dk, dv = (256, 128) if dt == "bf16" else (16, 16)
    mk = lambda seed, st, d: make_tensor(seed, st, (B, N, H, d), dt, dk ** -0.5 if st < 3 else 1.0)
    q, k, v = mk(800, 1, dk), mk(800, 2, dk), mk(800, 3, dv)
    q2, k2, v2 = mk(801, 1, dk), mk(801, 2, dk), mk(801, 3, dv)
    g = gamma_schedule(H)
    outs = []
    for tens in ((q, k, v), (q2, k2, v2)):
        qd, kd, vd = (dev(t) for t in (q, k, v))
        if tens[0] is q2:   # tokens from n0 on replaced by other values
            for a, b in zip((qd, kd, vd), (dev(q2), dev(k2), dev(v2))):
                a[:, n0:] = b[:, n0:]
        if dt == "bf16":
            nb = R.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, 128, torch.bfloat16, True)
            ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
            outs.append(R.ret_forward_chunkwise_ws(qd, kd, vd, g, 128, ws, out_dtype=torch.float32, xpos=True))
        else:
            outs.append(R.ret_forward_chunkwise(qd, kd, vd, g, 16, out_dtype=torch.float32))
    torch.cuda.synchronize()
    R.ret_check_device_error()
    assert torch.equal(outs[0][:, :n0], outs[1][:, :n0])
    assert not torch.equal(outs[0][:, n0:], outs[1][:, n0:])
