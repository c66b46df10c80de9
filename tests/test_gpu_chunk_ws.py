"""GPU parity of the workspace path of the chunkwise forward (the scores pass:
rotation, key scaling and the masked intra-chunk scores on the tensor cores;
then the warp-specialized tcgen05 kernel) against the fp64 oracle, through
the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import C3, C4, gamma_schedule, gamma_schedule_scaled, make_tensor
from tests.helpers import TOL_BF16, bf16_bound_check, dev, err_out, err_state, host64

pytestmark = pytest.mark.gpu

R = None


@pytest.fixture(scope="module", autouse=True)
def lib():
    global R
    import linear_recurrent_sequence_chunkwise_b200 as mod
    R = mod
    yield mod
    mod.ret_check_device_error()


def qkv(seed, B, N, H, dk, dv, scale):
    return (make_tensor(seed, 1, (B, N, H, dk), "bf16", scale), make_tensor(seed, 2, (B, N, H, dk), "bf16", scale),
            make_tensor(seed, 3, (B, N, H, dv), "bf16"))


def rotated(q, k, xpos, off=0):
    qf, kf = q.f64, k.f64
    if xpos:
        qf, kf = oracle.xpos_rotate(qf, off), oracle.xpos_rotate(kf, off)
    return qf, kf


def run_ws(q, k, v, g, chunk, **kw):
    B, N, H, dk = q.shape
    dv = v.shape[3]
    nb = R.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, chunk, torch.bfloat16, kw.get("xpos", False))
    assert nb > 0
    ws = torch.full((nb + 512,), 0xAB, dtype=torch.uint8, device="cuda")[256:256 + nb]
    assert ws.data_ptr() % 256 == 0
    return R.ret_forward_chunkwise_ws(dev(q), dev(k), dev(v), g, chunk, ws, **kw)


@pytest.mark.parametrize("B,N,H,dk,dv,xpos,off", [
    (1, 128, 1, 256, 64, True, 0),
    (2, 300, 2, 256, 128, True, 0),
    (1, 1, 2, 256, 64, True, 9),
    (1, 77, 1, 128, 64, False, 0),
    (2, 513, 3, 128, 192, True, 1000),
    (1, 640, 2, 256, 512, False, 0),
    (1, 1024, 2, 256, 512, True, 0),
])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_chunkwise_ws_small(B, N, H, dk, dv, xpos, off, out_dtype):
    q, k, v = qkv(70 + N, B, N, H, dk, dv, dk ** -0.5)
    g = gamma_schedule(H)
    out, fs = run_ws(q, k, v, g, 128, out_dtype=out_dtype, xpos=xpos, pos_offset=off, want_final_state=True)
    R.ret_check_device_error()
    qr, kr = rotated(q, k, xpos, off)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    bf16_bound_check(host64(out), host64(fs), qr, kr, v.f64, g, ref, S, out_dtype == torch.bfloat16)
    if N >= 256:
        assert err_out(host64(out), ref) < TOL_BF16
        assert err_state(host64(fs), S) < TOL_BF16


@pytest.mark.parametrize("gam", [1.0, 0.75, 0.6])
def test_chunkwise_ws_decays(gam):
    q, k, v = qkv(80, 1, 390, 2, 256, 64, 1 / 16)
    g = np.array([gam, 0.99])
    out, fs = run_ws(q, k, v, g, 128, out_dtype=torch.float32, xpos=True, want_final_state=True)
    R.ret_check_device_error()
    qr, kr = rotated(q, k, True)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    bf16_bound_check(host64(out), host64(fs), qr, kr, v.f64, g, ref, S, False)


def test_ws_long_sequence_workload_all_heads():
    w = C3
    q, k, v = w.qkv()
    qr, kr = rotated(q, k, True)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, w.gammas)
    for odt in (torch.bfloat16, torch.float32):
        out, fs = run_ws(q, k, v, w.gammas, w.chunk, out_dtype=odt, xpos=True, want_final_state=True)
        R.ret_check_device_error()
        assert err_out(host64(out), ref) < TOL_BF16
        assert err_state(host64(fs), S) < TOL_BF16


def test_ws_matches_fused_path():
    """Workspace path and single-kernel path agree (same arithmetic up to
    rounding order)."""
    q, k, v = qkv(81, 2, 700, 3, 256, 128, 1 / 16)
    g = gamma_schedule(3)
    a, fa = run_ws(q, k, v, g, 128, out_dtype=torch.float32, xpos=True, want_final_state=True)
    b, fb = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), g, 128, out_dtype=torch.float32, xpos=True,
                                    want_final_state=True)
    torch.cuda.synchronize()
    assert err_out(host64(a), host64(b)) < 1e-3
    assert err_state(host64(fa), host64(fb)) < 1e-3


def _picked(t, picks):
    return np.stack([t.f64_at((b, slice(None), h)) for b, h in picks], axis=1)[None]


def test_ws_prefill_workload_sampled():
    w = C4
    q, k, v = w.qkv()
    out, fs = run_ws(q, k, v, w.gammas, w.chunk, out_dtype=torch.float32, want_final_state=True)
    R.ret_check_device_error()
    picks = [(0, 0), (17, 5), (63, 15), (40, 11)]
    g = np.array([w.gammas[h] for _, h in picks])
    ref, S = oracle.retention_recurrent(_picked(q, picks), _picked(k, picks), _picked(v, picks), g)
    o = out.cpu().numpy()
    got = np.stack([o[b, :, h] for b, h in picks], axis=1)[None].astype(np.float64)
    assert err_out(got, ref) < TOL_BF16
    f = fs.cpu().numpy()
    assert err_state(np.stack([f[b, h] for b, h in picks])[None].astype(np.float64), S) < TOL_BF16


def test_ws_rejects_small_workspace():
    q, k, v = qkv(82, 1, 256, 1, 256, 64, 1 / 16)
    nb = R.ret_chunkwise_workspace_bytes(1, 256, 1, 256, 64, 128, torch.bfloat16, True)
    ws = torch.empty(nb - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(R.RetentionError):
        R.ret_forward_chunkwise_ws(dev(q), dev(k), dev(v), [0.9], 128, ws, xpos=True)


def run_two_pass(qd, kd, vd, g, chunk, init=None, fs=None, pos_offset=0, xpos=True, out_dtype=torch.float32):
    """ret_chunkwise_prepare then ret_forward_chunkwise_prepared on device tensors."""
    B, N, H, dk = qd.shape
    dv = vd.shape[3]
    nb = R.ret_chunkwise_prepare_workspace_bytes(B, N, H, dk, dv, chunk, torch.bfloat16, xpos)
    assert nb > 0
    ws = torch.full((nb,), 0xCD, dtype=torch.uint8, device="cuda")
    R.ret_chunkwise_prepare(qd, kd, g, chunk, ws, dv, xpos=xpos, pos_offset=pos_offset)
    return R.ret_forward_chunkwise_prepared(qd, kd, vd, g, chunk, ws, final_state=fs, initial_state=init,
                                            out_dtype=out_dtype, xpos=xpos, pos_offset=pos_offset,
                                            want_final_state=True)


def test_two_pass_equals_one_call():
    """prepare + prepared is the workspace call split in two (the scores pass,
    then the tensor-core kernel on its output): identical bits."""
    q, k, v = qkv(83, 2, 300, 3, 256, 128, 1 / 16)
    g = gamma_schedule(3)
    a, fa = run_ws(q, k, v, g, 128, out_dtype=torch.float32, xpos=True, pos_offset=5, want_final_state=True)
    b, fb = run_two_pass(dev(q), dev(k), dev(v), g, 128, pos_offset=5)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    assert torch.equal(a, b) and torch.equal(fa, fb)


@pytest.mark.parametrize("N,split,dk,dv,xpos,in_place", [
    (300, 128, 256, 128, True, False),     # split on a chunk boundary
    (300, 77, 128, 64, False, False),      # ragged: both calls end in a partial chunk
    (1100, 513, 256, 512, True, True),     # final_state written over initial_state
    (260, 1, 256, 64, True, False),        # a one-token first call
])
def test_continuation_from_state_matches_whole_sequence(N, split, dk, dv, xpos, in_place):
    """Two calls, the second starting from the first's final state at position
    `split`, reproduce the oracle's recurrence over the whole sequence."""
    B, H = 2, 2
    q, k, v = qkv(90 + split, B, N, H, dk, dv, dk ** -0.5)
    g = gamma_schedule(H)
    qd, kd, vd = dev(q), dev(k), dev(v)
    o1, s1 = run_two_pass(qd[:, :split].contiguous(), kd[:, :split].contiguous(), vd[:, :split].contiguous(), g,
                          128, xpos=xpos)
    s1_copy = s1.clone()
    o2, s2 = run_two_pass(qd[:, split:].contiguous(), kd[:, split:].contiguous(), vd[:, split:].contiguous(), g,
                          128, init=s1, fs=s1 if in_place else None, pos_offset=split, xpos=xpos)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    if not in_place:
        assert torch.equal(s1, s1_copy)          # the initial state is only read
    qr, kr = rotated(q, k, xpos)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    got = np.concatenate([host64(o1), host64(o2)], axis=1)
    assert err_out(got, ref) < TOL_BF16
    assert err_state(host64(s2), S) < TOL_BF16


def test_ws_scaled_gamma_schedule():
    """The larger models' decay schedule (1 - gamma log-spaced from 1/32 to
    1/512) through the same path, 16 heads."""
    q, k, v = qkv(83, 1, 1000, 16, 256, 128, 256 ** -0.5)
    g = gamma_schedule_scaled(16)
    out, fs = run_ws(q, k, v, g, 128, out_dtype=torch.float32, xpos=True, want_final_state=True)
    R.ret_check_device_error()
    qr, kr = rotated(q, k, True)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    assert err_out(host64(out), ref) < TOL_BF16
    assert err_state(host64(fs), S) < TOL_BF16


@pytest.mark.parametrize("B,N,H,dv,chunk,xpos,off", [
    (4, 2048, 8, 64, 64, True, 0),       # the pages' cost-analysis shape (d_model 512, 8 heads of 64)
    (1, 300, 2, 128, 64, False, 0),      # ragged, no rotation
    (2, 513, 3, 64, 128, True, 77),      # chunk 128, a position offset
])
def test_ws_d64_padded(B, N, H, dv, chunk, xpos, off):
    """d_k = 64 on the tensor-core path, zero-padded to 128 (rotation at the
    caller's d_k; states with 64 rows)."""
    dk = 64
    q, k, v = qkv(84 + N, B, N, H, dk, dv, dk ** -0.5)
    g = gamma_schedule(H)
    assert R.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, chunk, torch.bfloat16, xpos) > 0
    out, fs = run_ws(q, k, v, g, chunk, out_dtype=torch.float32, xpos=xpos, pos_offset=off, want_final_state=True)
    R.ret_check_device_error()
    assert fs.shape == (B, H, dk, dv)
    qr, kr = rotated(q, k, xpos, off)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    assert err_out(host64(out), ref) < TOL_BF16
    assert err_state(host64(fs), S) < TOL_BF16


def test_ws_d64_continuation():
    """Two calls of the prepared path at d_k = 64 handing the 64-row state on."""
    B, N, H, dk, dv, split = 1, 400, 2, 64, 128, 200
    q, k, v = qkv(85, B, N, H, dk, dv, dk ** -0.5)
    g = gamma_schedule(H)
    qd, kd, vd = dev(q), dev(k), dev(v)
    S = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    outs = []
    for lo, hi, init in ((0, split, None), (split, N, S)):
        n = hi - lo
        nb = R.ret_chunkwise_prepare_workspace_bytes(B, n, H, dk, dv, 64, torch.bfloat16, True)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        qs, ks, vs = (t[:, lo:hi].contiguous() for t in (qd, kd, vd))
        R.ret_chunkwise_prepare(qs, ks, g, 64, ws, dv, xpos=True, pos_offset=lo)
        o, _ = R.ret_forward_chunkwise_prepared(qs, ks, vs, g, 64, ws, out_dtype=torch.float32, xpos=True,
                                                pos_offset=lo, initial_state=init, final_state=S)
        outs.append(host64(o))
    torch.cuda.synchronize()
    R.ret_check_device_error()
    qr, kr = rotated(q, k, True)
    ref, Sref = oracle.retention_recurrent(qr, kr, v.f64, g)
    assert err_out(np.concatenate(outs, axis=1), ref) < TOL_BF16
    assert err_state(host64(S), Sref) < TOL_BF16


def test_ws_long_sequence_32k():
    """32768 tokens (256 chunks in sequence per CTA) with the fastest and the
    slowest decay of the schedule: the fp32 state and its bf16 read-out copy
    carried across the whole sequence, every output and the final state
    against the oracle."""
    B, N, H, dk, dv = 1, 32768, 2, 256, 256
    q, k, v = qkv(86, B, N, H, dk, dv, dk ** -0.5)
    g = np.array([1 - 2.0 ** -5, 1 - 2.0 ** -12])
    out, fs = run_ws(q, k, v, g, 128, out_dtype=torch.float32, xpos=True, want_final_state=True)
    R.ret_check_device_error()
    qr, kr = rotated(q, k, True)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    assert err_out(host64(out), ref) < TOL_BF16
    assert err_state(host64(fs), S) < TOL_BF16


def test_ws_repeatable_under_memory_contention():
    """Every tile is consumed only after its own TMA barrier: 60 calls at
    4096 tokens x 16 heads (d_k 256, d_v 512) while a second stream keeps
    copying 512 MiB (the loads land late and in varying order) give the same
    bits every time, and the bits of the first call made on an idle GPU."""
    B, N, H, dk, dv = 1, 4096, 16, 256, 512
    gen = torch.Generator(device="cuda").manual_seed(87)
    q = (torch.randn((B, N, H, dk), generator=gen, device="cuda") * dk ** -0.5).to(torch.bfloat16)
    k = (torch.randn((B, N, H, dk), generator=gen, device="cuda") * dk ** -0.5).to(torch.bfloat16)
    v = torch.randn((B, N, H, dv), generator=gen, device="cuda").to(torch.bfloat16)
    g = gamma_schedule(H)
    nb = R.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, 128, torch.bfloat16, True)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    ref, fref = R.ret_forward_chunkwise_ws(q, k, v, g, 128, ws, xpos=True, want_final_state=True)
    torch.cuda.synchronize()
    src = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    dst = torch.empty_like(src)
    side = torch.cuda.Stream()
    outs = [(torch.empty_like(ref), torch.empty_like(fref)) for _ in range(4)]
    for i in range(60):
        with torch.cuda.stream(side):
            for _ in range(2):
                dst.copy_(src)
        o, f = outs[i % 4]
        R.ret_forward_chunkwise_ws(q, k, v, g, 128, ws, out=o, final_state=f, xpos=True)
        if i % 4 == 3:
            torch.cuda.synchronize()
            for o2, f2 in outs:
                assert torch.equal(o2, ref) and torch.equal(f2, fref), i
    R.ret_check_device_error()
