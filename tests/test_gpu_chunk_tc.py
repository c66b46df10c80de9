"""GPU parity of the tensor-core chunkwise forward (bf16 in, fp32
accumulate) against the fp64 oracle through the C ABI: small multi-chunk and
ragged shapes, the degenerate decays, the 8k-token d_k 256 / d_v 512
workload on every head, and agreement of the chunkwise, parallel and
recurrent GPU paths with each other."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import C3, C4, C5, gamma_schedule, make_tensor
from tests.helpers import TOL_BF16, bf16_bound_check, dev, err_out, err_state, host64, max_rel_l2

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


def ref_of(q, k, v, g, xpos, off=0):
    qf, kf = rotated(q, k, xpos, off)
    return oracle.retention_recurrent(qf, kf, v.f64, g)


@pytest.mark.parametrize("B,N,H,dk,dv,xpos,off", [
    (1, 128, 1, 256, 64, True, 0),       # exactly one chunk
    (2, 300, 2, 256, 128, True, 0),      # two full chunks and a 44-row tail
    (1, 1, 2, 256, 64, True, 9),         # a single token
    (1, 77, 1, 128, 64, False, 0),       # one partial chunk, d_k 128
    (2, 513, 3, 128, 192, True, 1000),   # tail of 1 row, three d_v tiles
    (1, 1024, 2, 256, 512, True, 0),     # d_v 512 (eight tiles)
])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_chunkwise_tc_small(B, N, H, dk, dv, xpos, off, out_dtype):
    q, k, v = qkv(40 + N, B, N, H, dk, dv, dk ** -0.5)
    g = gamma_schedule(H)
    out, fs = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), g, 128, out_dtype=out_dtype, xpos=xpos,
                                      pos_offset=off, want_final_state=True)
    R.ret_check_device_error()
    qr, kr = rotated(q, k, xpos, off)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    # every shape: element-wise rounding bound; from 256 tokens on also the relative L2 bar
    bf16_bound_check(host64(out), host64(fs), qr, kr, v.f64, g, ref, S, out_dtype == torch.bfloat16)
    if N >= 256:
        assert err_out(host64(out), ref) < TOL_BF16
        assert err_state(host64(fs), S) < TOL_BF16


@pytest.mark.parametrize("gam", [1.0, 0.75, 0.6, 0.0])
def test_chunkwise_degenerate_decays(gam):
    """gamma 1 and 0.75 (0.75^128 = 2^-53) run on the tensor cores with the
    decay anchored at the chunk's last row; 0.6 (0.6^128 below 2^-60, 0.6^64
    above 2^-100) with the anchor at row 63; gamma 0 is left to the recurrent
    kernel while the other head stays on the tensor cores; all must match the
    oracle."""
    q, k, v = qkv(50, 1, 260, 2, 256, 64, 1 / 16)
    g = np.array([gam, 0.99])
    out, fs = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), g, 128, out_dtype=torch.float32, xpos=True,
                                      want_final_state=True)
    R.ret_check_device_error()
    qr, kr = rotated(q, k, True)
    ref, S = oracle.retention_recurrent(qr, kr, v.f64, g)
    bf16_bound_check(host64(out), host64(fs), qr, kr, v.f64, g, ref, S, False)


def test_long_sequence_workload_all_heads():
    """B=1, N=8192, H=16, d_k 256, d_v 512, xPos, chunk 128, with the final
    state: every head against the oracle, for both output dtypes."""
    w = C3
    q, k, v = w.qkv()
    ref, S = ref_of(q, k, v, w.gammas, True)
    qd, kd, vd = dev(q), dev(k), dev(v)
    for odt in (torch.bfloat16, torch.float32):
        out, fs = R.ret_forward_chunkwise(qd, kd, vd, w.gammas, w.chunk, out_dtype=odt, xpos=True,
                                          want_final_state=True)
        R.ret_check_device_error()
        assert err_out(host64(out), ref) < TOL_BF16
        assert err_state(host64(fs), S) < TOL_BF16


def test_gpu_forms_agree():
    """Chunkwise (tensor cores), parallel and recurrent GPU paths agree with
    each other within the bf16 bound, on a 2-sequence, 1000-token shape."""
    q, k, v = qkv(60, 2, 1000, 4, 256, 128, 1 / 16)
    g = gamma_schedule(4)
    qd, kd, vd = dev(q), dev(k), dev(v)
    chk, fs_c = R.ret_forward_chunkwise(qd, kd, vd, g, 128, out_dtype=torch.float32, xpos=True,
                                        want_final_state=True)
    par = R.ret_forward_parallel(qd, kd, vd, g, out_dtype=torch.float32, xpos=True)
    rec, fs_r = R.ret_forward_recurrent(qd, kd, vd, g, out_dtype=torch.float32, xpos=True, want_final_state=True)
    torch.cuda.synchronize()
    c, p_, r_ = host64(chk), host64(par), host64(rec)
    assert err_out(c, r_) < TOL_BF16
    assert err_out(p_, r_) < TOL_BF16
    assert err_out(c, p_) < TOL_BF16
    assert err_state(host64(fs_c), host64(fs_r)) < TOL_BF16
    ref, S = ref_of(q, k, v, g, True)
    assert err_out(c, ref) < TOL_BF16


def _picked(t, picks):
    return np.stack([t.f64_at((b, slice(None), h)) for b, h in picks], axis=1)[None]


def test_prefill_workload_sampled():
    """The 64-sequence, 1024-token prefill (no xPos) on the tensor cores;
    sampled (batch, head) slices of the output and the final state."""
    w = C4
    q, k, v = w.qkv()
    out, fs = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), w.gammas, w.chunk, out_dtype=torch.float32,
                                      want_final_state=True)
    R.ret_check_device_error()
    picks = [(0, 0), (17, 5), (63, 15), (40, 11)]
    g = np.array([w.gammas[h] for _, h in picks])
    ref, S = oracle.retention_recurrent(_picked(q, picks), _picked(k, picks), _picked(v, picks), g)
    o = out.cpu().numpy()
    got = np.stack([o[b, :, h] for b, h in picks], axis=1)[None].astype(np.float64)
    assert err_out(got, ref) < TOL_BF16
    f = fs.cpu().numpy()
    gs = np.stack([f[b, h] for b, h in picks])[None].astype(np.float64)
    assert err_state(gs, S) < TOL_BF16


def test_msr_core_shape():
    """The retention core at the MSR layer's head shape: B=2, N=4096, H=8,
    d_k 256, d_v 512 with xPos, two sampled heads per sequence."""
    w = C5
    q, k, v = qkv(w.seed, 2, 4096, 8, 256, 512, 1 / 16)
    out = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), w.gammas, 128, out_dtype=torch.float32, xpos=True)
    R.ret_check_device_error()
    picks = [(0, 0), (1, 7), (0, 4), (1, 2)]
    g = np.array([w.gammas[h] for _, h in picks])
    qf = oracle.xpos_rotate(_picked(q, picks))
    kf = oracle.xpos_rotate(_picked(k, picks))
    ref, _ = oracle.retention_recurrent(qf, kf, _picked(v, picks), g)
    o = out.cpu().numpy()
    got = np.stack([o[b, :, h] for b, h in picks], axis=1)[None].astype(np.float64)
    assert err_out(got, ref) < TOL_BF16


def _kernels_launched(fn):
    """Names of the CUDA kernels fn() launches, from torch's profiler (CUPTI);
    None when the profiler records no device activity here."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    names = {e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA}
    return names or None


@pytest.mark.parametrize("slow", [0.5, 0.36])
def test_mixed_decays_stay_on_the_tensor_cores(slow):
    """One fast-decaying head (gamma 0.5 or 0.36: gamma^128 far below 2^-60)
    among heads on the pages' schedule: every head runs on the fused
    tensor-core kernel (the fast one with its decay anchored at row 63), no
    CUDA-core kernel is launched, and the result matches the oracle at the
    workload's bar (RetNet paper summary, multi-scale decay; the pages'
    schedule has no such head, a caller may)."""
    B, N, H, dk, dv = 1, 1000, 4, 256, 128
    q, k, v = qkv(61, B, N, H, dk, dv, dk ** -0.5)
    g = np.array(list(gamma_schedule(H - 1)) + [slow])
    qd, kd, vd = dev(q), dev(k), dev(v)
    res = {}

    def run():
        res["o"], res["s"] = R.ret_forward_chunkwise(qd, kd, vd, g, 128, out_dtype=torch.float32, xpos=True,
                                                     want_final_state=True)
    names = _kernels_launched(run)
    R.ret_check_device_error()
    if names is not None:
        assert any("k_chunkwise_ws" in n for n in names), names
        assert not any("simt" in n for n in names), names
    ref, S = ref_of(q, k, v, g, True)
    assert err_out(host64(res["o"]), ref) < TOL_BF16
    assert err_state(host64(res["s"]), S) < TOL_BF16


def test_very_fast_head_goes_to_the_recurrent_kernel_alone():
    """gamma 0.2 (0.2^64 below 2^-100) is computed token by token while the
    other heads stay on the tensor cores; both kernels run, and every head
    matches the oracle."""
    B, N, H, dk, dv = 2, 300, 3, 128, 64
    q, k, v = qkv(62, B, N, H, dk, dv, dk ** -0.5)
    g = np.array([0.96875, 0.2, 0.99])
    qd, kd, vd = dev(q), dev(k), dev(v)
    res = {}

    def run():
        res["o"], res["s"] = R.ret_forward_chunkwise(qd, kd, vd, g, 128, out_dtype=torch.float32, xpos=True,
                                                     want_final_state=True)
    names = _kernels_launched(run)
    R.ret_check_device_error()
    if names is not None:
        assert any("k_chunkwise_ws" in n for n in names), names
        assert any("k_recurrent_simt" in n for n in names), names
    ref, S = ref_of(q, k, v, g, True)
    assert err_out(host64(res["o"]), ref) < TOL_BF16
    assert err_state(host64(res["s"]), S) < TOL_BF16
