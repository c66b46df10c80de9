"""GPU parity of the CUDA-core paths against the fp64 oracle, through the
C ABI: rotation, the fp32 chunkwise kernel (full fp32 workload and ragged
shapes), the parallel and recurrent cross-check forms and the decode step."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import C1, C2, C3, C4, make_tensor, gamma_schedule
from tests.helpers import TOL_BF16, TOL_F32, dev, err_out, err_state, host64, max_rel_l2, tol_for

pytestmark = pytest.mark.gpu

R = None


@pytest.fixture(scope="module", autouse=True)
def lib():
    global R
    import linear_recurrent_sequence_chunkwise_b200 as mod
    R = mod
    assert torch.cuda.is_available()
    yield mod


def qkv(seed, B, N, H, dk, dv, dtype, scale=1.0):
    return (make_tensor(seed, 1, (B, N, H, dk), dtype, scale), make_tensor(seed, 2, (B, N, H, dk), dtype, scale),
            make_tensor(seed, 3, (B, N, H, dv), dtype))


def oracle_ref(q, k, v, gammas, xpos=False, pos_offset=0, theta=10000.0):
    qf, kf = q.f64, k.f64
    if xpos:
        qf = oracle.xpos_rotate(qf, pos_offset, theta)
        kf = oracle.xpos_rotate(kf, pos_offset, theta)
    return oracle.retention_recurrent(qf, kf, v.f64, gammas)


# ------------------------------------------------------------------ rotation

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape,off", [((2, 37, 3, 16), 0), ((1, 300, 2, 64), 5000), ((1, 9, 1, 2), 7)])
def test_rotate_matches_oracle(dtype, shape, off):
    x = make_tensor(11, 1, shape, dtype)
    xd = dev(x)
    R.ret_xpos_rotate(xd, pos_offset=off)
    torch.cuda.synchronize()
    ref = oracle.xpos_rotate(x.f64, off)
    tol = 2e-6 if dtype == "f32" else 4e-3
    assert max_rel_l2(host64(xd), ref, (0, 2)) < tol


# ------------------------------------------------------ fp32 chunkwise path

def test_chunkwise_fp32_workload():
    w = C1
    q, k, v = w.qkv()
    out, fs = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), w.gammas, w.chunk, want_final_state=True)
    torch.cuda.synchronize()
    ref, S = oracle_ref(q, k, v, w.gammas)
    assert err_out(host64(out), ref) < TOL_F32
    assert err_state(host64(fs), S) < TOL_F32


@pytest.mark.parametrize("B,N,H,dk,dv,chunk,xpos", [
    (1, 1, 1, 16, 16, 16, False),     # a single token
    (2, 37, 3, 16, 16, 16, False),    # ragged tail chunk
    (1, 50, 2, 12, 20, 7, True),      # odd chunk, dv not a multiple of the tile
    (1, 64, 1, 32, 96, 64, True),     # chunk == N, two dv tiles
    (3, 33, 2, 8, 8, 40, False),      # chunk > N
])
def test_chunkwise_fp32_ragged(B, N, H, dk, dv, chunk, xpos):
    q, k, v = qkv(21, B, N, H, dk, dv, "f32", 0.5)
    g = np.array([0.5, 0.9, 0.999][:H])
    out, fs = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), g, chunk, xpos=xpos, pos_offset=3,
                                      want_final_state=True)
    torch.cuda.synchronize()
    ref, S = oracle_ref(q, k, v, g, xpos, 3)
    assert err_out(host64(out), ref) < TOL_F32
    assert err_state(host64(fs), S) < TOL_F32


@pytest.mark.parametrize("gam", [0.0, 1.0, 1e-30])
def test_chunkwise_fp32_degenerate_gamma(gam):
    q, k, v = qkv(22, 1, 40, 2, 16, 16, "f32", 0.5)
    g = np.array([gam, gam])
    out, fs = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), g, 16, want_final_state=True)
    torch.cuda.synchronize()
    ref, S = oracle_ref(q, k, v, g)
    assert err_out(host64(out), ref) < TOL_F32
    assert err_state(host64(fs), S) < TOL_F32


def test_chunkwise_bf16_small_cost_model_shape_on_cuda_cores():
    """bf16 inputs on a shape the tensor-core kernel does not take (dk 32)."""
    q, k, v = qkv(23, 2, 130, 4, 32, 32, "bf16", 32 ** -0.5)
    g = gamma_schedule(4)
    for odt in (torch.float32, torch.bfloat16):
        out = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), g, 32, xpos=True, out_dtype=odt)
        torch.cuda.synchronize()
        ref, _ = oracle_ref(q, k, v, g, True)
        assert err_out(host64(out), ref) < TOL_BF16


# -------------------------------------------- parallel and recurrent forms

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_parallel_and_recurrent_match_oracle(dtype):
    q, k, v = qkv(24, 2, 97, 3, 32, 48, dtype, 32 ** -0.5)
    g = np.array([0.9, 0.99, 1.0])
    ref, S = oracle_ref(q, k, v, g, True, 11)
    par = R.ret_forward_parallel(dev(q), dev(k), dev(v), g, out_dtype=torch.float32, xpos=True, pos_offset=11)
    rec, fs = R.ret_forward_recurrent(dev(q), dev(k), dev(v), g, out_dtype=torch.float32, xpos=True,
                                      pos_offset=11, want_final_state=True)
    torch.cuda.synchronize()
    tol = tol_for(dtype)
    assert err_out(host64(par), ref) < tol
    assert err_out(host64(rec), ref) < tol
    assert err_state(host64(fs), S) < tol


def test_cost_model_workload_cuda_core_forms():
    """The d_model-512 cost-analysis workload through the fp32 CUDA-core
    chunkwise kernel, the parallel form and the recurrent form."""
    w = C2
    q, k, v = w.qkv()
    ref, S = oracle_ref(q, k, v, w.gammas, True)
    qd, kd, vd = dev(q), dev(k), dev(v)
    rec, fs = R.ret_forward_recurrent(qd, kd, vd, w.gammas, out_dtype=torch.float32, xpos=True,
                                      want_final_state=True)
    par = R.ret_forward_parallel(qd, kd, vd, w.gammas, out_dtype=torch.float32, xpos=True)
    torch.cuda.synchronize()
    assert err_out(host64(rec), ref) < TOL_BF16
    assert err_state(host64(fs), S) < TOL_BF16
    assert err_out(host64(par), ref) < TOL_BF16


def test_long_sequence_recurrent_form():
    """The 8k-token, d_k 256 / d_v 512 workload through the GPU recurrent
    form, against the oracle on every head."""
    w = C3
    q, k, v = w.qkv()
    ref, S = oracle_ref(q, k, v, w.gammas, True)
    rec, fs = R.ret_forward_recurrent(dev(q), dev(k), dev(v), w.gammas, out_dtype=torch.float32, xpos=True,
                                      want_final_state=True)
    torch.cuda.synchronize()
    assert err_out(host64(rec), ref) < TOL_BF16
    assert err_state(host64(fs), S) < TOL_BF16


# -------------------------------------------------------------- decode step

@pytest.mark.parametrize("dtype,B,H,dk,dv", [("f32", 3, 2, 16, 16), ("bf16", 2, 3, 256, 512), ("f32", 1, 1, 7, 132)])
def test_decode_steps_match_oracle(dtype, B, H, dk, dv):
    g = np.array([0.9, 0.99, 0.999][:H])
    s0 = make_tensor(30, 9, (B, H, dk, dv), "f32")
    state = dev(s0).clone()
    S = s0.f64.copy()
    for t in range(5):
        q = make_tensor(31 + t, 1, (B, H, dk), dtype)
        k = make_tensor(31 + t, 2, (B, H, dk), dtype)
        v = make_tensor(31 + t, 3, (B, H, dv), dtype)
        out = R.ret_decode_step(dev(q), dev(k), dev(v), g, state)
        o_ref, S = oracle.decode_step(q.f64, k.f64, v.f64, g, S)
        torch.cuda.synchronize()
        assert max_rel_l2(host64(out), o_ref, (0, 1)) < TOL_F32
    assert err_state(host64(state), S) < TOL_F32


def _picked(x, picks):
    """Stack the (batch, head) slices ``picks`` of x [B, N, H, d] (or
    [B, H, d]) along the head axis of a batch of one.  x is an array or a
    seeded Tensor (widened slice by slice)."""
    get = (lambda i: x.f64_at(i)) if hasattr(x, "f64_at") else (lambda i: x[i])
    if len(x.shape) == 4:
        return np.stack([get((b, slice(None), h)) for b, h in picks], axis=1)[None]
    return np.stack([get((b, h)) for b, h in picks], axis=0)[None]


def test_decode_workload_sampled():
    """The whole decode workload: 64 sequences x 16 heads of 256 x 512 fp32
    states, prefilled by the chunkwise forward (chunk 128) over the seeded
    1024-token prompt, then all 512 decode steps with fresh seeded q, k, v.
    Sampled (batch, head) slices against the oracle: the prefill state,
    every step's output and the final state."""
    w = C4
    q, k, v = w.qkv()
    _, state = R.ret_forward_chunkwise(dev(q), dev(k), dev(v), w.gammas, w.chunk, out_dtype=torch.float32,
                                       want_final_state=True)
    picks = [(0, 0), (5, 7), (63, 15), (31, 3)]
    g = np.array([w.gammas[h] for _, h in picks])
    _, S_ref = oracle.retention_recurrent(_picked(q, picks), _picked(k, picks), _picked(v, picks), g)
    st = state.cpu().double().numpy()
    assert max_rel_l2(np.stack([st[b, h] for b, h in picks])[None], S_ref, (0, 1)) < TOL_BF16
    worst = 0.0
    for s in range(w.decode_steps):
        qs, ks, vs = w.decode_qkv(s)
        out = R.ret_decode_step(dev(qs), dev(ks), dev(vs), w.gammas, state).cpu().double().numpy()
        o_ref, S_ref = oracle.decode_step(_picked(qs, picks), _picked(ks, picks), _picked(vs, picks), g, S_ref)
        worst = max(worst, max_rel_l2(_picked(out, picks), o_ref, (0, 1)))
    assert worst < TOL_BF16, worst
    st = state.cpu().double().numpy()
    assert max_rel_l2(np.stack([st[b, h] for b, h in picks])[None], S_ref, (0, 1)) < TOL_BF16
