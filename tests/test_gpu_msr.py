"""GPU parity of the MultiScaleRetention layer (tcgen05 GEMMs with the fused
projection epilogue, chunkwise retention, GroupNorm + swish gate, output
projection) and of its GEMM, against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from oracle import msr as omsr
from retention_inputs import C5, gamma_schedule, make_tensor, msr_input, msr_weights
from tests.helpers import TOL_BF16, dev, host64

pytestmark = pytest.mark.gpu

R = None


@pytest.fixture(scope="module", autouse=True)
def lib():
    global R
    import linear_recurrent_sequence_chunkwise_b200 as mod
    R = mod
    yield mod
    mod.ret_check_device_error()


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 512, 192), (8192, 2048, 4096), (77, 40, 24)])
@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16])
def test_linear_matches_oracle(M, N, K, odt):
    x = make_tensor(90, 1, (M, K), "bf16")
    w = make_tensor(90, 2, (K, N), "bf16", 0.05)
    y = R.ret_linear_bf16(dev(x), dev(w), out_dtype=odt)
    torch.cuda.synchronize()
    ref = omsr.project(x.f64, w.f64)
    got = host64(y)
    e = rel(got, ref)
    assert e < (2e-6 * np.sqrt(K) + 1e-6 if odt == torch.float32 else 5e-3), e
    # the first rows element by element (fp32 accumulation over K terms)
    if odt == torch.float32:
        bound = 2 ** -22 * K * np.abs(x.f64[:4]) @ np.abs(w.f64) + 1e-6
        assert (np.abs(got[:4] - ref[:4]) <= bound).all()


def msr_case(B, N, dm, H, dk, dv, seed, xpos=True):
    x = make_tensor(seed, 4, (B, N, dm), "bf16")
    W = {"wq": make_tensor(seed, 5, (dm, H * dk), "bf16", 0.02), "wk": make_tensor(seed, 6, (dm, H * dk), "bf16", 0.02),
         "wv": make_tensor(seed, 7, (dm, H * dv), "bf16", 0.02), "wg": make_tensor(seed, 8, (dm, H * dv), "bf16", 0.02),
         "wo": make_tensor(seed, 9, (H * dv, dm), "bf16", 0.02)}
    return x, W


@pytest.mark.parametrize("B,N,dm,H,dk,dv,xpos", [
    (1, 300, 256, 2, 128, 256, True),
    (2, 256, 512, 2, 256, 512, True),
    (1, 200, 256, 1, 128, 128, False),
])
def test_msr_small_matches_oracle(B, N, dm, H, dk, dv, xpos):
    x, W = msr_case(B, N, dm, H, dk, dv, 91, xpos)
    g = gamma_schedule(H)
    ks = dk ** -0.5
    out = R.ret_msr_forward(dev(x), *(dev(W[n]) for n in ("wq", "wk", "wv", "wg", "wo")), g, H=H, chunk=128,
                            k_scale=ks, eps=1e-5, xpos=xpos, out_dtype=torch.float32)
    R.ret_check_device_error()
    if xpos:
        ref = omsr.msr_forward(x.f64, *(W[n].f64 for n in ("wq", "wk", "wv", "wg", "wo")), gammas=g, H=H,
                               k_scale=ks, eps=1e-5)
    else:
        # the oracle without rotation: same composition, rotation by angle 0
        q = omsr.project(x.f64, W["wq"].f64).reshape(B, N, H, dk)
        k = omsr.project(x.f64, W["wk"].f64).reshape(B, N, H, dk) * ks
        v = omsr.project(x.f64, W["wv"].f64).reshape(B, N, H, dv)
        gg = omsr.project(x.f64, W["wg"].f64).reshape(B, N, H, dv)
        y, _ = oracle.retention_recurrent(q, k, v, g)
        z = omsr.swish(gg) * omsr.group_norm_heads(y, 1e-5)
        ref = omsr.project(z.reshape(B, N, H * dv), W["wo"].f64)
    got = host64(out)
    for b in range(B):
        assert rel(got[b], ref[b]) < TOL_BF16


def test_msr_layer_workload():
    """The full MSR layer workload: X [2, 4096, 2048], H 8, d_k 256, d_v 512,
    xPos, chunk 128; every output against the oracle."""
    w = C5
    x = msr_input(w)
    W = msr_weights(w)
    out = R.ret_msr_forward(dev(x), *(dev(W[n]) for n in ("wq", "wk", "wv", "wg", "wo")), w.gammas, H=w.H,
                            chunk=w.chunk, k_scale=w.qk_scale, eps=w.gn_eps, xpos=True, out_dtype=torch.float32)
    R.ret_check_device_error()
    ref = omsr.msr_forward(x.f64, *(W[n].f64 for n in ("wq", "wk", "wv", "wg", "wo")), gammas=w.gammas, H=w.H,
                           k_scale=w.qk_scale, eps=w.gn_eps)
    got = host64(out)
    for b in range(w.B):
        assert rel(got[b], ref[b]) < TOL_BF16
