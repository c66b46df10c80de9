"""GPU parity of one RetNet block (LayerNorm, the MSR layer with the residual
in its output projection, LayerNorm, the gelu FFN with the residual in its
second GEMM) against the fp64 oracle's composition, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import msr as omsr
from retention_inputs import C5, ffn_weights, gamma_schedule, make_tensor, msr_input, msr_weights
from tests.helpers import TOL_BF16, dev, host64

pytestmark = pytest.mark.gpu

R = None
NAMES = ("wq", "wk", "wv", "wg", "wo")


@pytest.fixture(scope="module", autouse=True)
def lib():
    global R
    import linear_recurrent_sequence_chunkwise_b200 as mod
    R = mod
    yield mod
    mod.ret_check_device_error()


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


@pytest.mark.parametrize("B,N,dm,H,dk,dv,ln_params", [
    (1, 300, 256, 2, 128, 256, True),      # ragged last chunk, LayerNorm gains and biases
    (2, 256, 512, 2, 256, 512, False),
])
def test_block_small_matches_oracle(B, N, dm, H, dk, dv, ln_params):
    seed = 95
    x = make_tensor(seed, 4, (B, N, dm), "bf16")
    W = {"wq": make_tensor(seed, 5, (dm, H * dk), "bf16", 0.05), "wk": make_tensor(seed, 6, (dm, H * dk), "bf16", 0.05),
         "wv": make_tensor(seed, 7, (dm, H * dv), "bf16", 0.05), "wg": make_tensor(seed, 8, (dm, H * dv), "bf16", 0.05),
         "wo": make_tensor(seed, 9, (H * dv, dm), "bf16", 0.05), "w1": make_tensor(seed, 10, (dm, 2 * dm), "bf16", 0.05),
         "w2": make_tensor(seed, 11, (2 * dm, dm), "bf16", 0.05)}
    ln = {}
    if ln_params:
        for i, n in enumerate(("ln1_gain", "ln1_bias", "ln2_gain", "ln2_bias")):
            base = 1.0 if "gain" in n else 0.0
            t = make_tensor(seed, 20 + i, (dm,), "bf16", 0.2)
            ln[n] = (t, t.f64 + base)
    g = gamma_schedule(H)
    ks = dk ** -0.5
    dev_ln = {n: (dev(t) + (1.0 if "gain" in n else 0.0)).to(torch.bfloat16).contiguous() for n, (t, _) in ln.items()}
    out = R.ret_retnet_block_forward(dev(x), *(dev(W[n]) for n in NAMES), dev(W["w1"]), dev(W["w2"]), g, H=H,
                                     chunk=128, k_scale=ks, out_dtype=torch.float32, **dev_ln)
    R.ret_check_device_error()
    # the oracle takes the bf16 values the device holds
    host_ln = {n: host64(t) for n, t in dev_ln.items()}
    ref = omsr.retnet_block(x.f64, *(W[n].f64 for n in NAMES), W["w1"].f64, W["w2"].f64, gammas=g, H=H,
                            k_scale=ks, ln1=(host_ln.get("ln1_gain"), host_ln.get("ln1_bias")),
                            ln2=(host_ln.get("ln2_gain"), host_ln.get("ln2_bias")))
    got = host64(out)
    for b in range(B):
        assert rel(got[b], ref[b]) < TOL_BF16


def test_block_zero_branches_pass_the_input_through():
    """W_O = 0 and W2 = 0: both residual branches add exactly zero."""
    B, N, dm, H, dk, dv = 1, 200, 256, 2, 128, 256
    x = make_tensor(96, 4, (B, N, dm), "bf16")
    W = {n: torch.zeros(s, dtype=torch.bfloat16, device="cuda") if n in ("wo", "w2") else
         dev(make_tensor(96, 5 + i, s, "bf16", 0.05))
         for i, (n, s) in enumerate((("wq", (dm, H * dk)), ("wk", (dm, H * dk)), ("wv", (dm, H * dv)),
                                     ("wg", (dm, H * dv)), ("wo", (H * dv, dm)), ("w1", (dm, 2 * dm)),
                                     ("w2", (2 * dm, dm))))}
    out = R.ret_retnet_block_forward(dev(x), *(W[n] for n in NAMES), W["w1"], W["w2"], gamma_schedule(H), H=H,
                                     k_scale=dk ** -0.5, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(out, dev(x))


def test_block_workload():
    """The MSR layer workload as a full block: X [2, 4096, 2048], H 8, d_k 256,
    d_v 512, d_ff 4096, xPos, chunk 128; every output against the oracle."""
    w = C5
    x = msr_input(w)
    W = msr_weights(w)
    F = ffn_weights(w)
    out = R.ret_retnet_block_forward(dev(x), *(dev(W[n]) for n in NAMES), dev(F["w1"]), dev(F["w2"]), w.gammas,
                                     H=w.H, chunk=w.chunk, k_scale=w.qk_scale, gn_eps=w.gn_eps,
                                     out_dtype=torch.float32)
    R.ret_check_device_error()
    ref = omsr.retnet_block(x.f64, *(W[n].f64 for n in NAMES), F["w1"].f64, F["w2"].f64, gammas=w.gammas, H=w.H,
                            k_scale=w.qk_scale, gn_eps=w.gn_eps)
    got = host64(out)
    for b in range(w.B):
        assert rel(got[b], ref[b]) < TOL_BF16
