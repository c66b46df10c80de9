"""The C ABI under CUDA-graph capture: calls enqueue only stream work (no
synchronisation, no allocation), so a captured sequence replays correctly --
the recurrent path as a graph of decode steps, and the two-kernel chunkwise
forward."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import gamma_schedule, make_tensor
from tests.helpers import TOL_BF16, dev, err_out, err_state, host64

pytestmark = pytest.mark.gpu


def test_decode_steps_replayed_from_a_graph():
    import linear_recurrent_sequence_chunkwise_b200 as R
    B, T, H, dk, dv = 4, 16, 2, 128, 128
    q = make_tensor(501, 1, (B, T, H, dk), "bf16", dk ** -0.5)
    k = make_tensor(501, 2, (B, T, H, dk), "bf16", dk ** -0.5)
    v = make_tensor(501, 3, (B, T, H, dv), "bf16")
    g = gamma_schedule(H)
    qs, ks, vs = ([dev(x)[:, t].contiguous() for t in range(T)] for x in (q, k, v))
    S = torch.zeros((B, H, dk, dv), dtype=torch.float32, device="cuda")
    outs = [torch.empty((B, H, dv), dtype=torch.float32, device="cuda") for _ in range(T)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for t in range(T):
            R.ret_decode_step(qs[t], ks[t], vs[t], g, S, out=outs[t])
    torch.cuda.synchronize()
    for rep in range(2):            # replay twice from the zero state: same result
        S.zero_()
        graph.replay()
        torch.cuda.synchronize()
        R.ret_check_device_error()
        got = np.stack([host64(o) for o in outs], axis=1)
        ref, Sref = oracle.retention_recurrent(q.f64, k.f64, v.f64, g)
        assert err_out(got, ref) < TOL_BF16
        assert err_state(host64(S), Sref) < TOL_BF16


def test_chunkwise_forward_replayed_from_a_graph():
    import linear_recurrent_sequence_chunkwise_b200 as R
    B, N, H, dk, dv = 1, 700, 2, 256, 128
    q = make_tensor(502, 1, (B, N, H, dk), "bf16", dk ** -0.5)
    k = make_tensor(502, 2, (B, N, H, dk), "bf16", dk ** -0.5)
    v = make_tensor(502, 3, (B, N, H, dv), "bf16")
    g = gamma_schedule(H)
    qd, kd, vd = dev(q), dev(k), dev(v)
    nb = R.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, 128, torch.bfloat16, True)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    out = torch.empty((B, N, H, dv), dtype=torch.float32, device="cuda")
    fs = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    R.ret_forward_chunkwise_ws(qd, kd, vd, g, 128, ws, out=out, final_state=fs, xpos=True)  # warm-up outside
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        R.ret_forward_chunkwise_ws(qd, kd, vd, g, 128, ws, out=out, final_state=fs, xpos=True)
    out.zero_()
    fs.zero_()
    graph.replay()
    torch.cuda.synchronize()
    R.ret_check_device_error()
    ref, Sref = oracle.retention_recurrent(oracle.xpos_rotate(q.f64), oracle.xpos_rotate(k.f64), v.f64, g)
    assert err_out(host64(out), ref) < TOL_BF16
    assert err_state(host64(fs), Sref) < TOL_BF16


def test_backward_replayed_from_a_graph():
    """The backward forks its dk passes onto a second stream and joins back
    with events: under capture that is a fork/join in the graph."""
    import linear_recurrent_sequence_chunkwise_b200 as R
    B, N, H, dk, dv = 1, 300, 2, 128, 256
    q = make_tensor(503, 1, (B, N, H, dk), "bf16", dk ** -0.5)
    k = make_tensor(503, 2, (B, N, H, dk), "bf16", dk ** -0.5)
    v = make_tensor(503, 3, (B, N, H, dv), "bf16")
    do = make_tensor(503, 4, (B, N, H, dv), "bf16")
    g = gamma_schedule(H)
    qd, kd, vd, dod = dev(q), dev(k), dev(v), dev(do)
    nb = R.ret_backward_workspace_bytes(B, N, H, dk, dv, 128, torch.bfloat16, True)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    dq = torch.empty((B, N, H, dk), dtype=torch.float32, device="cuda")
    dkk = torch.empty_like(dq)
    dvv = torch.empty((B, N, H, dv), dtype=torch.float32, device="cuda")
    R.ret_backward_chunkwise(qd, kd, vd, dod, g, 128, workspace=ws, dq=dq, dk=dkk, dv=dvv, xpos=True)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        R.ret_backward_chunkwise(qd, kd, vd, dod, g, 128, workspace=ws, dq=dq, dk=dkk, dv=dvv, xpos=True)
    for t in (dq, dkk, dvv):
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    R.ret_check_device_error()
    ref = oracle.retention_backward(q.f64, k.f64, v.f64, do.f64, g, xpos=True)
    for name, a, r in zip(("dq", "dk", "dv"), (dq, dkk, dvv), ref):
        assert err_out(host64(a), r) < TOL_BF16, name
