"""The allocation-free chunkwise entry point (ret_forward_chunkwise_noalloc).

Some callers cannot allocate device memory when they call the library (a
plug-in inside a framework that owns all device memory, a service that fixes
its footprint at start-up).  This entry point runs the two kernels of the
workspace path (the rotation / zeta pass, then the tensor-core kernel) on a
fixed device array inside the library instead of a caller-provided buffer.

The test calls it through the C ABI on two calls in a row with different
inputs (the array keeps the first call's contents) and compares it with the
entry point that allocates (ret_forward_chunkwise) and with the fp64 oracle,
within the bf16 bar of the other tests, for each layout of the scratch:
rotated queries and keys (xpos), keys only (no xpos), and the d_k = 64 shape
padded to 128 with the queries always copied.  Two calls on the same inputs
give the same bits.  It also checks that problems too large for the array are
refused.  The file name sorts last so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import gamma_schedule, make_tensor
from tests.helpers import TOL_BF16, dev, err_out, err_state, host64

pytestmark = pytest.mark.gpu


def _scratch_bytes(B, N, H, dk, xpos):
    """What the array must hold: k' (and the copied queries) at the kernel's d_k."""
    dkk = 128 if dk == 64 else dk
    copied = xpos or dk == 64
    return B * N * H * dkk * 2 * (2 if copied else 1)


@pytest.mark.parametrize("B,N,H,dk,dv,chunk,xpos", [
    (1, 2000, 8, 256, 256, 128, True),
    (2, 1500, 4, 256, 128, 128, False),
    (4, 1000, 8, 64, 64, 64, True),
])
def test_noalloc_matches_the_allocating_entry_point_on_two_calls(B, N, H, dk, dv, chunk, xpos):
    import linear_recurrent_sequence_chunkwise_b200 as R
    g = gamma_schedule(H)
    assert _scratch_bytes(B, N, H, dk, xpos) <= R.ret_chunkwise_noalloc_max_bytes()
    for call, seed in enumerate((301, 302)):
        qt = make_tensor(seed, 1, (B, N, H, dk), "bf16", dk ** -0.5)
        kt = make_tensor(seed, 2, (B, N, H, dk), "bf16", dk ** -0.5)
        vt = make_tensor(seed, 3, (B, N, H, dv), "bf16")
        q, k, v = dev(qt), dev(kt), dev(vt)
        out = torch.empty((B, N, H, dv), dtype=torch.float32, device="cuda")
        fs = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
        R.ret_forward_chunkwise_noalloc(q, k, v, g, chunk, out=out, final_state=fs, xpos=xpos, pos_offset=call)
        R.ret_check_device_error()
        again = torch.empty_like(out)
        R.ret_forward_chunkwise_noalloc(q, k, v, g, chunk, out=again, xpos=xpos, pos_offset=call)
        ref, fref = R.ret_forward_chunkwise(q, k, v, g, chunk, out_dtype=torch.float32, xpos=xpos, pos_offset=call,
                                            want_final_state=True)
        R.ret_check_device_error()
        assert torch.equal(out, again)
        assert err_out(host64(out), host64(ref)) < TOL_BF16
        assert err_state(host64(fs), host64(fref)) < TOL_BF16
        qf, kf = qt.f64, kt.f64
        if xpos:
            qf, kf = oracle.xpos_rotate(qf, call), oracle.xpos_rotate(kf, call)
        o_ref, s_ref = oracle.retention_recurrent(qf, kf, vt.f64, g)
        assert err_out(host64(out), o_ref) < TOL_BF16
        assert err_state(host64(fs), s_ref) < TOL_BF16


@pytest.mark.parametrize("B,N,H,dk,dv,xpos", [
    (1, 16384, 16, 256, 64, True),    # 256 MiB of rotated queries and keys
    (1, 4096, 16, 256, 64, False),    # exactly 32 MiB of keys: accepted
    (4, 4097, 8, 64, 64, False),      # d_k 64 padded to 128, queries copied: just above 64 MiB
])
def test_noalloc_limit(B, N, H, dk, dv, xpos):
    import linear_recurrent_sequence_chunkwise_b200 as R
    q = torch.zeros((B, N, H, dk), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((B, N, H, dv), dtype=torch.bfloat16, device="cuda")
    fits = _scratch_bytes(B, N, H, dk, xpos) <= R.ret_chunkwise_noalloc_max_bytes()
    if fits:
        out = R.ret_forward_chunkwise_noalloc(q, q.clone(), v, gamma_schedule(H), 128, xpos=xpos)
        R.ret_check_device_error()
        assert torch.count_nonzero(out) == 0
        return
    with pytest.raises(R.RetentionError) as e:
        R.ret_forward_chunkwise_noalloc(q, q.clone(), v, gamma_schedule(H), 128, xpos=xpos)
    assert e.value.status == R.RET_ERR_INVALID_ARG
    assert "scratch" in str(e.value)
