"""The allocation-free chunkwise entry point (ret_forward_chunkwise_noalloc).

Some callers cannot allocate device memory when they call the library (a
plug-in inside a framework that owns all device memory, a service that fixes
its footprint at start-up).  This entry point runs the workspace path on a
fixed device array inside the library instead of a caller-provided buffer.
The test compares it, through the C ABI, with the workspace entry point on
two calls in a row with different inputs (the array keeps the first call's
contents), and checks that a problem too large for the array is refused.
The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from retention_inputs import gamma_schedule, make_tensor
from tests.helpers import TOL_BF16, dev, err_out, err_state, host64

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import linear_recurrent_sequence_chunkwise_b200 as R
    B, N, H, dk, dv = 1, 2000, 8, 256, 256
    g = gamma_schedule(H)
    assert B * N * H * dk * 4 <= R.ret_chunkwise_noalloc_max_bytes()
    for call, seed in enumerate((301, 302)):
        q = dev(make_tensor(seed, 1, (B, N, H, dk), "bf16", dk ** -0.5))
        k = dev(make_tensor(seed, 2, (B, N, H, dk), "bf16", dk ** -0.5))
        v = dev(make_tensor(seed, 3, (B, N, H, dv), "bf16"))
        out = torch.empty((B, N, H, dv), dtype=torch.float32, device="cuda")
        fs = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
        R.ret_forward_chunkwise_noalloc(q, k, v, g, 128, out=out, final_state=fs, xpos=True, pos_offset=call)
        R.ret_check_device_error()
        nb = R.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, 128, torch.bfloat16, True)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        ref, fref = R.ret_forward_chunkwise_ws(q, k, v, g, 128, ws, out_dtype=torch.float32, xpos=True,
                                               pos_offset=call, want_final_state=True)
        R.ret_check_device_error()
        assert err_out(host64(out), host64(ref)) < TOL_BF16
        assert err_state(host64(fs), host64(fref)) < TOL_BF16


def test_noalloc_refuses_problems_above_its_array():
    import linear_recurrent_sequence_chunkwise_b200 as R
    B, N, H, dk, dv = 1, 16384, 16, 256, 64     # 256 MiB of scratch with xpos
    q = torch.zeros((B, N, H, dk), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((B, N, H, dv), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(R.RetentionError) as e:
        R.ret_forward_chunkwise_noalloc(q, q.clone(), v, gamma_schedule(H), 128, xpos=True)
    assert e.value.status == R.RET_ERR_INVALID_ARG
