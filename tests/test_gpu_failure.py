"""The timeout path of the device waits, exercised without a hang or a fault:
a wait that nothing completes gives up after its bound, the host reads
RET_ERR_TIMEOUT, and the context stays usable for the next call."""
import numpy as np
import pytest
import torch

import oracle
from retention_inputs import gamma_schedule, make_tensor
from tests.helpers import TOL_BF16, dev, err_out, host64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_the_context_survives():
    import linear_recurrent_sequence_chunkwise_b200 as R
    R.ret_check_device_error()                      # nothing pending
    R.ret_selftest_bounded_wait(1 << 12)
    with pytest.raises(R.RetentionError) as e:
        R.ret_check_device_error()
    assert e.value.status == R.RET_ERR_TIMEOUT
    R.ret_check_device_error()                      # the word was cleared
    # a normal forward afterwards still runs and is right
    B, N, H, dk, dv = 1, 300, 2, 256, 128
    q = make_tensor(401, 1, (B, N, H, dk), "bf16", dk ** -0.5)
    k = make_tensor(401, 2, (B, N, H, dk), "bf16", dk ** -0.5)
    v = make_tensor(401, 3, (B, N, H, dv), "bf16")
    g = gamma_schedule(H)
    nb = R.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, 128, torch.bfloat16, True)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    out = R.ret_forward_chunkwise_ws(dev(q), dev(k), dev(v), g, 128, ws, out_dtype=torch.float32, xpos=True)
    R.ret_check_device_error()
    ref, _ = oracle.retention_recurrent(oracle.xpos_rotate(q.f64), oracle.xpos_rotate(k.f64), v.f64, g)
    assert err_out(host64(out), ref) < TOL_BF16


def test_selftest_rejects_bad_polls():
    import linear_recurrent_sequence_chunkwise_b200 as R
    for polls in (0, (1 << 24) + 1):
        with pytest.raises(R.RetentionError):
            R.ret_selftest_bounded_wait(polls)
