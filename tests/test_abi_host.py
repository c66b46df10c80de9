"""Host-side checks of the C ABI: the library loads, exports every entry point
that include/*.h declares, and rejects bad arguments before launching
anything.  No GPU work happens here."""
import ctypes
import glob
import os
import re

import pytest
import torch

import linear_recurrent_sequence_chunkwise_b200 as R

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s+(ret_[a-z_0-9]+)\s*\(", text, flags=re.M))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for must in ("ret_xpos_rotate", "ret_forward_chunkwise", "ret_decode_step", "ret_forward_parallel",
                 "ret_forward_recurrent", "ret_check_device_error", "ret_last_error_string"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(R.LIB_PATH)
    missing = [n for n in declared_entry_points() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_exports_nothing_undeclared():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", R.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and l.split()[-1].startswith("ret_")}
    assert exported == set(declared_entry_points())


# Fake, never-dereferenced device addresses.  Every call below fails argument
# validation before any launch; the cases are skipped on a machine with a GPU
# so that a validation bug can never turn into a launch on a bogus address.
needs_no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers: host-only checks")
P = ctypes.c_void_p(0x10000)
P2 = ctypes.c_void_p(0x20000)
P3 = ctypes.c_void_p(0x30000)
P4 = ctypes.c_void_p(0x90000000)
G2 = (ctypes.c_double * 2)(0.9, 0.99)
S0 = ctypes.c_void_p(0)


def chunk_call(q=P, k=P2, v=P3, g=G2, B=1, N=8, H=2, dk=16, dv=16, chunk=4, out=P4, fs=None, in_dt=1, out_dt=1,
               xpos=0, theta=10000.0):
    return R.lib.ret_forward_chunkwise(q, k, v, g, B, N, H, dk, dv, chunk, out, fs, S0, in_dt, out_dt, xpos, 0,
                                       theta)


@needs_no_gpu
@pytest.mark.parametrize("kw", [
    dict(q=None), dict(k=None), dict(v=None), dict(out=None), dict(g=None),
    dict(B=0), dict(N=0), dict(H=0), dict(dk=0), dict(dv=-1), dict(chunk=0),
    dict(in_dt=7), dict(out_dt=-1),
    dict(g=(ctypes.c_double * 2)(0.9, 1.5)), dict(g=(ctypes.c_double * 2)(-0.1, 0.5)),
    dict(g=(ctypes.c_double * 2)(float("nan"), 0.5)),
    dict(xpos=1, dk=15), dict(xpos=1, theta=0.0), dict(xpos=1, theta=float("inf")),
    dict(q=ctypes.c_void_p(0x10004)), dict(out=ctypes.c_void_p(0x90000002)),
    dict(out=ctypes.c_void_p(0x10000)),            # out aliases q
    dict(fs=ctypes.c_void_p(0x90000008)),          # misaligned state
    dict(H=200, g=(ctypes.c_double * 200)(*([0.9] * 200))),
])
def test_chunkwise_rejects_bad_arguments(kw):
    st = chunk_call(**kw)
    assert st == R.RET_ERR_INVALID_ARG, (kw, st, R.ret_last_error_string())
    assert R.ret_last_error_string()


@needs_no_gpu
@pytest.mark.parametrize("fn", ["ret_forward_parallel", "ret_forward_recurrent"])
def test_cross_check_paths_reject_bad_arguments(fn):
    f = getattr(R.lib, fn)
    if fn == "ret_forward_parallel":
        st = f(P, P2, P3, G2, 1, 8, 2, 16, 16, None, S0, 1, 1, 0, 0, 1e4)
    else:
        st = f(P, P2, P3, G2, 1, 8, 2, 16, 16, None, None, S0, 1, 1, 0, 0, 1e4)
    assert st == R.RET_ERR_INVALID_ARG


@needs_no_gpu
@pytest.mark.parametrize("args", [
    (None, P2, P3, G2, P4, P, 1, 2, 16, 16),
    (P, P2, P3, G2, ctypes.c_void_p(0x90000004), P, 1, 2, 16, 16),   # misaligned state
    (P, P2, P3, G2, P4, P, 1, 2, 16, 18),                            # dv % 4
    (P, P2, P3, (ctypes.c_double * 2)(0.9, 2.0), P4, P, 1, 2, 16, 16),
    (P, P2, P3, G2, P4, P4, 1, 2, 16, 16),                           # out aliases state
    (P, P2, P3, G2, P4, P, 0, 2, 16, 16),
])
def test_decode_rejects_bad_arguments(args):
    q, k, v, g, state, out, B, H, dk, dv = args
    st = R.lib.ret_decode_step(q, k, v, g, state, out, S0, B, H, dk, dv, 1, 0)
    assert st == R.RET_ERR_INVALID_ARG, R.ret_last_error_string()


@needs_no_gpu
def test_rotate_rejects_bad_arguments():
    assert R.lib.ret_xpos_rotate(None, 1, 1, 4, 2, 8, 0, 1e4, S0) == R.RET_ERR_INVALID_ARG
    assert R.lib.ret_xpos_rotate(P, 1, 1, 4, 2, 7, 0, 1e4, S0) == R.RET_ERR_INVALID_ARG
    assert R.lib.ret_xpos_rotate(P, 1, 1, 4, 2, 8, 0, -1.0, S0) == R.RET_ERR_INVALID_ARG
    assert R.lib.ret_xpos_rotate(P, 9, 1, 4, 2, 8, 0, 1e4, S0) == R.RET_ERR_INVALID_ARG


def test_binding_requires_cuda_tensors():
    q = torch.zeros(1, 4, 1, 8)
    with pytest.raises(ValueError):
        R.ret_forward_chunkwise(q, q, q, [0.9], chunk=4, out=torch.zeros(1, 4, 1, 8))


# The two-pass workspace entry points.  Shape on the workspace path: bf16,
# chunk 128, dk 128, dv 64 (q, k 64 KB each at the fake addresses above).
WS = ctypes.c_void_p(0xA0000000)
QK_BYTES = 1 * 128 * 2 * 128 * 2          # one bf16 [B, N, H, dk] tensor
P_BYTES = 1 * 2 * 1 * 128 * 128 * 2       # the masked scores of every (b, h, chunk), bf16
WS_BYTES = QK_BYTES + P_BYTES             # k' alone (no rotation), then the scores


def prepare_call(q=P, k=P2, g=G2, dk=128, dv=64, ws=WS, nbytes=WS_BYTES, xpos=0):
    return R.lib.ret_chunkwise_prepare(q, k, g, 1, 128, 2, dk, dv, 128, S0, 1, xpos, 0, 1e4, ws, nbytes)


def prepared_call(ws=WS, nbytes=WS_BYTES, init=None, fs=None, dk=128, out=P4):
    return R.lib.ret_forward_chunkwise_prepared(P, P2, P3, G2, 1, 128, 2, dk, 64, 128, out, fs, init, S0, 1, 1, 0, 0,
                                                1e4, ws, nbytes)


def _scores_bytes(B, N, H, dk, copied):
    """Workspace of the scores form: k' (and the copied queries) [B, N, H, dk]
    bf16, 256-byte aligned, then P [B, H, ceil(N / 128), 128, 128] bf16."""
    qk = B * N * H * dk * 2 * (2 if copied else 1)
    return (qk + 255) // 256 * 256 + B * H * ((N + 127) // 128) * 128 * 128 * 2


def test_workspace_size_matches_the_two_pass_shape():
    ws = R.ret_chunkwise_prepare_workspace_bytes
    assert ws(1, 128, 2, 128, 64, 128, torch.bfloat16, False) == WS_BYTES
    assert ws(1, 128, 2, 128, 64, 128, torch.bfloat16, True) == 2 * QK_BYTES + P_BYTES
    assert ws(3, 1000, 2, 128, 64, 128, torch.bfloat16, True) == _scores_bytes(3, 1000, 2, 128, True)
    assert ws(1, 128, 2, 16, 64, 128, torch.bfloat16, False) == 0


@pytest.mark.parametrize("B,N,H,dk,dv,xpos", [
    (1, 128, 2, 128, 64, False), (1, 8192, 16, 256, 512, True), (64, 1024, 16, 256, 512, False),
    (4, 2048, 8, 64, 64, True), (2, 300, 3, 128, 192, True),
])
def test_single_call_workspace_is_the_scores_form(B, N, H, dk, dv, xpos):
    dkk, chunk = (128, 64) if dk == 64 else (dk, 128)
    want = _scores_bytes(B, N, H, dkk, xpos or dk == 64)
    assert R.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, chunk, torch.bfloat16, xpos) == want
    assert R.ret_chunkwise_prepare_workspace_bytes(B, N, H, dk, dv, chunk, torch.bfloat16, xpos) == want


@needs_no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(ws=None), 1), (dict(nbytes=100), 1), (dict(nbytes=2 * QK_BYTES + P_BYTES - 1, xpos=1), 1),
    (dict(ws=ctypes.c_void_p(0xA0000010)), 1), (dict(ws=ctypes.c_void_p(0x10000)), 1),
    (dict(g=(ctypes.c_double * 2)(0.9, 1.5)), 1), (dict(dk=16), 2), (dict(dv=48), 2),
])
def test_prepare_rejects_bad_arguments(kw, status):
    assert prepare_call(**kw) == status, (kw, R.ret_last_error_string())
    assert R.ret_last_error_string()


@needs_no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(ws=None), 1), (dict(nbytes=1000), 1), (dict(ws=ctypes.c_void_p(0x90000000)), 1),
    (dict(init=ctypes.c_void_p(0xB0000004)), 1),                 # misaligned initial state
    (dict(init=ctypes.c_void_p(0x90000000)), 1),                 # initial state overlaps out
    (dict(init=ctypes.c_void_p(0xB0000000), fs=ctypes.c_void_p(0xB0000100)), 1),  # partial overlap
    (dict(out=None), 1), (dict(dk=16), 2),
])
def test_prepared_rejects_bad_arguments(kw, status):
    assert prepared_call(**kw) == status, (kw, R.ret_last_error_string())
    assert R.ret_last_error_string()


def backward_call(q=P, k=P2, v=P3, do=ctypes.c_void_p(0x40000), dq=ctypes.c_void_p(0xC0000000),
                  dk_=ctypes.c_void_p(0xD0000000), dv_=ctypes.c_void_p(0xE0000000), dk=128, dv=128, in_dt=1,
                  ws=WS, nbytes=None):
    if nbytes is None:   # exactly the workspace this shape needs: [WS, WS + nbytes) overlaps nothing above
        nbytes = R.ret_backward_workspace_bytes(1, 64, 2, 128, 128, 128, torch.bfloat16, False)
        assert 0 < nbytes < 0x20000000
    return R.lib.ret_backward_chunkwise(q, k, v, do, G2, 1, 64, 2, dk, dv, 128, dq, dk_, dv_, S0, in_dt, 0, 0, 1e4,
                                        ws, nbytes)


def test_backward_workspace_size():
    assert R.ret_backward_workspace_bytes(1, 64, 2, 128, 128, 128, torch.bfloat16, False) > 0
    assert R.ret_backward_workspace_bytes(1, 64, 2, 128, 192, 128, torch.bfloat16, False) == 0   # dv % 128
    assert R.ret_backward_workspace_bytes(1, 64, 2, 64, 128, 128, torch.bfloat16, False) == 0    # dk
    assert R.ret_backward_workspace_bytes(1, 64, 2, 128, 128, 64, torch.bfloat16, False) == 0    # chunk
    assert R.ret_backward_workspace_bytes(1, 64, 2, 128, 128, 128, torch.float32, False) == 0    # fp32 inputs


@needs_no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(dq=None), 1), (dict(ws=None), 1), (dict(nbytes=1000), 1),
    (dict(dq=ctypes.c_void_p(0xC0000004)), 1),                    # misaligned gradient
    (dict(dk_=ctypes.c_void_p(0xC0000000)), 1),                   # dk overlaps dq
    (dict(dq=ctypes.c_void_p(0x10000)), 1),                       # dq overlaps q
    (dict(ws=ctypes.c_void_p(0xC0000000)), 1),                    # workspace overlaps dq
    (dict(dk=64), 2), (dict(dv=192), 2), (dict(in_dt=0), 2),
])
def test_backward_rejects_bad_arguments(kw, status):
    assert backward_call(**kw) == status, (kw, R.ret_last_error_string())
    assert R.ret_last_error_string()


def test_normalized_workspace_size():
    nb = R.ret_normalized_workspace_bytes(1, 200, 2, 128, 64, 128, torch.bfloat16, True)
    ws = 2 * 200 * 2 * 128 * 2
    # the scores form's q_rot, k' and P tiles [B, H, 2 chunks, 128, 128], then row
    # factors [B, N, H], key sums per 32 rows and per chunk start
    al = lambda x: (x + 255) // 256 * 256
    assert nb == al(ws) + 2 * 2 * 128 * 128 * 2 + al(200 * 2 * 4) + al(2 * 7 * 128 * 4) + al(2 * 2 * 128 * 4)
    assert R.ret_normalized_workspace_bytes(1, 200, 2, 16, 64, 128, torch.bfloat16, True) == 0
    assert R.ret_normalized_workspace_bytes(1, 200, 2, 128, 64, 128, torch.float32, True) == 0


def normalized_call(flags=3, out=P4, init=None, fs=None, z0=None, z1=None, ws=WS, nbytes=None, dk=128, pos=0):
    if nbytes is None:
        nbytes = R.ret_normalized_workspace_bytes(1, 128, 2, 128, 64, 128, torch.bfloat16, False)
        assert 0 < nbytes < 0x20000000
    return R.lib.ret_forward_chunkwise_normalized(P, P2, P3, G2, 1, 128, 2, dk, 64, 128, flags, out, init, fs, z0, z1,
                                                  S0, 1, 1, 0, pos, 1e4, ws, nbytes)


@needs_no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(flags=4), 1), (dict(flags=-1), 1), (dict(pos=-1), 1), (dict(out=None), 1),
    (dict(ws=None), 1), (dict(nbytes=1000), 1),
    (dict(z0=ctypes.c_void_p(0xB0000004)), 1),                              # misaligned z
    (dict(z1=ctypes.c_void_p(0x90000000)), 1),                              # z overlaps out
    (dict(z0=ctypes.c_void_p(0xB0000000), z1=ctypes.c_void_p(0xB0000100)), 1),  # partial overlap
    (dict(ws=ctypes.c_void_p(0x90000000)), 1),                              # workspace overlaps out
    (dict(dk=16), 2),
])
def test_normalized_rejects_bad_arguments(kw, status):
    assert normalized_call(**kw) == status, (kw, R.ret_last_error_string())
    assert R.ret_last_error_string()


def decode_normalized_call(z=ctypes.c_void_p(0xB0000000), pos=5, flags=3, state=ctypes.c_void_p(0xC0000000), dv=64):
    return R.lib.ret_decode_step_normalized(P, P2, P3, G2, state, z, P4, pos, flags, S0, 1, 2, 16, dv, 1, 1)


@needs_no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(z=None), 1), (dict(pos=-1), 1), (dict(flags=8), 1), (dict(state=None), 1),
    (dict(z=ctypes.c_void_p(0xB0000008)), 1),                    # misaligned z
    (dict(z=ctypes.c_void_p(0xC0000000)), 1),                    # z overlaps the state
    (dict(dv=6), 1),
])
def test_decode_normalized_rejects_bad_arguments(kw, status):
    assert decode_normalized_call(**kw) == status, (kw, R.ret_last_error_string())
    assert R.ret_last_error_string()


def decode_positions_call(pos=ctypes.c_void_p(0xD0000000), z=ctypes.c_void_p(0xB0000000), xpos=1, flags=3, dk=16,
                          theta=1e4):
    return R.lib.ret_decode_step_positions(P, P2, P3, G2, ctypes.c_void_p(0xC0000000), z, P4, pos, xpos, theta, flags,
                                           S0, 1, 2, dk, 64, 1, 1)


@needs_no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(pos=None), 1), (dict(pos=ctypes.c_void_p(0xD0000004)), 1), (dict(z=None), 1), (dict(dk=15), 1),
    (dict(theta=0.0), 1), (dict(flags=4), 1), (dict(pos=ctypes.c_void_p(0xC0000000)), 1),   # positions in the state
])
def test_decode_positions_rejects_bad_arguments(kw, status):
    assert decode_positions_call(**kw) == status, (kw, R.ret_last_error_string())
    assert R.ret_last_error_string()


# The binding checks every caller-provided buffer (shape, dtype, device)
# before it marshals a pointer: the C ABI cannot see how large a buffer is.
# These run on host tensors, so the checks fire before the CUDA-tensor one.
def _seq(B=1, N=8, H=2, dk=16, dv=8, dt=torch.bfloat16):
    return (torch.zeros(B, N, H, dk, dtype=dt), torch.zeros(B, N, H, dk, dtype=dt), torch.zeros(B, N, H, dv, dtype=dt))


@pytest.mark.parametrize("kw,exc,msg", [
    (dict(out=torch.zeros(1, 8, 2, 4, dtype=torch.bfloat16)), ValueError, "out must have shape"),
    (dict(out=torch.zeros(1, 8, 2, 8, dtype=torch.float16)), TypeError, "out must be"),
    (dict(final_state=torch.zeros(1, 2, 16, 4)), ValueError, "final_state must have shape"),
    (dict(final_state=torch.zeros(1, 2, 16, 8, dtype=torch.bfloat16)), TypeError, "final_state must be"),
])
def test_binding_checks_output_buffers(kw, exc, msg):
    q, k, v = _seq()
    for fn in (lambda: R.ret_forward_chunkwise(q, k, v, [0.9, 0.8], 4, **kw),
               lambda: R.ret_forward_chunkwise_ws(q, k, v, [0.9, 0.8], 4, torch.zeros(16, dtype=torch.uint8), **kw),
               lambda: R.ret_forward_chunkwise_noalloc(q, k, v, [0.9, 0.8], 4, **kw),
               lambda: R.ret_forward_recurrent(q, k, v, [0.9, 0.8], **kw)):
        with pytest.raises(exc, match=msg):
            fn()


def test_binding_checks_initial_state_and_gradients():
    q, k, v = _seq()
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="initial_state must have shape"):
        R.ret_forward_chunkwise_prepared(q, k, v, [0.9, 0.8], 128, ws, initial_state=torch.zeros(1, 2, 8, 16))
    with pytest.raises(ValueError, match="dout must have shape"):
        R.ret_backward_chunkwise(q, k, v, torch.zeros(1, 8, 2, 16, dtype=torch.bfloat16), [0.9, 0.8], 128)
    with pytest.raises(TypeError, match="dout must be"):
        R.ret_backward_chunkwise(q, k, v, torch.zeros(1, 8, 2, 8), [0.9, 0.8], 128)
    with pytest.raises(ValueError, match="dq must have shape"):
        R.ret_backward_chunkwise(q, k, v, torch.zeros(1, 8, 2, 8, dtype=torch.bfloat16), [0.9, 0.8], 128,
                                 workspace=ws, dq=torch.zeros(1, 8, 2, 8))
    with pytest.raises(ValueError, match="final_z must have shape"):
        R.ret_forward_chunkwise_normalized(q, k, v, [0.9, 0.8], 128, workspace=ws, final_z=torch.zeros(1, 2, 8))


def test_binding_checks_decode_buffers():
    q, k, v = torch.zeros(3, 2, 16), torch.zeros(3, 2, 16), torch.zeros(3, 2, 8)
    S = torch.zeros(3, 2, 16, 8)
    with pytest.raises(ValueError, match="state must have shape"):
        R.ret_decode_step(q, k, v, [0.9, 0.8], torch.zeros(3, 2, 8, 16))
    with pytest.raises(TypeError, match="state must be"):
        R.ret_decode_step(q, k, v, [0.9, 0.8], S.double())
    with pytest.raises(ValueError, match="out must have shape"):
        R.ret_decode_step(q, k, v, [0.9, 0.8], S, out=torch.zeros(3, 2, 16))
    with pytest.raises(ValueError, match="z must have shape"):
        R.ret_decode_step_normalized(q, k, v, [0.9, 0.8], S, torch.zeros(3, 16), 5)
    with pytest.raises(TypeError, match="positions must be"):
        R.ret_decode_step_positions(q, k, v, [0.9, 0.8], S, torch.zeros(3, dtype=torch.int32))
    with pytest.raises(ValueError, match="positions must have shape"):
        R.ret_decode_step_positions(q, k, v, [0.9, 0.8], S, torch.zeros(2, dtype=torch.int64))
    with pytest.raises(TypeError, match="share a dtype"):
        R.ret_decode_step(q, k.bfloat16(), v, [0.9, 0.8], S)


def test_binding_checks_layer_weights():
    B, N, dm, H, dk, dv = 1, 8, 32, 2, 16, 8
    x = torch.zeros(B, N, dm, dtype=torch.bfloat16)
    w = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    good = dict(wq=w(dm, H * dk), wk=w(dm, H * dk), wv=w(dm, H * dv), wg=w(dm, H * dv), wo=w(H * dv, dm))
    for name, bad in (("wk", w(dm, H * dk + 2)), ("wg", w(dm, H * dk)), ("wo", w(dm, H * dv))):
        ws = dict(good, **{name: bad})
        with pytest.raises(ValueError, match=f"{name} must have shape"):
            R.ret_msr_forward(x, ws["wq"], ws["wk"], ws["wv"], ws["wg"], ws["wo"], [0.9, 0.8], H)
    with pytest.raises(ValueError, match="w2 must have shape"):
        R.ret_retnet_block_forward(x, *good.values(), w(dm, 64), w(64, dm + 8), [0.9, 0.8], H)
    with pytest.raises(ValueError, match="ln1_gain must have shape"):
        R.ret_retnet_block_forward(x, *good.values(), w(dm, 64), w(64, dm), [0.9, 0.8], H, ln1_gain=w(dm + 1))
    with pytest.raises(ValueError, match="x must be bfloat16"):
        R.ret_msr_forward(x.float(), *good.values(), [0.9, 0.8], H)


@needs_no_gpu
@pytest.mark.parametrize("B,N,H,dk,xpos,refused", [
    (4, 4097, 8, 64, 0, True),     # d_k 64 padded to 128 with the queries copied: 4*4097*8*128*4 > 64 MiB
    (4, 4097, 8, 64, 1, True),
    (1, 8193, 16, 256, 0, True),   # keys only: 8193*16*256*2 > 64 MiB
])
def test_noalloc_refuses_above_its_array_on_the_host(B, N, H, dk, xpos, refused):
    g = (ctypes.c_double * H)(*([0.99] * H))
    st = R.lib.ret_forward_chunkwise_noalloc(P, P2, P3, g, B, N, H, dk, 64, 128 if dk > 64 else 64, P4, None, S0,
                                             1, 1, xpos, 0, 10000.0)
    assert st == R.RET_ERR_INVALID_ARG
    msg = R.ret_last_error_string()
    assert "scratch" in msg and f"d_k = {dk}" in msg
