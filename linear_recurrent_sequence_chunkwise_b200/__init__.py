"""Multi-scale retention on B200: Python binding of the C ABI in
``include/retention.h``.

The functions below carry the C entry points' names and do argument
marshalling only (torch tensors -> device pointers, sizes, dtypes, the
current CUDA stream); every step of the computation runs in the CUDA library
``libretention.so`` built from ``csrc/``.  There is no fallback: importing
this package fails if the library is missing, and every call raises
``RetentionError`` when the library returns an error status.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "RetentionError", "lib", "ret_xpos_rotate", "ret_forward_chunkwise", "ret_forward_chunkwise_ws",
    "ret_chunkwise_workspace_bytes", "ret_chunkwise_prepare_workspace_bytes", "ret_chunkwise_prepare",
    "ret_forward_chunkwise_prepared",
    "ret_backward_chunkwise", "ret_backward_workspace_bytes",
    "ret_forward_chunkwise_noalloc", "ret_chunkwise_noalloc_max_bytes",
    "ret_decode_step", "ret_msr_forward", "ret_msr_workspace_bytes",
    "ret_forward_chunkwise_normalized", "ret_normalized_workspace_bytes", "ret_decode_step_normalized",
    "ret_decode_step_positions", "ret_selftest_bounded_wait",
    "NORM_DECAY", "NORM_SCORE",
    "ret_linear_bf16", "ret_retnet_block_forward", "ret_retnet_block_workspace_bytes",
    "ret_forward_parallel", "ret_forward_recurrent", "ret_check_device_error", "ret_last_error_string",
    "RET_OK", "RET_ERR_INVALID_ARG", "RET_ERR_UNSUPPORTED", "RET_ERR_CUDA", "RET_ERR_TIMEOUT",
    "RET_F32", "RET_BF16",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libretention.so")

RET_OK, RET_ERR_INVALID_ARG, RET_ERR_UNSUPPORTED, RET_ERR_CUDA, RET_ERR_TIMEOUT = 0, 1, 2, 3, 4
RET_F32, RET_BF16 = 0, 1
_STATUS = {0: "RET_OK", 1: "RET_ERR_INVALID_ARG", 2: "RET_ERR_UNSUPPORTED", 3: "RET_ERR_CUDA",
           4: "RET_ERR_TIMEOUT"}


class RetentionError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


def _load_library():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python linear_recurrent_sequence_chunkwise_b200/build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, d, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_int64
    dp = ctypes.POINTER(ctypes.c_double)
    L.ret_xpos_rotate.argtypes = [vp, i, i, i, i, i, i64, d, vp]
    L.ret_forward_chunkwise.argtypes = [vp, vp, vp, dp, i, i, i, i, i, i, vp, vp, vp, i, i, i, i64, d]
    L.ret_forward_chunkwise_ws.argtypes = [vp, vp, vp, dp, i, i, i, i, i, i, vp, vp, vp, i, i, i, i64, d, vp,
                                           ctypes.c_size_t]
    L.ret_forward_chunkwise_noalloc.argtypes = [vp, vp, vp, dp, i, i, i, i, i, i, vp, vp, vp, i, i, i, i64, d]
    L.ret_backward_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    L.ret_backward_workspace_bytes.restype = ctypes.c_size_t
    L.ret_backward_chunkwise.argtypes = [vp, vp, vp, vp, dp, i, i, i, i, i, i, vp, vp, vp, vp, i, i, i64, d, vp,
                                         ctypes.c_size_t]
    L.ret_chunkwise_prepare.argtypes = [vp, vp, dp, i, i, i, i, i, i, vp, i, i, i64, d, vp, ctypes.c_size_t]
    L.ret_forward_chunkwise_prepared.argtypes = [vp, vp, vp, dp, i, i, i, i, i, i, vp, vp, vp, vp, i, i, i, i64, d,
                                                 vp, ctypes.c_size_t]
    L.ret_chunkwise_noalloc_max_bytes.argtypes = []
    L.ret_chunkwise_noalloc_max_bytes.restype = ctypes.c_size_t
    L.ret_chunkwise_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    L.ret_chunkwise_workspace_bytes.restype = ctypes.c_size_t
    L.ret_chunkwise_prepare_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    L.ret_chunkwise_prepare_workspace_bytes.restype = ctypes.c_size_t
    L.ret_decode_step.argtypes = [vp, vp, vp, dp, vp, vp, vp, i, i, i, i, i, i]
    L.ret_normalized_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    L.ret_normalized_workspace_bytes.restype = ctypes.c_size_t
    L.ret_forward_chunkwise_normalized.argtypes = [vp, vp, vp, dp, i, i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, i,
                                                   i, i, i64, d, vp, ctypes.c_size_t]
    L.ret_decode_step_normalized.argtypes = [vp, vp, vp, dp, vp, vp, vp, i64, i, vp, i, i, i, i, i, i]
    L.ret_selftest_bounded_wait.argtypes = [ctypes.c_uint32, vp]
    L.ret_decode_step_positions.argtypes = [vp, vp, vp, dp, vp, vp, vp, vp, i, d, i, vp, i, i, i, i, i, i]
    L.ret_forward_parallel.argtypes = [vp, vp, vp, dp, i, i, i, i, i, vp, vp, i, i, i, i64, d]
    L.ret_forward_recurrent.argtypes = [vp, vp, vp, dp, i, i, i, i, i, vp, vp, vp, i, i, i, i64, d]
    L.ret_msr_workspace_bytes.argtypes = [i, i, i, i, i, i]
    L.ret_msr_workspace_bytes.restype = ctypes.c_size_t
    L.ret_msr_forward.argtypes = [vp, vp, vp, vp, vp, vp, dp, i, i, i, i, i, i, i, d, d, i, i64, d, vp, i, vp,
                                  ctypes.c_size_t, vp]
    L.ret_linear_bf16.argtypes = [vp, vp, vp, i, i, i, i, vp]
    L.ret_retnet_block_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    L.ret_retnet_block_workspace_bytes.restype = ctypes.c_size_t
    L.ret_retnet_block_forward.argtypes = [vp] * 12 + [dp, i, i, i, i, i, i, i, i, d, d, d, i, i64, d, vp, i, vp,
                                                       ctypes.c_size_t, vp]
    L.ret_check_device_error.argtypes = [vp]
    L.ret_last_error_string.restype = ctypes.c_char_p
    L.ret_last_error_string.argtypes = []
    for name in ("ret_xpos_rotate", "ret_forward_chunkwise", "ret_forward_chunkwise_ws",
                 "ret_forward_chunkwise_noalloc", "ret_chunkwise_prepare", "ret_forward_chunkwise_prepared",
                 "ret_backward_chunkwise", "ret_decode_step",
                 "ret_forward_parallel",
                 "ret_forward_recurrent", "ret_check_device_error", "ret_msr_forward", "ret_linear_bf16"):
        getattr(L, name).restype = ctypes.c_int
    return L


lib = _load_library()


def ret_last_error_string() -> str:
    return lib.ret_last_error_string().decode(errors="replace")


def _check(status: int):
    if status != RET_OK:
        raise RetentionError(status, ret_last_error_string())


def _dt(t: torch.dtype) -> int:
    if t == torch.float32:
        return RET_F32
    if t == torch.bfloat16:
        return RET_BF16
    raise TypeError(f"unsupported dtype {t}; expected float32 or bfloat16")


def _ptr(t: Optional[torch.Tensor], name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


F32 = (torch.float32,)
FLOATS = (torch.float32, torch.bfloat16)


def _buf(t: Optional[torch.Tensor], name: str, shape, dtypes, like: torch.Tensor):
    """A caller-provided buffer must have the shape and dtype the call reads or
    writes and sit on the inputs' device: the C ABI takes plain pointers and
    cannot check either."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {list(shape)} (got {list(t.shape)})")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must be {' or '.join(str(d) for d in dtypes)} (got {t.dtype})")
    if t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, the inputs on {like.device}")


def _same_device(like: torch.Tensor, **tensors):
    for name, t in tensors.items():
        if t is not None and t.device != like.device:
            raise ValueError(f"{name} is on {t.device}, the inputs on {like.device}")


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _gammas(gammas: Sequence[float], H: int):
    g = [float(x) for x in gammas]
    if len(g) != H:
        raise ValueError(f"gammas has {len(g)} entries, expected H={H}")
    return (ctypes.c_double * H)(*g)


def ret_xpos_rotate(x: torch.Tensor, pos_offset: int = 0, theta_base: float = 10000.0, stream=None) -> torch.Tensor:
    """Rotate x [B, N, H, d] in place (xPos / rotary, consecutive pairs)."""
    B, N, H, d = x.shape
    _check(lib.ret_xpos_rotate(_ptr(x, "x"), _dt(x.dtype), B, N, H, d, int(pos_offset), float(theta_base),
                               _stream(stream)))
    return x


def _seq_shapes(q, k, v):
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q, k [B, N, H, dk] and v [B, N, H, dv]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share a dtype")
    _same_device(q, k=k, v=v)
    B, N, H, dk = q.shape
    return B, N, H, dk, v.shape[3]


def _seq_outputs(q, out, final_state, B, N, H, dk, dv, initial_state=None):
    _buf(out, "out", (B, N, H, dv), FLOATS, q)
    _buf(final_state, "final_state", (B, H, dk, dv), F32, q)
    _buf(initial_state, "initial_state", (B, H, dk, dv), F32, q)


def ret_forward_chunkwise(q, k, v, gammas, chunk: int, out=None, final_state=None, out_dtype=None,
                          xpos: bool = False, pos_offset: int = 0, theta_base: float = 10000.0,
                          want_final_state: bool = False, stream=None):
    """Chunkwise retention forward.  Returns ``out`` [B, N, H, dv], or
    ``(out, final_state)`` when a final state is requested (passed in or
    ``want_final_state``)."""
    B, N, H, dk, dv = _seq_shapes(q, k, v)
    if out is None:
        out = torch.empty((B, N, H, dv), dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and want_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _seq_outputs(q, out, final_state, B, N, H, dk, dv)
    _check(lib.ret_forward_chunkwise(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H), B, N, H, dk,
                                     dv, int(chunk), _ptr(out, "out"), _ptr(final_state, "final_state"),
                                     _stream(stream), _dt(q.dtype), _dt(out.dtype), int(bool(xpos)),
                                     int(pos_offset), float(theta_base)))
    return (out, final_state) if final_state is not None else out


def ret_chunkwise_workspace_bytes(B, N, H, dk, dv, chunk, dtype=torch.bfloat16, xpos: bool = False) -> int:
    """Workspace bytes ret_forward_chunkwise_ws needs for this shape (0: the
    shape does not take the workspace path)."""
    return int(lib.ret_chunkwise_workspace_bytes(B, N, H, dk, dv, int(chunk), _dt(dtype), int(bool(xpos))))


def ret_forward_chunkwise_ws(q, k, v, gammas, chunk: int, workspace, out=None, final_state=None, out_dtype=None,
                             xpos: bool = False, pos_offset: int = 0, theta_base: float = 10000.0,
                             want_final_state: bool = False, stream=None):
    """Chunkwise forward with a caller-provided workspace (a CUDA uint8 tensor
    of at least ret_chunkwise_workspace_bytes bytes)."""
    B, N, H, dk, dv = _seq_shapes(q, k, v)
    if out is None:
        out = torch.empty((B, N, H, dv), dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and want_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _seq_outputs(q, out, final_state, B, N, H, dk, dv)
    _same_device(q, workspace=workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.ret_forward_chunkwise_ws(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H), B, N, H, dk,
                                        dv, int(chunk), _ptr(out, "out"), _ptr(final_state, "final_state"),
                                        _stream(stream), _dt(q.dtype), _dt(out.dtype), int(bool(xpos)),
                                        int(pos_offset), float(theta_base), _ptr(workspace, "workspace"), nbytes))
    return (out, final_state) if final_state is not None else out


def ret_chunkwise_prepare_workspace_bytes(B, N, H, dk, dv, chunk, dtype=torch.bfloat16, xpos: bool = False) -> int:
    """Workspace bytes of ret_chunkwise_prepare / ret_forward_chunkwise_prepared (0: shape not on that path)."""
    return int(lib.ret_chunkwise_prepare_workspace_bytes(B, N, H, dk, dv, chunk, _dt(dtype), int(bool(xpos))))


def ret_chunkwise_prepare(q, k, gammas, chunk: int, workspace, dv: int, xpos: bool = False, pos_offset: int = 0,
                          theta_base: float = 10000.0, stream=None):
    """First pass of the workspace path: rotated queries (xpos) and rotated,
    zeta-scaled keys into ``workspace``."""
    if q.shape != k.shape or q.dim() != 4:
        raise ValueError("q and k must both be [B, N, H, dk]")
    B, N, H, dk = q.shape
    _same_device(q, k=k, workspace=workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.ret_chunkwise_prepare(_ptr(q, "q"), _ptr(k, "k"), _gammas(gammas, H), B, N, H, dk, int(dv),
                                     int(chunk), _stream(stream), _dt(q.dtype), int(bool(xpos)), int(pos_offset),
                                     float(theta_base), _ptr(workspace, "workspace"), nbytes))


def ret_forward_chunkwise_prepared(q, k, v, gammas, chunk: int, workspace, out=None, final_state=None,
                                   initial_state=None, out_dtype=None, xpos: bool = False, pos_offset: int = 0,
                                   theta_base: float = 10000.0, want_final_state: bool = False, stream=None):
    """Second pass of the workspace path on a workspace filled by
    ret_chunkwise_prepare with the same arguments; ``initial_state`` (fp32
    [B, H, dk, dv], or None for zero) continues a sequence."""
    B, N, H, dk, dv = _seq_shapes(q, k, v)
    if out is None:
        out = torch.empty((B, N, H, dv), dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and want_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _seq_outputs(q, out, final_state, B, N, H, dk, dv, initial_state)
    _same_device(q, workspace=workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.ret_forward_chunkwise_prepared(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H), B, N,
                                              H, dk, dv, int(chunk), _ptr(out, "out"),
                                              _ptr(final_state, "final_state"),
                                              _ptr(initial_state, "initial_state"), _stream(stream), _dt(q.dtype),
                                              _dt(out.dtype), int(bool(xpos)), int(pos_offset), float(theta_base),
                                              _ptr(workspace, "workspace"), nbytes))
    return (out, final_state) if final_state is not None else out


def ret_backward_workspace_bytes(B, N, H, dk, dv, chunk, in_dtype=torch.bfloat16, xpos: bool = False) -> int:
    """Workspace bytes of ret_backward_chunkwise (0: shape not supported)."""
    return int(lib.ret_backward_workspace_bytes(B, N, H, dk, dv, int(chunk), _dt(in_dtype), int(bool(xpos))))


def ret_backward_chunkwise(q, k, v, dout, gammas, chunk: int, workspace=None, dq=None, dk=None, dv=None,
                           xpos: bool = False, pos_offset: int = 0, theta_base: float = 10000.0, stream=None):
    """Gradients (dq, dk, dv) in fp32 of sum(out * dout) for the chunkwise
    forward of the same arguments."""
    B, N, H, dk_, dv_ = _seq_shapes(q, k, v)
    _buf(dout, "dout", (B, N, H, dv_), (q.dtype,), q)
    dq = torch.empty((B, N, H, dk_), dtype=torch.float32, device=q.device) if dq is None else dq
    dk = torch.empty((B, N, H, dk_), dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.empty((B, N, H, dv_), dtype=torch.float32, device=q.device) if dv is None else dv
    if workspace is None:
        nb = ret_backward_workspace_bytes(B, N, H, dk_, dv_, chunk, q.dtype, xpos)
        workspace = torch.empty(max(nb, 1), dtype=torch.uint8, device=q.device)
    _buf(dq, "dq", (B, N, H, dk_), F32, q)
    _buf(dk, "dk", (B, N, H, dk_), F32, q)
    _buf(dv, "dv", (B, N, H, dv_), F32, q)
    _same_device(q, workspace=workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.ret_backward_chunkwise(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(dout, "dout"),
                                      _gammas(gammas, H), B, N, H, dk_, dv_, int(chunk), _ptr(dq, "dq"),
                                      _ptr(dk, "dk"), _ptr(dv, "dv"), _stream(stream), _dt(q.dtype),
                                      int(bool(xpos)), int(pos_offset), float(theta_base),
                                      _ptr(workspace, "workspace"), nbytes))
    return dq, dk, dv


def ret_chunkwise_noalloc_max_bytes() -> int:
    """Bytes of the library's fixed scratch array used by
    ret_forward_chunkwise_noalloc."""
    return int(lib.ret_chunkwise_noalloc_max_bytes())


def ret_forward_chunkwise_noalloc(q, k, v, gammas, chunk: int, out=None, final_state=None, out_dtype=None,
                                  xpos: bool = False, pos_offset: int = 0, theta_base: float = 10000.0,
                                  want_final_state: bool = False, stream=None):
    """Chunkwise forward whose scratch is a fixed device array inside the
    library: for callers that cannot allocate device memory at call time.
    Pass ``out`` / ``final_state`` to avoid the allocations this wrapper would
    otherwise make for them."""
    B, N, H, dk, dv = _seq_shapes(q, k, v)
    if out is None:
        out = torch.empty((B, N, H, dv), dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and want_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _seq_outputs(q, out, final_state, B, N, H, dk, dv)
    _check(lib.ret_forward_chunkwise_noalloc(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H), B, N,
                                             H, dk, dv, int(chunk), _ptr(out, "out"),
                                             _ptr(final_state, "final_state"), _stream(stream), _dt(q.dtype),
                                             _dt(out.dtype), int(bool(xpos)), int(pos_offset), float(theta_base)))
    return (out, final_state) if final_state is not None else out


def ret_forward_parallel(q, k, v, gammas, out=None, out_dtype=None, xpos: bool = False, pos_offset: int = 0,
                         theta_base: float = 10000.0, stream=None):
    """Parallel form (Q K^T (.) D) V, for cross-checks.  Returns ``out``."""
    B, N, H, dk, dv = _seq_shapes(q, k, v)
    if out is None:
        out = torch.empty((B, N, H, dv), dtype=out_dtype or q.dtype, device=q.device)
    _seq_outputs(q, out, None, B, N, H, dk, dv)
    _check(lib.ret_forward_parallel(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H), B, N, H, dk,
                                    dv, _ptr(out, "out"), _stream(stream), _dt(q.dtype), _dt(out.dtype),
                                    int(bool(xpos)), int(pos_offset), float(theta_base)))
    return out


def ret_forward_recurrent(q, k, v, gammas, out=None, final_state=None, out_dtype=None, xpos: bool = False,
                          pos_offset: int = 0, theta_base: float = 10000.0, want_final_state: bool = False,
                          stream=None):
    """Recurrent form token by token, for cross-checks."""
    B, N, H, dk, dv = _seq_shapes(q, k, v)
    if out is None:
        out = torch.empty((B, N, H, dv), dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and want_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _seq_outputs(q, out, final_state, B, N, H, dk, dv)
    _check(lib.ret_forward_recurrent(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H), B, N, H, dk,
                                     dv, _ptr(out, "out"), _ptr(final_state, "final_state"), _stream(stream),
                                     _dt(q.dtype), _dt(out.dtype), int(bool(xpos)), int(pos_offset),
                                     float(theta_base)))
    return (out, final_state) if final_state is not None else out


def _step_shapes(q, k, v, state):
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise ValueError("expected q, k [B, H, dk] and v [B, H, dv]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share a dtype")
    _same_device(q, k=k, v=v)
    B, H, dk = q.shape
    dv = v.shape[2]
    if state is None:
        raise ValueError("state must be float32 [B, H, dk, dv]")
    _buf(state, "state", (B, H, dk, dv), F32, q)
    return B, H, dk, dv


def ret_decode_step(q, k, v, gammas, state, out=None, out_dtype=None, stream=None):
    """One decode step: state [B, H, dk, dv] fp32 updated in place; returns
    out [B, H, dv]."""
    B, H, dk, dv = _step_shapes(q, k, v, state)
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype or torch.float32, device=q.device)
    _buf(out, "out", (B, H, dv), FLOATS, q)
    _check(lib.ret_decode_step(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H),
                               _ptr(state, "state"), _ptr(out, "out"), _stream(stream), B, H, dk, dv,
                               _dt(q.dtype), _dt(out.dtype)))
    return out


NORM_DECAY = 1  # RET_NORM_DECAY
NORM_SCORE = 2  # RET_NORM_SCORE


def ret_normalized_workspace_bytes(B, N, H, dk, dv, chunk, in_dtype=torch.bfloat16, xpos: bool = False) -> int:
    """Workspace bytes of ret_forward_chunkwise_normalized (0: shape not supported)."""
    return int(lib.ret_normalized_workspace_bytes(B, N, H, dk, dv, int(chunk), _dt(in_dtype), int(bool(xpos))))


def ret_forward_chunkwise_normalized(q, k, v, gammas, chunk: int, norm_flags: int = NORM_DECAY | NORM_SCORE,
                                     workspace=None, out=None, out_dtype=None, initial_state=None,
                                     final_state=None, initial_z=None, final_z=None, xpos: bool = False,
                                     pos_offset: int = 0, theta_base: float = 10000.0, stream=None):
    """Chunkwise forward with the score normalizations (norm_flags: NORM_DECAY,
    NORM_SCORE); states S [B, H, dk, dv] and z [B, H, dk] fp32, optional."""
    B, N, H, dk, dv = _seq_shapes(q, k, v)
    if out is None:
        out = torch.empty((B, N, H, dv), dtype=out_dtype or q.dtype, device=q.device)
    _seq_outputs(q, out, final_state, B, N, H, dk, dv, initial_state)
    _buf(initial_z, "initial_z", (B, H, dk), F32, q)
    _buf(final_z, "final_z", (B, H, dk), F32, q)
    if workspace is None:
        nb = ret_normalized_workspace_bytes(B, N, H, dk, dv, chunk, q.dtype, xpos)
        workspace = torch.empty(max(nb, 1), dtype=torch.uint8, device=q.device)
    _same_device(q, workspace=workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.ret_forward_chunkwise_normalized(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H), B, N,
                                                H, dk, dv, int(chunk), int(norm_flags), _ptr(out, "out"),
                                                _ptr(initial_state, "initial_state"), _ptr(final_state, "final_state"),
                                                _ptr(initial_z, "initial_z"), _ptr(final_z, "final_z"),
                                                _stream(stream), _dt(q.dtype), _dt(out.dtype), int(bool(xpos)),
                                                int(pos_offset), float(theta_base), _ptr(workspace, "workspace"),
                                                nbytes))
    return out


def ret_decode_step_normalized(q, k, v, gammas, state, z, position: int, norm_flags: int = NORM_DECAY | NORM_SCORE,
                               out=None, out_dtype=None, stream=None):
    """One decode step with the score normalizations at 0-based ``position``:
    state [B, H, dk, dv] and z [B, H, dk] (fp32) updated in place."""
    B, H, dk, dv = _step_shapes(q, k, v, state)
    _buf(z, "z", (B, H, dk), F32, q)
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype or torch.float32, device=q.device)
    _buf(out, "out", (B, H, dv), FLOATS, q)
    _check(lib.ret_decode_step_normalized(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H),
                                          _ptr(state, "state"), _ptr(z, "z"), _ptr(out, "out"), int(position),
                                          int(norm_flags), _stream(stream), B, H, dk, dv, _dt(q.dtype),
                                          _dt(out.dtype)))
    return out


def ret_decode_step_positions(q, k, v, gammas, state, positions, z=None, xpos: bool = True,
                              theta_base: float = 10000.0, norm_flags: int = 0, out=None, out_dtype=None,
                              stream=None):
    """One decode step with each sequence at its own position: positions int64
    [B] on the device; xPos rotation of q, k inside the step; optional score
    normalizations with z [B, H, dk] fp32 (in place)."""
    B, H, dk, dv = _step_shapes(q, k, v, state)
    _buf(positions, "positions", (B,), (torch.int64,), q)
    _buf(z, "z", (B, H, dk), F32, q)
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype or torch.float32, device=q.device)
    _buf(out, "out", (B, H, dv), FLOATS, q)
    _check(lib.ret_decode_step_positions(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _gammas(gammas, H),
                                         _ptr(state, "state"), _ptr(z, "z"), _ptr(out, "out"),
                                         _ptr(positions, "positions"), int(bool(xpos)), float(theta_base),
                                         int(norm_flags), _stream(stream), B, H, dk, dv, _dt(q.dtype),
                                         _dt(out.dtype)))
    return out


def ret_selftest_bounded_wait(polls: int = 1 << 12, stream=None):
    """Run the bounded-wait self-test: the next ret_check_device_error raises
    with RET_ERR_TIMEOUT."""
    _check(lib.ret_selftest_bounded_wait(int(polls), _stream(stream)))


def ret_check_device_error(stream=None):
    """Synchronise the stream and raise if a kernel gave up a bounded wait."""
    _check(lib.ret_check_device_error(_stream(stream)))


BF16 = (torch.bfloat16,)


def _msr_shapes(x, wq, wk, wv, wg, wo, H: int):
    """B, N, d_model, dk, dv of an MSR layer from x [B, N, d_model] and the
    (input, output) weights W_Q, W_K [d_model, H dk], W_V, W_G [d_model, H dv],
    W_O [H dv, d_model], all bf16 on x's device."""
    if x.dim() != 3 or x.dtype != torch.bfloat16:
        raise ValueError("x must be bfloat16 [B, N, d_model]")
    B, N, dm = x.shape
    if H < 1 or wq.dim() != 2 or wv.dim() != 2 or wq.shape[1] % H or wv.shape[1] % H:
        raise ValueError("W_Q and W_V must be [d_model, H * d] with H dividing their widths")
    dk, dv = wq.shape[1] // H, wv.shape[1] // H
    _buf(wq, "wq", (dm, H * dk), BF16, x)
    _buf(wk, "wk", (dm, H * dk), BF16, x)
    _buf(wv, "wv", (dm, H * dv), BF16, x)
    _buf(wg, "wg", (dm, H * dv), BF16, x)
    _buf(wo, "wo", (H * dv, dm), BF16, x)
    return B, N, dm, dk, dv


def ret_retnet_block_workspace_bytes(B, N, dmodel, H, dk, dv, dff) -> int:
    return int(lib.ret_retnet_block_workspace_bytes(B, N, dmodel, H, dk, dv, dff))


def ret_retnet_block_forward(x, wq, wk, wv, wg, wo, w1, w2, gammas, H: int, ln1_gain=None, ln1_bias=None,
                             ln2_gain=None, ln2_bias=None, chunk: int = 128, k_scale: float = 1.0,
                             gn_eps: float = 1e-5, ln_eps: float = 1e-5, xpos: bool = True, pos_offset: int = 0,
                             theta_base: float = 10000.0, out=None, out_dtype=torch.bfloat16, workspace=None,
                             stream=None):
    """One pre-LayerNorm RetNet block: Y = MSR(LN1(x)) + x, out = gelu(LN2(Y) W1) W2 + Y.
    x [B, N, d_model] bf16; weights bf16 [in, out]; LayerNorm gains/biases bf16
    [d_model] or None (1 / 0)."""
    B, N, dm, dk, dv = _msr_shapes(x, wq, wk, wv, wg, wo, H)
    dff = w1.shape[1]
    _buf(w1, "w1", (dm, dff), BF16, x)
    _buf(w2, "w2", (dff, dm), BF16, x)
    for name, t in (("ln1_gain", ln1_gain), ("ln1_bias", ln1_bias), ("ln2_gain", ln2_gain), ("ln2_bias", ln2_bias)):
        _buf(t, name, (dm,), BF16, x)
    if out is None:
        out = torch.empty((B, N, dm), dtype=out_dtype, device=x.device)
    _buf(out, "out", (B, N, dm), FLOATS, x)
    if workspace is None:
        workspace = torch.empty(ret_retnet_block_workspace_bytes(B, N, dm, H, dk, dv, dff), dtype=torch.uint8,
                                device=x.device)
    _same_device(x, workspace=workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.ret_retnet_block_forward(_ptr(x, "x"), _ptr(ln1_gain, "ln1_gain"), _ptr(ln1_bias, "ln1_bias"),
                                        _ptr(wq, "wq"), _ptr(wk, "wk"), _ptr(wv, "wv"), _ptr(wg, "wg"),
                                        _ptr(wo, "wo"), _ptr(ln2_gain, "ln2_gain"), _ptr(ln2_bias, "ln2_bias"),
                                        _ptr(w1, "w1"), _ptr(w2, "w2"), _gammas(gammas, H), B, N, dm, H, dk, dv,
                                        dff, int(chunk), float(k_scale), float(gn_eps), float(ln_eps),
                                        int(bool(xpos)), int(pos_offset), float(theta_base), _ptr(out, "out"),
                                        _dt(out.dtype), _ptr(workspace, "workspace"), nbytes, _stream(stream)))
    return out


def ret_linear_bf16(x, w, out=None, out_dtype=torch.bfloat16, stream=None):
    """Y = X W on the tensor cores; x [..., K] bf16, w [K, N] bf16."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise TypeError("x and w must be bfloat16")
    K = x.shape[-1]
    if w.dim() != 2 or w.shape[0] != K:
        raise ValueError("w must be [K, N]")
    N = w.shape[1]
    M = x.numel() // K
    _same_device(x, w=w)
    if out is None:
        out = torch.empty((*x.shape[:-1], N), dtype=out_dtype, device=x.device)
    _buf(out, "out", (*x.shape[:-1], N), FLOATS, x)
    _check(lib.ret_linear_bf16(_ptr(x, "x"), _ptr(w, "w"), _ptr(out, "out"), M, N, K, _dt(out.dtype),
                               _stream(stream)))
    return out


def ret_msr_workspace_bytes(B, N, dmodel, H, dk, dv) -> int:
    return int(lib.ret_msr_workspace_bytes(B, N, dmodel, H, dk, dv))


def ret_msr_forward(x, wq, wk, wv, wg, wo, gammas, H: int, chunk: int = 128, k_scale: float = 1.0,
                    eps: float = 1e-5, xpos: bool = True, pos_offset: int = 0, theta_base: float = 10000.0,
                    out=None, out_dtype=torch.bfloat16, workspace=None, stream=None):
    """MultiScaleRetention layer forward.  x [B, N, d_model] bf16; weights
    bf16 [in, out]; returns out [B, N, d_model]."""
    B, N, dm, dk, dv = _msr_shapes(x, wq, wk, wv, wg, wo, H)
    if out is None:
        out = torch.empty((B, N, dm), dtype=out_dtype, device=x.device)
    _buf(out, "out", (B, N, dm), FLOATS, x)
    need = ret_msr_workspace_bytes(B, N, dm, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _same_device(x, workspace=workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.ret_msr_forward(_ptr(x, "x"), _ptr(wq, "wq"), _ptr(wk, "wk"), _ptr(wv, "wv"), _ptr(wg, "wg"),
                               _ptr(wo, "wo"), _gammas(gammas, H), B, N, dm, H, dk, dv, int(chunk), float(k_scale),
                               float(eps), int(bool(xpos)), int(pos_offset), float(theta_base), _ptr(out, "out"),
                               _dt(out.dtype), _ptr(workspace, "workspace"), nbytes, _stream(stream)))
    return out
