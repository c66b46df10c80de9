"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the retention method: it only draws
numbers, rounds them to the storage dtype and names the workloads.  Both the
oracle side and the CUDA side receive their inputs from here.

Generator: numpy's Philox4x64-10 counter-based bit generator (Salmon et al.,
"Parallel random numbers: as easy as 1, 2, 3", SC'11), keyed by
(seed << 32) | stream, feeding numpy's standard-normal sampler in float32.
bf16 storage is IEEE round-to-nearest-even of those float32 draws.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------- drawing ---


def normal_f32(seed: int, stream: int, shape, scale: float = 1.0) -> np.ndarray:
    """iid N(0, 1) * scale as float32, reproducible from (seed, stream)."""
    gen = np.random.Generator(np.random.Philox(key=(int(seed) << 32) | int(stream)))
    x = gen.standard_normal(size=tuple(shape), dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 -> bf16 (round to nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


class Tensor:
    """One synthetic tensor: its stored form (uint16 bf16 bits or float32)
    and, on demand, the stored values widened exactly to float64."""

    def __init__(self, dtype: str, stored: np.ndarray):
        self.dtype = dtype
        self.stored = stored
        self._f64 = None

    @property
    def shape(self):
        return self.stored.shape

    def f64_at(self, index) -> np.ndarray:
        """Widened values of ``stored[index]`` (no full-size copy)."""
        part = self.stored[index]
        if self.dtype == "bf16":
            return bf16_bits_to_f32(part).astype(np.float64)
        return np.asarray(part, dtype=np.float64)

    @property
    def f64(self) -> np.ndarray:
        if self._f64 is None:
            self._f64 = self.f64_at(...)
        return self._f64


def make_tensor(seed: int, stream: int, shape, dtype: str, scale: float = 1.0) -> Tensor:
    x = normal_f32(seed, stream, shape, scale)
    if dtype == "bf16":
        return Tensor("bf16", f32_to_bf16_bits(x))
    if dtype == "f32":
        return Tensor("f32", x)
    raise ValueError(dtype)


def to_torch(t: Tensor, device="cpu"):
    """The stored form as a torch tensor (bf16 or float32) on ``device``."""
    import torch
    if t.dtype == "bf16":
        return torch.from_numpy(t.stored.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(t.stored.copy()).to(device)


# ------------------------------------------------------------- workloads ---


def gamma_schedule(H: int) -> np.ndarray:
    """Per-head decay gamma_h = 1 - 2^(-5-h), h = 0..H-1 (multi-scale
    retention schedule; exact in binary floating point)."""
    return 1.0 - np.exp2(-5.0 - np.arange(H, dtype=np.float64))


def gamma_schedule_scaled(H: int) -> np.ndarray:
    """The schedule of the larger models: gamma = 1 - exp(linspace(log 1/32,
    log 1/512, H)), 1 - gamma log-spaced from 1/32 to 1/512 (RetNet paper
    summary, multi-scale decay).  H = 1 takes the first end point."""
    if H == 1:
        return np.array([1.0 - 1.0 / 32])
    return 1.0 - np.exp(np.linspace(np.log(1.0 / 32), np.log(1.0 / 512), H))


SEED_BASE = 0x5EED0000
# sub-streams of a workload's seed
STREAM_Q, STREAM_K, STREAM_V = 1, 2, 3
STREAM_X, STREAM_WQ, STREAM_WK, STREAM_WV, STREAM_WG, STREAM_WO = 4, 5, 6, 7, 8, 9
STREAM_W1, STREAM_W2 = 10, 11     # the RetNet block's FFN
STREAM_DECODE0 = 1000   # decode step s draws q, k, v from streams 1000 + 3s + {0, 1, 2}


@dataclass
class Workload:
    name: str
    B: int
    N: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str
    qk_scale: float
    xpos: bool
    final_state: bool = False
    decode_steps: int = 0
    dmodel: int = 0
    w_std: float = 0.0
    gn_eps: float = 1e-5
    seed: int = SEED_BASE
    notes: str = ""
    gammas: np.ndarray = field(default=None)

    def __post_init__(self):
        if self.gammas is None:
            self.gammas = gamma_schedule(self.H)

    def qkv(self, B=None, N=None, seed=None, stream_base=0):
        """(q, k, v) Tensors of shape [B, N, H, d]; q and k carry qk_scale."""
        B = self.B if B is None else B
        N = self.N if N is None else N
        s = self.seed if seed is None else seed
        q = make_tensor(s, stream_base + STREAM_Q, (B, N, self.H, self.dk), self.dtype, self.qk_scale)
        k = make_tensor(s, stream_base + STREAM_K, (B, N, self.H, self.dk), self.dtype, self.qk_scale)
        v = make_tensor(s, stream_base + STREAM_V, (B, N, self.H, self.dv), self.dtype)
        return q, k, v

    def decode_qkv(self, step: int):
        """Fresh (q, k, v) for decode step ``step``: [B, H, d]."""
        base = STREAM_DECODE0 + 3 * step
        q = make_tensor(self.seed, base + 0, (self.B, self.H, self.dk), self.dtype, self.qk_scale)
        k = make_tensor(self.seed, base + 1, (self.B, self.H, self.dk), self.dtype, self.qk_scale)
        v = make_tensor(self.seed, base + 2, (self.B, self.H, self.dv), self.dtype)
        return q, k, v


# The five workloads.  Shapes follow the pages: P5's exercise (1, 64, 8, 16),
# P1's cost-analysis model (d_model 512, 8 heads of 64), and the 6.7B-class
# heads of the RetNet paper (d_k 256, d_v 512) at 8k length.
WORKLOADS = {
    "retention_fp32_1x64x8x16": Workload(
        "retention_fp32_1x64x8x16", B=1, N=64, H=8, dk=16, dv=16, chunk=16, dtype="f32",
        qk_scale=1.0, xpos=False, final_state=True, seed=SEED_BASE + 1),
    "retention_bf16_4x2048x8x64": Workload(
        "retention_bf16_4x2048x8x64", B=4, N=2048, H=8, dk=64, dv=64, chunk=64, dtype="bf16",
        qk_scale=64 ** -0.5, xpos=True, final_state=True, seed=SEED_BASE + 2),
    "retention_bf16_1x8192x16x256x512": Workload(
        "retention_bf16_1x8192x16x256x512", B=1, N=8192, H=16, dk=256, dv=512, chunk=128,
        dtype="bf16", qk_scale=256 ** -0.5, xpos=True, final_state=True, seed=SEED_BASE + 3),
    "decode_bf16_64x16x256x512": Workload(
        "decode_bf16_64x16x256x512", B=64, N=1024, H=16, dk=256, dv=512, chunk=128,
        dtype="bf16", qk_scale=1.0, xpos=False, final_state=True, decode_steps=512,
        seed=SEED_BASE + 4),
    "msr_layer_2x4096x2048": Workload(
        "msr_layer_2x4096x2048", B=2, N=4096, H=8, dk=256, dv=512, chunk=128, dtype="bf16",
        qk_scale=256 ** -0.5, xpos=True, dmodel=2048, w_std=0.02, seed=SEED_BASE + 5),
}
C1, C2, C3, C4, C5 = (WORKLOADS[k] for k in WORKLOADS)


def msr_weights(w: Workload, dmodel=None, H=None, dk=None, dv=None, seed=None):
    """X and the five projection matrices of the MSR layer, bf16."""
    dm = w.dmodel if dmodel is None else dmodel
    H = w.H if H is None else H
    dk = w.dk if dk is None else dk
    dv = w.dv if dv is None else dv
    s = w.seed if seed is None else seed
    return {
        "wq": make_tensor(s, STREAM_WQ, (dm, H * dk), "bf16", w.w_std),
        "wk": make_tensor(s, STREAM_WK, (dm, H * dk), "bf16", w.w_std),
        "wv": make_tensor(s, STREAM_WV, (dm, H * dv), "bf16", w.w_std),
        "wg": make_tensor(s, STREAM_WG, (dm, H * dv), "bf16", w.w_std),
        "wo": make_tensor(s, STREAM_WO, (H * dv, dm), "bf16", w.w_std),
    }


def ffn_weights(w: Workload, dmodel=None, dff=None, seed=None):
    """W1 [d_model, d_ff] and W2 [d_ff, d_model] of the RetNet block's FFN,
    bf16, with the layer's weight scale; d_ff = 2 d_model unless given."""
    dm = w.dmodel if dmodel is None else dmodel
    dff = 2 * dm if dff is None else dff
    s = w.seed if seed is None else seed
    return {"w1": make_tensor(s, STREAM_W1, (dm, dff), "bf16", w.w_std),
            "w2": make_tensor(s, STREAM_W2, (dff, dm), "bf16", w.w_std)}


def msr_input(w: Workload, B=None, N=None, dmodel=None, seed=None):
    B = w.B if B is None else B
    N = w.N if N is None else N
    dm = w.dmodel if dmodel is None else dmodel
    s = w.seed if seed is None else seed
    return make_tensor(s, STREAM_X, (B, N, dm), "bf16")
