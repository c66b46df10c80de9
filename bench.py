#!/usr/bin/env python
"""Throughput of the chunkwise retention forward on B200 (one JSON line).

Step: one chunkwise retention forward (xPos rotation, fp32 inter-chunk
state, final state written) over the long-sequence workload B=1, N=8192,
H=16, d_k=256, d_v=512, chunk 128, bf16 in / bf16 out, through the C ABI
call ret_forward_chunkwise (a tensor-core scores pass, then the
warp-specialized tensor-core kernel).  value = tokens/s of the whole job
(B*N per step per rank, summed over ranks; weak scaling, one replica per
GPU, no collective on the data path).  The decode step (64 sequences x 16
heads of 256x512 fp32 state) is timed in the same run and reported under
"decode" in state GB/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the fp64 CPU oracle (the correctness reference) on
bounded samples of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = dict(workload="retention_bf16_1x8192x16x256x512", B=1, N=8192, H=16, dk=256, dv=512, chunk=128)
DECODE = dict(workload="decode_bf16_64x16x256x512", B=64, H=16, dk=256, dv=512, prefill=1024, chunk=128, steps=512)
METRIC = "chunkwise retention fwd tokens/s"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20


def max_over_ranks(x: float, world: int, dist=None, device="cpu") -> float:
    """The maximum of ``x`` over all ranks (device time of the slowest rank)."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes
    ``units_per_rank`` per step and the job takes the slowest rank's time."""
    return world * units_per_rank / (ms_max / 1e3)


def gammas(H):
    return [1.0 - 2.0 ** (-5 - h) for h in range(H)]


def flops_per_token_head(chunk, dk, dv):
    """Algorithmic FLOPs of the chunkwise form per (token, head), full-chunk
    count: Q K^T (2 C dk) + P V (2 C dv) + cross read-out (2 dk dv) + state
    update (2 dk dv)."""
    return 2 * chunk * dk + 2 * chunk * dv + 4 * dk * dv


def flops_per_token_head_causal(chunk, dk, dv):
    """The same count with only the causal half of each chunk's score block:
    C replaced by (C + 1) / 2 in the two intra-chunk terms."""
    return (chunk + 1) * dk + (chunk + 1) * dv + 4 * dk * dv


def algo_bytes(w, out_bytes=2):
    """Read q, k, v once, write out once, write the final fp32 state once."""
    tok = w["B"] * w["N"] * w["H"]
    return tok * (2 * w["dk"] * 2 + w["dv"] * 2 + w["dv"] * out_bytes) + w["B"] * w["H"] * w["dk"] * w["dv"] * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_traffic(kernel):
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f).get(kernel)
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        loaded = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ ours ---

def run_ours(args):
    import torch
    import torch.distributed as dist

    import linear_recurrent_sequence_chunkwise_b200 as R

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    w = dict(WORKLOAD)
    if args.seq != w["N"]:
        w["N"] = args.seq
        w["workload"] = f"retention_bf16_1x{args.seq}x16x256x512"
    B, N, H, dk, dv, C = w["B"], w["N"], w["H"], w["dk"], w["dv"], w["chunk"]
    g = gammas(H)
    if args.only:
        peaks = load_peaks()
        stream = torch.cuda.current_stream()
        if args.only == "backward":
            res = {"backward": bench_backward(R, torch, dev, stream, w, g, args, peaks, world, dist)}
        elif args.only == "block":
            res = {"retnet_block": bench_block(R, torch, dev, stream, args, peaks, world, dist)}
        elif args.only == "normalized":
            res = {"normalized": bench_normalized(R, torch, dev, stream, w, g, args, peaks, world, dist)}
        else:
            res = {"msr_layer": bench_msr(R, torch, dev, stream, args, peaks, world, dist)}
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    if args.no_chunkwise:
        peaks = load_peaks()
        res = {"decode": bench_decode(R, torch, dev, torch.cuda.current_stream(), args, peaks, world, barrier, dist,
                                      rank)}
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    gen = torch.Generator(device=dev)
    gen.manual_seed(0x5EED0003 + rank)
    sc = dk ** -0.5
    q = (torch.randn((B, N, H, dk), generator=gen, device=dev) * sc).to(torch.bfloat16)
    k = (torch.randn((B, N, H, dk), generator=gen, device=dev) * sc).to(torch.bfloat16)
    v = torch.randn((B, N, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((B, N, H, dv), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # One step = one call of the library's chunkwise entry point ret_forward_chunkwise:
    # the scores pass (rotation, key scaling, masked intra-chunk scores on the
    # tensor cores) and the warp-specialized tensor-core kernel, on scratch
    # from the library's stream-ordered pool.
    def step(ev=None):
        if ev:
            ev[0].record(stream)
        R.ret_forward_chunkwise(q, k, v, g, C, out=out, final_state=fs, xpos=True, stream=stream)
        if ev:
            ev[1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    R.ret_check_device_error()
    torch.cuda.synchronize()

    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(2)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
        barrier()
    R.ret_check_device_error()
    times = [a.elapsed_time(b) for a, b in evs]  # ms per step

    # The same forward through the two-call form (same kernels, same work),
    # with CUDA events between the two launches, to time each kernel alone.
    ws2 = torch.empty(R.ret_chunkwise_prepare_workspace_bytes(B, N, H, dk, dv, C, torch.bfloat16, True),
                      dtype=torch.uint8, device=dev)
    split = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    for i in range(args.warmup + args.steps):
        flush.zero_()
        e = split[i - args.warmup] if i >= args.warmup else None
        if e:
            e[0].record(stream)
        R.ret_chunkwise_prepare(q, k, g, C, ws2, dv, xpos=True, stream=stream)
        if e:
            e[1].record(stream)
        R.ret_forward_chunkwise_prepared(q, k, v, g, C, ws2, out=out, final_state=fs, xpos=True, stream=stream)
        if e:
            e[2].record(stream)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    del ws2
    t_prep = statistics.mean(a.elapsed_time(b) for a, b, c in split) / 1e3
    t_main = statistics.mean(b.elapsed_time(c) for a, b, c in split) / 1e3
    total_ms = sum(times)
    total_ms = max_over_ranks(total_ms, world, dist, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(B * N, world, ms_per_step)

    peaks = load_peaks()
    # Dominant kernel: k_chunkwise_ws (the read-out, P V and the state
    # update on the scores pass's output), timed with CUDA events around its
    # launch on the launching stream, mean over the timed steps.  Its
    # algorithmic work is taken as the whole chunkwise forward: FLOPs of the
    # method, bytes = read q, k, v once, write out and the final state once.
    flops = flops_per_token_head(C, dk, dv) * B * N * H
    nbytes = algo_bytes(w, out_bytes=2)
    tflops = flops / t_main / 1e12
    gbs = nbytes / t_main / 1e9
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    traffic = load_traffic("k_chunkwise_ws_scores")
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4)}
    else:
        roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(tflops / peaks["bf16_tflops"], 4)}
    roof["traffic"] = traffic["bytes_per_launch"] if traffic else None
    roof["peak_source"] = peaks["source"] + " (burst; the kernel is timed alone)"
    roof["kernel"] = "k_chunkwise_ws<256, bf16, scores given>"
    roof["kernel_ms"] = round(t_main * 1e3, 4)
    roof["algo_flops"] = flops
    roof["algo_bytes"] = nbytes
    roof["tensor_tflops"] = round(tflops, 1)
    flops_causal = flops_per_token_head_causal(C, dk, dv) * B * N * H
    roof["algo_flops_causal"] = flops_causal
    roof["tensor_tflops_causal"] = round(flops_causal / t_main / 1e12, 1)
    roof["tensor_frac"] = round(tflops / peaks["bf16_tflops"], 4)
    roof["hbm_gbs"] = round(gbs, 1)
    roof["hbm_frac"] = round(gbs / peaks["hbm_gbs"], 4)
    # the same algorithmic work over the whole step (both kernels, mean step)
    t_step = ms_per_step / 1e3
    roof["step"] = {"ms": round(ms_per_step, 4), "hbm_frac": round(nbytes / t_step / 1e9 / peaks["hbm_gbs"], 4),
                    "tensor_frac": round(flops / t_step / 1e12 / peaks["bf16_tflops"], 4),
                    "roofline_ms": round(max(t_tc, t_hbm) * 1e3, 4)}
    # The scores pass: reads q, k; writes q_rot, k' and P (bf16); 2 C dk
    # FLOPs per (token, head) for the scores.
    nchunks = (N + C - 1) // C
    sc_bytes = 4 * B * N * H * dk * 2 + B * H * nchunks * C * C * 2
    scores = {"kernel": "k_prep_scores<256>", "bound": "hbm", "ms": round(t_prep * 1e3, 4),
              "achieved": round(sc_bytes / t_prep / 1e9, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
              "frac": round(sc_bytes / t_prep / 1e9 / peaks["hbm_gbs"], 4), "algo_bytes": sc_bytes,
              "traffic": (load_traffic("k_prep_scores") or {}).get("bytes_per_launch")}
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "ms_per_step_median": round(statistics.median(times), 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1); q, k scaled by d_k^-0.5)",
        "config": {"workload": w["workload"], "B": B, "N": N, "H": H, "dk": dk, "dv": dv, "chunk": C, "xpos": True,
                   "out_dtype": "bf16", "final_state": True, "global_batch": B * world, "seq_len": N,
                   "parallelism": f"replicas x{world}", "l2": "flushed before every timed step (256 MiB write)"},
        "roofline": roof, "scores_pass": scores, "clocks": clk.summary(), "gpu_launches": 2 * args.steps,
        "path": "ret_forward_chunkwise: k_prep_scores (rotation, key scaling and the masked intra-chunk scores "
                "on tcgen05, once per head) then k_chunkwise_ws (read-out, P V, state update on tcgen05)",
    }
    if not args.no_e2e:
        result["e2e"] = e2e_ours(R, torch, dev, stream, w, g, args, world, barrier, dist)
    if not args.no_decode:
        result["decode"] = bench_decode(R, torch, dev, stream, args, peaks, world, barrier, dist, rank)
    if not args.no_layer:
        result["backward"] = bench_backward(R, torch, dev, stream, w, g, args, peaks, world, dist)
        result["normalized"] = bench_normalized(R, torch, dev, stream, w, g, args, peaks, world, dist)
        result["msr_layer"] = bench_msr(R, torch, dev, stream, args, peaks, world, dist)
        result["retnet_block"] = bench_block(R, torch, dev, stream, args, peaks, world, dist)
        result["c2_d64"] = bench_c2(R, torch, dev, stream, args, peaks, world, dist)
        result["fp32_small"] = bench_fp32_small(R, torch, dev, stream, args, world, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def e2e_ours(R, torch, dev, stream, w, g, args, world, barrier, dist):
    """Same metric through the C ABI from pinned host buffers: every step
    copies q, k, v host->device, runs the forward, copies out device->host.
    The steps are pipelined the way a serving loop would run them: inputs on
    a copy-in stream, the forward on the compute stream, the output on a
    copy-out stream, two device buffers each, so that step i's output goes
    back over PCIe while step i+1's inputs come in (the link is full
    duplex).  The timed region runs from before the first copy-in to after
    the last copy-out."""
    B, N, H, dk, dv, C = w["B"], w["N"], w["H"], w["dk"], w["dv"], w["chunk"]
    hq = torch.empty((B, N, H, dk), dtype=torch.bfloat16, pin_memory=True).normal_().mul_(dk ** -0.5)
    hk = torch.empty((B, N, H, dk), dtype=torch.bfloat16, pin_memory=True).normal_().mul_(dk ** -0.5)
    hv = torch.empty((B, N, H, dv), dtype=torch.bfloat16, pin_memory=True).normal_()
    ho = [torch.empty((B, N, H, dv), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    dbuf = [tuple(torch.empty_like(x, device=dev) for x in (hq, hk, hv)) for _ in range(2)]
    do = [torch.empty((B, N, H, dv), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    steps = max(3, min(args.steps, 10))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    in_ready = [ev() for _ in range(2)]
    comp_done = [ev() for _ in range(2)]
    out_free = [ev() for _ in range(2)]
    used = [False, False]

    def step(i):
        b = i % 2
        dq, dk_, dv_ = dbuf[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(comp_done[b])        # the forward of step i-2 has read this buffer
            dq.copy_(hq, non_blocking=True)
            dk_.copy_(hk, non_blocking=True)
            dv_.copy_(hv, non_blocking=True)
            in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        if used[b]:
            stream.wait_event(out_free[b])           # step i-2's output has left this buffer
        R.ret_forward_chunkwise(dq, dk_, dv_, g, C, out=do[b], xpos=True, stream=stream)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            ho[b].copy_(do[b], non_blocking=True)
            out_free[b].record(s_out)
        used[b] = True

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev) / steps
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    return {"value": round(world * B * N / (ms / 1e3), 1), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": ho[0].numel() * ho[0].element_size(), "steps": steps,
            "pipelined": "copy-in, forward and copy-out on three streams, two buffers"}


def bench_decode(R, torch, dev, stream, args, peaks, world, barrier, dist, rank):
    """Decode step on 64 sequences x 16 heads of 256x512 fp32 state, the state
    initialised by a chunkwise prefill of a 1024-token prompt."""
    d = DECODE
    B, H, dk, dv = d["B"], d["H"], d["dk"], d["dv"]
    g = gammas(H)
    gen = torch.Generator(device=dev)
    gen.manual_seed(0x5EED0004 + rank)
    P = d["prefill"]
    pq = torch.randn((B, P, H, dk), generator=gen, device=dev).to(torch.bfloat16)
    pk = torch.randn((B, P, H, dk), generator=gen, device=dev).to(torch.bfloat16)
    pv = torch.randn((B, P, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    po = torch.empty((B, P, H, dv), dtype=torch.bfloat16, device=dev)
    state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    R.ret_forward_chunkwise(pq, pk, pv, g, d["chunk"], out=po, final_state=state, stream=stream)
    del pq, pk, pv, po
    pool = 16
    sq = torch.randn((pool, B, H, dk), generator=gen, device=dev).to(torch.bfloat16)
    sk = torch.randn((pool, B, H, dk), generator=gen, device=dev).to(torch.bfloat16)
    sv = torch.randn((pool, B, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    so = torch.empty((B, H, dv), dtype=torch.float32, device=dev)
    steps = max(args.steps, 20)
    for i in range(max(args.warmup, 3)):
        R.ret_decode_step(sq[i % pool], sk[i % pool], sv[i % pool], g, state, out=so, stream=stream)
    torch.cuda.synchronize()
    barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        evs[i][0].record(stream)
        R.ret_decode_step(sq[i % pool], sk[i % pool], sv[i % pool], g, state, out=so, stream=stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    per_step = [a.elapsed_time(b) for a, b in evs]
    ms = statistics.mean(per_step)
    ms = max_over_ranks(ms, world, dist, dev)
    # The workload's whole generation loop: 512 steps back to back after the
    # prefill, timed as one region, eagerly and replayed from a CUDA graph.
    loop = d["steps"]

    def run_loop(st):
        for i in range(loop):
            R.ret_decode_step(sq[i % pool], sk[i % pool], sv[i % pool], g, state, out=so, stream=st)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run_loop(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    loop_ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        run_loop(None)  # the capturing stream
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    graph_ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev)
    del graph
    nbytes = 2 * B * H * dk * dv * 4 + B * H * (2 * dk * 2 + dv * 2 + dv * 4)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": d["workload"], "metric": "decode-step state HBM GB/s", "value": round(gbs * world, 1),
            "unit": "GB/s", "ms_per_step": round(ms, 4), "ms_per_step_median": round(statistics.median(per_step), 4),
            "steps": steps, "bytes_per_step": nbytes,
            "loop": {"steps": loop, "ms_total": round(loop_ms, 3), "ms_total_graph": round(graph_ms, 3),
                     "ms_per_step": round(loop_ms / loop, 4), "ms_per_step_graph": round(graph_ms / loop, 4)},
            "tokens_per_s": round(world * B / (ms / 1e3), 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "kernel": "k_decode_step",
                         "traffic": (load_traffic("k_decode_step") or {}).get("bytes_per_launch")},
            "l2": "state (537 MB) larger than L2"}


def _timed(torch, stream, fn, steps, warmup, world, dist, dev):
    """Mean CUDA-event time (ms) of fn() over `steps` calls after `warmup`,
    max over ranks."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), world, dist, dev)


def bench_backward(R, torch, dev, stream, w, g, args, peaks, world, dist):
    """Gradients of the chunkwise forward (dq, dk, dv in fp32) on the same
    workload: three tensor-core retention passes (dq and dk in two d_v slices
    each), the anti-causal two on the time-reversed sequence.  Algorithmic
    FLOPs: three times the forward's."""
    B, N, H, dk, dv, C = w["B"], w["N"], w["H"], w["dk"], w["dv"], w["chunk"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(0x5EED0006)
    sc = dk ** -0.5
    q = (torch.randn((B, N, H, dk), generator=gen, device=dev) * sc).to(torch.bfloat16)
    k = (torch.randn((B, N, H, dk), generator=gen, device=dev) * sc).to(torch.bfloat16)
    v = torch.randn((B, N, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    do = torch.randn((B, N, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    dq = torch.empty((B, N, H, dk), dtype=torch.float32, device=dev)
    dkk = torch.empty_like(dq)
    dvv = torch.empty((B, N, H, dv), dtype=torch.float32, device=dev)
    ws = torch.empty(R.ret_backward_workspace_bytes(B, N, H, dk, dv, C, torch.bfloat16, True), dtype=torch.uint8,
                     device=dev)

    def fn():
        R.ret_backward_chunkwise(q, k, v, do, g, C, workspace=ws, dq=dq, dk=dkk, dv=dvv, xpos=True, stream=stream)

    ms = _timed(torch, stream, fn, max(3, min(args.steps, 10)), 3, world, dist, dev)
    R.ret_check_device_error()
    flops = 3 * flops_per_token_head(C, dk, dv) * B * N * H
    tf = flops / (ms / 1e3) / 1e12
    return {"workload": w["workload"], "ms_per_step": round(ms, 4), "tokens_per_s": round(world * B * N / (ms / 1e3), 1),
            "algo_flops": flops,
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tf / peaks["bf16_tflops"], 4),
                         "kernels": "5 x (k_prep_qk + k_chunkwise_ws), 6 x k_row_transform"}}


def bench_normalized(R, torch, dev, stream, w, g, args, peaks, world, dist):
    """The chunkwise forward with the score normalizations 2 and 3 on the same
    workload (one call: the rotation + zeta pass, three passes for the row
    factors, the tensor-core kernel with the factors in its epilogue), final
    S and z written.  Compared with the plain forward of the same call
    shape, timed the same way."""
    B, N, H, dk, dv, C = w["B"], w["N"], w["H"], w["dk"], w["dv"], w["chunk"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(0x5EED0007)
    sc = dk ** -0.5
    q = (torch.randn((B, N, H, dk), generator=gen, device=dev) * sc).to(torch.bfloat16)
    k = (torch.randn((B, N, H, dk), generator=gen, device=dev) * sc).to(torch.bfloat16)
    v = torch.randn((B, N, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((B, N, H, dv), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    fz = torch.empty((B, H, dk), dtype=torch.float32, device=dev)
    ws = torch.empty(R.ret_normalized_workspace_bytes(B, N, H, dk, dv, C, torch.bfloat16, True), dtype=torch.uint8,
                     device=dev)

    def norm():
        R.ret_forward_chunkwise_normalized(q, k, v, g, C, norm_flags=R.NORM_DECAY | R.NORM_SCORE, workspace=ws,
                                           out=out, final_state=fs, final_z=fz, xpos=True, stream=stream)

    def plain():
        R.ret_forward_chunkwise(q, k, v, g, C, out=out, final_state=fs, xpos=True, stream=stream)

    steps = max(5, min(args.steps, 20))
    ms = _timed(torch, stream, norm, steps, 3, world, dist, dev)
    ms_plain = _timed(torch, stream, plain, steps, 3, world, dist, dev)
    R.ret_check_device_error()
    return {"workload": w["workload"], "flags": "decay + score", "ms_per_step": round(ms, 4),
            "tokens_per_s": round(world * B * N / (ms / 1e3), 1), "plain_ms_per_step": round(ms_plain, 4),
            "overhead": round(ms / ms_plain - 1.0, 4),
            "kernels": "k_prep_scores, k_keysum, k_keycarry, k_rowscale, k_chunkwise_ws (scores given, row factors in the epilogue)",
            "plain": "ret_forward_chunkwise (k_prep_scores + k_chunkwise_ws)"}


def bench_msr(R, torch, dev, stream, args, peaks, world, dist):
    """The MultiScaleRetention layer forward on X [2, 4096, 2048] (H 8, d_k 256,
    d_v 512, xPos, chunk 128): four projections, retention, GroupNorm + swish
    gate and the output projection.  Tensor-bound: 549.8 GFLOP of GEMMs plus
    47.2 GFLOP of retention."""
    B, N, dm, H, dk, dv = 2, 4096, 2048, 8, 256, 512
    gen = torch.Generator(device=dev)
    gen.manual_seed(0x5EED0005)
    x = torch.randn((B, N, dm), generator=gen, device=dev).to(torch.bfloat16)
    w = {n: (torch.randn(shape, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
         for n, shape in (("wq", (dm, H * dk)), ("wk", (dm, H * dk)), ("wv", (dm, H * dv)), ("wg", (dm, H * dv)),
                          ("wo", (H * dv, dm)))}
    out = torch.empty((B, N, dm), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(R.ret_msr_workspace_bytes(B, N, dm, H, dk, dv), dtype=torch.uint8, device=dev)
    g = gammas(H)

    def fn():
        R.ret_msr_forward(x, w["wq"], w["wk"], w["wv"], w["wg"], w["wo"], g, H=H, chunk=128, k_scale=dk ** -0.5,
                          xpos=True, out=out, workspace=ws, stream=stream)

    ms = _timed(torch, stream, fn, max(5, min(args.steps, 20)), 3, world, dist, dev)
    R.ret_check_device_error()
    M = B * N
    gemm = 2 * M * dm * (2 * H * dk + 2 * H * dv) + 2 * M * H * dv * dm
    ret = flops_per_token_head(128, dk, dv) * B * N * H
    tf = (gemm + ret) / (ms / 1e3) / 1e12
    return {"workload": "msr_layer_bf16_2x4096x2048_h8_256_512", "ms_per_step": round(ms, 4),
            "tokens_per_s": round(world * M / (ms / 1e3), 1), "algo_flops": gemm + ret,
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4),
                         "kernels": "k_gemm (the 4 projections, fused rotation/zeta/swish epilogue), "
                                    "k_chunkwise_ws, k_gn_gate, k_gemm (W_O)"}}


def bench_block(R, torch, dev, stream, args, peaks, world, dist):
    """One RetNet block on the MSR layer's shapes plus the FFN (d_ff = 2
    d_model = 4096): LayerNorm, the MSR layer with the residual fused in
    W_O, LayerNorm, gelu(Y W1) W2 + Y.  Tensor-bound: the MSR's FLOPs plus
    2 x 2 M d_model d_ff for the FFN."""
    B, N, dm, H, dk, dv, dff = 2, 4096, 2048, 8, 256, 512, 4096
    gen = torch.Generator(device=dev)
    gen.manual_seed(0x5EED0008)
    x = torch.randn((B, N, dm), generator=gen, device=dev).to(torch.bfloat16)
    w = {n: (torch.randn(shape, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
         for n, shape in (("wq", (dm, H * dk)), ("wk", (dm, H * dk)), ("wv", (dm, H * dv)), ("wg", (dm, H * dv)),
                          ("wo", (H * dv, dm)), ("w1", (dm, dff)), ("w2", (dff, dm)))}
    out = torch.empty((B, N, dm), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(R.ret_retnet_block_workspace_bytes(B, N, dm, H, dk, dv, dff), dtype=torch.uint8, device=dev)
    g = gammas(H)

    def fn():
        R.ret_retnet_block_forward(x, w["wq"], w["wk"], w["wv"], w["wg"], w["wo"], w["w1"], w["w2"], g, H=H,
                                   chunk=128, k_scale=dk ** -0.5, xpos=True, out=out, workspace=ws, stream=stream)

    ms = _timed(torch, stream, fn, max(5, min(args.steps, 20)), 3, world, dist, dev)
    R.ret_check_device_error()
    M = B * N
    gemm = 2 * M * dm * (2 * H * dk + 2 * H * dv) + 2 * M * H * dv * dm + 2 * 2 * M * dm * dff
    ret = flops_per_token_head(128, dk, dv) * B * N * H
    tf = (gemm + ret) / (ms / 1e3) / 1e12
    return {"workload": "retnet_block_bf16_2x4096x2048_h8_256_512_ff4096", "ms_per_step": round(ms, 4),
            "tokens_per_s": round(world * M / (ms / 1e3), 1), "algo_flops": gemm + ret,
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4),
                         "kernels": "k_layernorm, the MSR layer's four, k_layernorm, k_gemm (W1, gelu), "
                                    "k_gemm (W2, residual)"}}


def _timed_flushed(torch, stream, fn, steps, warmup, world, dist, dev, flush):
    """Mean CUDA-event time (ms) of fn() over `steps` calls after `warmup`,
    with the L2 flushed (a 256 MiB write) before every call, outside the
    events; max over ranks."""
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), world, dist, dev)


def bench_c2(R, torch, dev, stream, args, peaks, world, dist):
    """The pages' cost-analysis shape [4, 2048, 8 heads of 64], bf16, xPos,
    chunk 64, L2 flushed before every call: the single allocating call
    ret_forward_chunkwise (d_k padded to 128 on the tensor cores, 128-token
    blocks).  HBM-bound: algorithmic bytes = read q, k, v once, write out
    once (bf16)."""
    B, N, H, dk, dv, C = 4, 2048, 8, 64, 64, 64
    gen = torch.Generator(device=dev)
    gen.manual_seed(0x5EED0009)
    q = (torch.randn((B, N, H, dk), generator=gen, device=dev) * dk ** -0.5).to(torch.bfloat16)
    k = (torch.randn((B, N, H, dk), generator=gen, device=dev) * dk ** -0.5).to(torch.bfloat16)
    v = torch.randn((B, N, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((B, N, H, dv), dtype=torch.bfloat16, device=dev)
    g = gammas(H)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def fused():
        R.ret_forward_chunkwise(q, k, v, g, C, out=out, xpos=True, stream=stream)

    steps = max(5, min(args.steps, 20))
    ms = _timed_flushed(torch, stream, fused, steps, 3, world, dist, dev, flush)
    R.ret_check_device_error()
    nbytes = B * N * H * (2 * dk * 2 + dv * 2 + dv * 2)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": "retention_bf16_4x2048x8x64", "tokens_per_s": round(world * B * N / (ms / 1e3), 1),
            "ms_per_step": round(ms, 4),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "algo_bytes": nbytes,
                         "peak_source": peaks["source"]},
            "l2": "flushed before every timed call (256 MiB write)",
            "path": "ret_forward_chunkwise: k_prep_scores<128> + k_chunkwise_ws<128>, d_k padded to 128, "
                    "128-token blocks"}


def bench_fp32_small(R, torch, dev, stream, args, world, dist):
    """The fp32 path at the exercise shape [1, 64, 8, 16], chunk 16 (CUDA cores;
    136 KB of I/O, so the figure is launch latency)."""
    B, N, H, d = 1, 64, 8, 16
    gen = torch.Generator(device=dev)
    gen.manual_seed(0x5EED0001)
    q, k, v = (torch.randn((B, N, H, d), generator=gen, device=dev) for _ in range(3))
    out = torch.empty((B, N, H, d), dtype=torch.float32, device=dev)
    g = gammas(H)

    def fn():
        R.ret_forward_chunkwise(q, k, v, g, 16, out=out, stream=stream)

    ms = _timed(torch, stream, fn, 50, 5, world, dist, dev)
    R.ret_check_device_error()
    # The same call replayed from a CUDA graph of 100 calls: the launch cost
    # a serving loop pays when it captures its steps.
    reps = 100
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for _ in range(reps):
            R.ret_forward_chunkwise(q, k, v, g, 16, out=out)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    graph.replay()
    b.record(stream)
    torch.cuda.synchronize()
    R.ret_check_device_error()
    us_graph = max_over_ranks(a.elapsed_time(b), world, dist, dev) * 1e3 / reps
    del graph
    return {"workload": "retention_f32_1x64x8x16", "us_per_call": round(ms * 1e3, 2),
            "us_per_call_graph_replay": round(us_graph, 2), "bound": "latency", "kernel": "k_chunkwise_simt"}


# ---------------------------------------------------------- the oracle ---

def oracle_sample(w, heads, n_tok, nthreads=0):
    """One bounded oracle run: ``heads`` heads of the workload over the first
    ``n_tok`` tokens (rotation + recurrent definition, fp64, all host cores).
    Returns (seconds, tokens of the full workload this sample stands for)."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(1)
    B, dk, dv = w["B"], w["dk"], w["dv"]
    q = rng.standard_normal((B, n_tok, heads, dk)) / 16
    k = rng.standard_normal((B, n_tok, heads, dk)) / 16
    v = rng.standard_normal((B, n_tok, heads, dv))
    g = np.array(gammas(w["H"])[:heads])
    t0 = time.perf_counter()
    oracle.retention_recurrent(oracle.xpos_rotate(q), oracle.xpos_rotate(k), v, g, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return dt, B * n_tok * heads / w["H"]


def cpu_baseline(w, budget_s=20.0):
    import oracle
    cores = oracle.max_threads()
    heads = min(w["H"], cores)
    dt, tok = oracle_sample(w, heads, 256)           # calibrate
    n = int(min(w["N"], max(256, 256 * budget_s / max(dt, 1e-3))))
    dt, tok = oracle_sample(w, heads, n)
    # one host core: one head, a few seconds of work
    d1, t1 = oracle_sample(w, 1, 256, nthreads=1)
    n1 = int(min(w["N"], max(256, 256 * (budget_s / 5) / max(d1, 1e-3))))
    d1, t1 = oracle_sample(w, 1, n1, nthreads=1)
    return {"value": round(tok / dt, 2), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{heads} of {w['H']} heads x first {n} of {w['N']} tokens, fp64 recurrent definition "
                      f"with xPos, {dt:.1f} s; value scaled to tokens of the full workload",
            "single_core": {"value": round(t1 / d1, 2), "unit": UNIT, "cores": 1,
                            "sample": f"1 head x first {n1} tokens, {d1:.1f} s; scaled to the full workload"}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = dict(WORKLOAD)
    cores = oracle.max_threads()
    heads = min(w["H"], cores)
    n_tok = 512
    for _ in range(args.warmup):
        oracle_sample(w, heads, n_tok)
    times, tok = [], 0
    for _ in range(args.steps):
        dt, tok = oracle_sample(w, heads, n_tok)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = tok / (ms / 1e3)
    sample = (f"{heads} of {w['H']} heads x first {n_tok} of {w['N']} tokens per step, fp64 recurrent "
              f"definition with xPos; value scaled to tokens of the full workload")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1))",
        "config": {"workload": w["workload"], "B": w["B"], "N": w["N"], "H": w["H"], "dk": w["dk"], "dv": w["dv"],
                   "chunk": w["chunk"], "xpos": True, "global_batch": w["B"], "seq_len": w["N"],
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-layer", action="store_true", help="skip the MSR-layer and fp32 small-shape timings")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--seq", type=int, default=WORKLOAD["N"],
                    help="sequence length of the chunkwise workload (smaller values make ncu captures short)")
    ap.add_argument("--no-chunkwise", action="store_true", help="skip the chunkwise forward (decode only)")
    ap.add_argument("--only", choices=["backward", "msr", "normalized", "block"],
                    help="time only the backward or only the MSR layer (for ncu launch lists of one part)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
