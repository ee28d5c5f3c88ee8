#!/usr/bin/env python
"""Throughput benchmark of the sigmoid-attention library on B200.

One step = one pass of the whole hot path over one batch: the forward call and
both backward calls (dQ, then dK/dV), each of which runs the ragged plan and
its compute kernel. The headline value counts valid-token FLOPs only
(4*d per valid (i, j) pair forward + 10*d backward, the usual five-product
count) divided by the device time of the timed steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

With N > 1 every rank (one process per GPU, started by torch.distributed.run;
bench.py starts that launcher itself when it was not started by one) runs its
own batch of the same workload: the (b, h) slices are independent, so the work
shards with no collective on the data path (weak scaling). Rank 0 prints one
JSON line. A launcher whose WORLD_SIZE differs from --gpus is an error.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sigmoid-attn fwd & bwd TFLOPS (valid tokens) on 1 B200; % of BF16 tensor peak"
L2_BYTES = 126 * 1024 * 1024
# Matrix-product FLOPs each call performs per valid (i, j) pair, in units of d:
# forward S and PV; dQ kernel S, dP, dQ; dK/dV kernel S, dP, dV, dK.
KERNEL_FLOPS_PER_PAIR = {"fwd": 4, "bwd_dq": 6, "bwd_dkdv": 8}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"bf16_tflops": float(p["bf16_tflops"]), "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]),
                "hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def _csrc_hash() -> str:
    """Hash of the kernel sources with // comments and blank lines removed, so
    that the committed ncu traffic stays tied to the code, not to its comments."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sigmoid_attention_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                code = [line.split("//", 1)[0].rstrip() for line in f]
            h.update(name.encode() + "\n".join(line for line in code if line).encode())
    return h.hexdigest()[:16]


def _traffic(kernel: str, workload: str, launches_scale: float = 1.0):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when the summary was taken on other kernel sources or another workload."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("csrc_hash") != _csrc_hash():
        return None
    entry = t.get("kernels", {}).get(kernel, {}).get(workload)
    if not entry:
        return None
    return float(entry["dram_bytes_per_launch"]) * launches_scale


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[2:]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, max_seconds: float) -> float:
    """Units all ranks processed divided by the slowest rank's time."""
    return flops_per_rank * world / max_seconds / 1e12


def cpu_baseline(w, target_s: float = 12.0):
    """The fp64 oracle, as it stands, on the host cores: forward + backward of
    whole (b, h) slices of the workload's first sequence, as many heads as fit
    in about `target_s` seconds (at least one)."""
    import oracle
    from sigmoid_attention_b200 import workloads

    q, k, v, dout = workloads.make_inputs(1, w.H, w.L, w.d, w.seed)
    n = int(w.lengths()[0])
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    done_heads, spent = 0, 0.0
    while done_heads < w.H and (done_heads == 0 or spent * (done_heads + 1) / done_heads <= target_s):
        sl = slice(done_heads, done_heads + 1)
        t0 = time.perf_counter()
        oracle.forward(q[:, sl], k[:, sl], v[:, sl], [n])
        oracle.backward(q[:, sl], k[:, sl], v[:, sl], dout[:, sl], [n])
        spent += time.perf_counter() - t0
        done_heads += 1
    flops = 14.0 * w.d * n * n * done_heads
    return {"value": flops / spent / 1e12, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
            "sample": f"{done_heads} (b,h) slice(s) of sequence 0 (n={n}, d={w.d}), fwd+bwd in fp64, "
                      f"{spent:.1f} s"}


def run_reference(args, w):
    """The reference arm: the oracle timed on the host cores (rank 0 only)."""
    world, rank, _ = _dist_env()
    if rank != 0:
        return 0
    import oracle
    from sigmoid_attention_b200 import workloads

    q, k, v, dout = workloads.make_inputs(1, 1, w.L, w.d, w.seed)
    n = int(w.lengths()[0])
    # One step = forward + backward of one (b, h) slice, shortened to m query
    # rows and m key rows when a full slice would not fit the time budget.
    budget = 150.0 / max(1, args.steps + args.warmup)
    m0 = min(n, 512)
    t0 = time.perf_counter()
    oracle.forward(q[..., :m0, :], k[..., :m0, :], v[..., :m0, :], [m0])
    oracle.backward(q[..., :m0, :], k[..., :m0, :], v[..., :m0, :], dout[..., :m0, :], [m0])
    per_pair = (time.perf_counter() - t0) / (m0 * m0)
    m = n
    while m > 64 and per_pair * m * m > budget:
        m //= 2
    qs, ks, vs, ds = (t[:, :, :m].contiguous() for t in (q, k, v, dout))
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.forward(qs, ks, vs, [m])
        oracle.backward(qs, ks, vs, ds, [m])
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = float(np.mean(times))
    flops = 14.0 * w.d * m * m
    value = flops / sec / 1e12
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    sample = f"one (b,h) slice of sequence 0 cut to {m} of its {n} tokens, fwd+bwd in fp64"
    line = {"metric": METRIC, "value": value, "unit": "TFLOPS", "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**w.describe(), "step": "oracle fwd+bwd of a bounded sample"},
            "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _run_calls(calls, stream, ev=None):
    """One step: the forward, dQ and dK/dV calls (or the forward and the
    whole-backward call), with an event before each call and after the last
    when `ev` (len(calls) + 1 CUDA events) is given."""
    for i, call in enumerate(calls):
        if ev is not None:
            ev[i].record(stream)
        call()
    if ev is not None:
        ev[len(calls)].record(stream)


def _check_status(sa, ws, stream):
    st, site = sa.sigattn_read_error(ws, stream)
    if st != 0:
        raise SystemExit(f"kernel reported status {st} at site {site}")


def _device_steps(calls, stream, steps, warmup, flush_buf=None, sync_ranks=None, check=None, sampler=None,
                  names=("fwd", "bwd_dq", "bwd_dkdv")):
    """Device time of each call over `steps` timed steps after `warmup`
    untimed ones: CUDA events on the launching stream, a synchronize (and a
    barrier over ranks, when given) on both sides of the timed region, and an
    L2 flush (a write of flush_buf) between steps outside the events. A clock
    `sampler` (context manager) runs during the timed region only."""
    import contextlib

    import torch

    for _ in range(warmup):
        _run_calls(calls, stream)
        if flush_buf is not None:
            flush_buf.zero_()
    if check is not None:
        check()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
    if sync_ranks is not None:
        sync_ranks()
    torch.cuda.synchronize()
    with sampler if sampler is not None else contextlib.nullcontext():
        for i in range(steps):
            _run_calls(calls, stream, events[i])
            if flush_buf is not None:
                flush_buf.zero_()
        torch.cuda.synchronize()
    if sync_ranks is not None:
        sync_ranks()
    if check is not None:
        check()
    per_kernel = {name: [] for name in names}
    step_ms = []
    for ev in events:
        for i, name in enumerate(names):
            per_kernel[name].append(ev[i].elapsed_time(ev[i + 1]))
        step_ms.append(ev[0].elapsed_time(ev[-1]))
    return per_kernel, step_ms


def _fused_backward(per_kernel_sep, fused_calls, stream, steps, warmup, flush_buf, check, flops_fwd, flops_bwd):
    """The same step with the whole-backward call (sigattn_bwd: the dQ and
    dK/dV kernels overlapped) instead of the two backward calls, timed the
    same way right after the separate-call steps."""
    per_kernel, step_ms = _device_steps(fused_calls, stream, steps, warmup, flush_buf, check=check,
                                        names=("fwd", "bwd"))
    bwd_ms = float(np.mean(per_kernel["bwd"]))
    sep_ms = float(np.mean(per_kernel_sep["bwd_dq"])) + float(np.mean(per_kernel_sep["bwd_dkdv"]))
    return {"value": (flops_fwd + flops_bwd) / (np.mean(step_ms) / 1e3) / 1e12,
            "bwd_ms": bwd_ms, "bwd_tflops": flops_bwd / (bwd_ms / 1e3) / 1e12,
            "bwd_speedup_vs_two_calls": sep_ms / bwd_ms,
            "step": "sigattn_fwd + sigattn_bwd (dQ and dK/dV kernels overlapped)"}


def side_workloads(names, dev, steps: int, warmup: int) -> dict:
    """Device-timed fwd / bwd / step TFLOPS of other workloads in the same run
    (padded layout, L2 flushed between steps), with the padding-sweep ratio
    of 75 % padding to unpadded."""
    import torch

    import sigmoid_attention_b200 as sa
    from sigmoid_attention_b200 import workloads

    out = {}
    stream = torch.cuda.current_stream(dev)
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    for name in names:
        w = workloads.WORKLOADS[name]
        q, k, v, dout, lengths = workloads.workload_inputs(w)
        qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
        lens = lengths.to(dev)
        o, dq, dk, dv = (torch.empty_like(qd) for _ in range(4))
        ws = sa.make_workspace(w.B, w.H, w.L, w.d, dev)
        calls = (lambda: sa.sigattn_fwd(qd, kd, vd, o, lens, ws, stream),
                 lambda: sa.sigattn_bwd_dq(qd, kd, vd, dod, dq, lens, ws, stream),
                 lambda: sa.sigattn_bwd_dkdv(qd, kd, vd, dod, dk, dv, lens, ws, stream))
        per_kernel, step_ms = _device_steps(calls, stream, steps, warmup, flush_buf,
                                            check=lambda: _check_status(sa, ws, stream))
        f_fwd, f_bwd = w.fwd_flops(), w.bwd_flops()
        ms = {kname: float(np.mean(v_)) for kname, v_ in per_kernel.items()}
        fused_calls = (calls[0], lambda: sa.sigattn_bwd(qd, kd, vd, dod, dq, dk, dv, lens, ws, stream))
        out[name] = {"value": (f_fwd + f_bwd) / (np.mean(step_ms) / 1e3) / 1e12,
                     "fwd_tflops": f_fwd / (ms["fwd"] / 1e3) / 1e12,
                     "bwd_tflops": f_bwd / ((ms["bwd_dq"] + ms["bwd_dkdv"]) / 1e3) / 1e12,
                     "ms": ms, "steps": steps,
                     "step_fused": _fused_backward(per_kernel, fused_calls, stream, steps, warmup, flush_buf,
                                                   lambda: _check_status(sa, ws, stream), f_fwd, f_bwd)}
        del qd, kd, vd, dod, o, dq, dk, dv, ws
    if "pad_sweep_p00" in out and "pad_sweep_p75" in out:
        out["p75_over_p00"] = out["pad_sweep_p75"]["value"] / out["pad_sweep_p00"]["value"]
        out["p75_over_p00_fused"] = (out["pad_sweep_p75"]["step_fused"]["value"] /
                                     out["pad_sweep_p00"]["step_fused"]["value"])
    return out


def softmax_comparison(name: str, dev, steps: int = 10, warmup: int = 3) -> dict:
    """Forward TFLOPS of the sigmoid kernel and of its softmax counterpart
    (same plan, scheduler, loads and MMAs; softmax over the valid keys) on
    one workload, device-timed the same way (L2 flushed between steps): the
    comparison of "Better Models, Faster Training" sec. 4A, at its 25%
    padding when run on pad_sweep_p25."""
    import torch

    import sigmoid_attention_b200 as sa
    from sigmoid_attention_b200 import workloads

    w = workloads.WORKLOADS[name]
    q, k, v, _, lengths = workloads.workload_inputs(w)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    lens = lengths.to(dev)
    o = torch.empty_like(qd)
    ws = sa.make_workspace(w.B, w.H, w.L, w.d, dev)
    stream = torch.cuda.current_stream(dev)
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    out = {"workload": name, "steps": steps}
    for key, call in (("sigmoid", lambda: sa.sigattn_fwd(qd, kd, vd, o, lens, ws, stream)),
                      ("softmax", lambda: sa.sigattn_softmax_fwd(qd, kd, vd, o, lens, ws, stream))):
        for _ in range(warmup):
            call()
            flush_buf.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps)]
        torch.cuda.synchronize(dev)
        for i in range(steps):
            ev[2 * i].record(stream)
            call()
            ev[2 * i + 1].record(stream)
            flush_buf.zero_()
        torch.cuda.synchronize(dev)
        _check_status(sa, ws, stream)
        ms = float(np.mean([ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(steps)]))
        out[f"{key}_fwd_ms"] = ms
        out[f"{key}_fwd_tflops"] = w.fwd_flops() / (ms / 1e3) / 1e12
    out["sigmoid_over_softmax"] = out["sigmoid_fwd_tflops"] / out["softmax_fwd_tflops"]
    return out


def unfused_torch(w, q, k, v, dout, lengths, dev, steps: int = 5, warmup: int = 3) -> dict:
    """The comparison of "Better Models, Faster Training" sec. 4A: sigmoid
    attention written as plain PyTorch operations (bf16 matmuls, an explicit
    score tensor, sigmoid, mask, matmul; backward by autograd) on the same
    inputs, timed the same way, with the same valid-pair FLOP count. It is a
    baseline for the speed-up figures, not part of the library."""
    import math as _m

    import torch

    B, H, L, d = q.shape
    qd, kd, vd, dod = (t.to(dev).requires_grad_(i < 3) for i, t in enumerate((q, k, v, dout)))
    n = lengths.to(dev).to(torch.float32)
    bias = (-torch.log(n.clamp_min(1))).view(B, 1, 1, 1).to(torch.bfloat16)
    idx = torch.arange(L, device=dev)
    valid = idx.view(1, L) < lengths.to(dev).view(B, 1)
    mask = (valid.view(B, 1, L, 1) & valid.view(B, 1, 1, L))

    def fwd():
        s_ = torch.matmul(qd, kd.transpose(-1, -2)) * (1.0 / _m.sqrt(d)) + bias
        p_ = torch.where(mask, torch.sigmoid(s_), torch.zeros((), dtype=s_.dtype, device=dev))
        return torch.matmul(p_, vd)

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    fwd_ms, bwd_ms = [], []
    for i in range(warmup + steps):
        for t in (qd, kd, vd):
            t.grad = None
        ev[0].record()
        out = fwd()
        ev[1].record()
        out.backward(dod)
        ev[2].record()
        torch.cuda.synchronize(dev)
        if i >= warmup:
            fwd_ms.append(ev[0].elapsed_time(ev[1]))
            bwd_ms.append(ev[1].elapsed_time(ev[2]))
    f_fwd, f_bwd = w.fwd_flops(), w.bwd_flops()
    res = {"fwd_ms": float(np.mean(fwd_ms)), "bwd_ms": float(np.mean(bwd_ms)),
           "fwd_tflops": f_fwd / (np.mean(fwd_ms) / 1e3) / 1e12, "bwd_tflops": f_bwd / (np.mean(bwd_ms) / 1e3) / 1e12,
           "steps": steps, "what": "torch.matmul (bf16) -> scale + bias -> sigmoid -> mask -> torch.matmul; "
                                   "backward by autograd"}
    del qd, kd, vd, dod, out
    torch.cuda.empty_cache()
    return res


def pcie_bandwidth(dev, nbytes: int = 256 << 20, reps: int = 6) -> dict:
    """Pinned host <-> device copy bandwidth in GB/s: each direction alone, and
    per direction with both running at once (the bound of a pipelined step)."""
    import torch

    h_up, h_down = (torch.empty(nbytes, dtype=torch.uint8).pin_memory() for _ in range(2))
    d_up, d_down = (torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(2))
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def timed(up: bool, down: bool) -> float:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(s_up)
        s_down.wait_event(e0)
        for _ in range(reps):
            if up:
                with torch.cuda.stream(s_up):
                    d_up.copy_(h_up, non_blocking=True)
            if down:
                with torch.cuda.stream(s_down):
                    h_down.copy_(d_down, non_blocking=True)
        s_up.wait_stream(s_down)
        e1.record(s_up)
        torch.cuda.synchronize(dev)
        return reps * nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9

    timed(True, True)  # warm-up
    out = {"h2d": timed(True, False), "d2h": timed(False, True), "both_per_direction": timed(True, True)}
    del h_up, h_down, d_up, d_down
    return out


def run_gpu(args, w):
    import torch

    import sigmoid_attention_b200 as sa
    from sigmoid_attention_b200 import workloads

    world, rank, local = _dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    q, k, v, dout, lengths = workloads.workload_inputs(w)
    flops_fwd = w.fwd_flops()
    flops_bwd = w.bwd_flops()
    pairs = flops_fwd / (4.0 * w.d)
    packed = args.layout == "packed"
    if packed:
        # Valid tokens only, back to back: [total, H, d] and cu_seqlens [B + 1].
        q, k, v, dout = (torch.cat([t[b, :, :int(n)].permute(1, 0, 2) for b, n in enumerate(lengths.tolist())])
                         .contiguous() for t in (q, k, v, dout))
        lengths = torch.cat([torch.zeros(1, dtype=torch.int32), torch.cumsum(lengths, 0).to(torch.int32)])
        max_seqlen = max(1, int(w.lengths().max()))
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    lens = lengths.to(dev)
    o, dq, dk, dv = (torch.empty_like(qd) for _ in range(4))
    ws = sa.make_workspace(w.B, w.H, max_seqlen if packed else w.L, w.d, dev)
    stream = torch.cuda.current_stream(dev)
    tensor_bytes = qd.numel() * 2
    footprint = 8 * tensor_bytes
    flush = footprint < 4 * L2_BYTES
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if flush else None

    if packed:
        calls = (lambda: sa.sigattn_fwd_varlen(qd, kd, vd, o, lens, max_seqlen, ws, stream),
                 lambda: sa.sigattn_bwd_dq_varlen(qd, kd, vd, dod, dq, lens, max_seqlen, ws, stream),
                 lambda: sa.sigattn_bwd_dkdv_varlen(qd, kd, vd, dod, dk, dv, lens, max_seqlen, ws, stream))
    else:
        calls = (lambda: sa.sigattn_fwd(qd, kd, vd, o, lens, ws, stream),
                 lambda: sa.sigattn_bwd_dq(qd, kd, vd, dod, dq, lens, ws, stream),
                 lambda: sa.sigattn_bwd_dkdv(qd, kd, vd, dod, dk, dv, lens, ws, stream))

    def step(ev=None):
        _run_calls(calls, stream, ev)

    sync_ranks = (lambda: torch.distributed.barrier()) if world > 1 else None
    clocks = ClockSampler(local)
    per_kernel, step_ms = _device_steps(calls, stream, args.steps, args.warmup, scratch, sync_ranks,
                                        lambda: _check_status(sa, ws, stream), clocks)
    step_fused = None
    if not packed:
        fused_calls = (calls[0], lambda: sa.sigattn_bwd(qd, kd, vd, dod, dq, dk, dv, lens, ws, stream))
        step_fused = _fused_backward(per_kernel, fused_calls, stream, args.steps, args.warmup, scratch,
                                     lambda: _check_status(sa, ws, stream), flops_fwd, flops_bwd)
        if world > 1:  # whole-job figures: the slowest rank's time
            for key in ("value", "bwd_tflops"):
                step_fused[key] = world / reduce_max(world / step_fused[key], world, dev)
            step_fused.pop("bwd_speedup_vs_two_calls")
    total_s = reduce_max(sum(step_ms) / 1e3, world, dev)
    fwd_s = reduce_max(sum(per_kernel["fwd"]) / 1e3, world, dev)
    bwd_s = reduce_max((sum(per_kernel["bwd_dq"]) + sum(per_kernel["bwd_dkdv"])) / 1e3, world, dev)
    value = whole_job_tflops((flops_fwd + flops_bwd) * args.steps, world, total_s)
    fwd_tflops = whole_job_tflops(flops_fwd * args.steps, world, fwd_s)
    bwd_tflops = whole_job_tflops(flops_bwd * args.steps, world, bwd_s)

    # --- end to end through the public API with host buffers -------------
    pin = [t.pin_memory() for t in (q, k, v, dout)]
    lens_h = lengths.pin_memory()
    outs_h = [torch.empty_like(q).pin_memory() for _ in range(4)]
    h2d = sum(t.numel() * t.element_size() for t in pin) + lens_h.numel() * 4
    d2h = sum(t.numel() * t.element_size() for t in outs_h)
    e2e_steps = max(1, min(args.steps, 20))
    dev_in, dev_out = (qd, kd, vd, dod), (o, dq, dk, dv)

    def e2e_step():
        for src, dst in zip(pin, dev_in):
            dst.copy_(src, non_blocking=True)
        lens.copy_(lens_h, non_blocking=True)
        step()
        for src, dst in zip(dev_out, outs_h):
            dst.copy_(src, non_blocking=True)

    # Pipelined schedule: the batch in chunks of whole sequences. Chunk c's inputs
    # go up on one stream, its three calls run on the compute stream and its
    # outputs come back on a third, so the copies in both directions overlap the
    # compute of other chunks (and of the neighbouring steps). Events order each
    # chunk's copy -> calls -> copy back, and keep a step's copies off buffers
    # that the previous step still uses.
    nch = min(w.B, 8)
    bounds = [round(i * w.B / nch) for i in range(nch + 1)]
    chunks = [(b0, b1) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
    if packed:
        rows = [(int(lengths[b0]), int(lengths[b1])) for b0, b1 in chunks]
        cu_h = [(lengths[b0:b1 + 1] - lengths[b0]).to(torch.int32).pin_memory() for b0, b1 in chunks]
        cu_d = [torch.empty_like(c, device=dev) for c in cu_h]
    else:
        rows = chunks
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in rows]
    computed = [torch.cuda.Event() for _ in rows]
    out_back = [torch.cuda.Event() for _ in rows]

    def e2e_step_pipelined():
        for c, (r0, r1) in enumerate(rows):
            with torch.cuda.stream(s_in):
                s_in.wait_event(computed[c])  # the previous step's calls have read these inputs
                for src, dst in zip(pin, dev_in):
                    dst[r0:r1].copy_(src[r0:r1], non_blocking=True)
                if packed:
                    cu_d[c].copy_(cu_h[c], non_blocking=True)
                else:
                    lens[r0:r1].copy_(lens_h[r0:r1], non_blocking=True)
                in_ready[c].record(s_in)
            stream.wait_event(in_ready[c])
            stream.wait_event(out_back[c])  # the previous step's outputs of this chunk are on the host
            qc, kc, vc, dc = (t[r0:r1] for t in dev_in)
            oc, dqc, dkc, dvc = (t[r0:r1] for t in dev_out)
            if packed:
                sa.sigattn_fwd_varlen(qc, kc, vc, oc, cu_d[c], max_seqlen, ws, stream)
                sa.sigattn_bwd_varlen(qc, kc, vc, dc, dqc, dkc, dvc, cu_d[c], max_seqlen, ws, stream)
            else:
                lc = lens[r0:r1]
                sa.sigattn_fwd(qc, kc, vc, oc, lc, ws, stream)
                sa.sigattn_bwd(qc, kc, vc, dc, dqc, dkc, dvc, lc, ws, stream)
            computed[c].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[c])
                for src, dst in zip(dev_out, outs_h):
                    dst[r0:r1].copy_(src[r0:r1], non_blocking=True)
                out_back[c].record(s_out)

    def time_e2e(fn, first_stream, last_stream):
        fn()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(first_stream)
        for _ in range(e2e_steps):
            fn()
        last_stream.wait_stream(stream)
        last_stream.wait_stream(s_in)
        e1.record(last_stream)
        torch.cuda.synchronize(dev)
        sec = reduce_max(e0.elapsed_time(e1) / 1e3, world, dev)
        return whole_job_tflops((flops_fwd + flops_bwd) * e2e_steps, world, sec)

    e2e_serial = time_e2e(e2e_step, stream, stream)
    stream.wait_stream(s_in)
    s_in.wait_stream(stream)
    e2e_value = time_e2e(e2e_step_pipelined, s_in, s_out)
    torch.cuda.synchronize(dev)
    # Bound of the pipelined step: its larger copy direction at the measured
    # both-directions-at-once PCIe rate, with the compute fully hidden.
    pcie = pcie_bandwidth(dev)
    e2e_bound = world * (flops_fwd + flops_bwd) / (max(h2d, d2h) / (pcie["both_per_direction"] * 1e9)) / 1e12
    # The pipelined copies must bring back exactly what the calls wrote.
    for host, devt in zip(outs_h, dev_out):
        if not torch.equal(host, devt.cpu()):
            raise SystemExit("pipelined end-to-end outputs differ from the device results")
    st, site = sa.sigattn_read_error(ws, stream)
    if st != 0:
        raise SystemExit(f"kernel reported status {st} at site {site}")

    peaks = _peaks()
    peak = peaks["bf16_tflops"]
    avg_ms = {kname: float(np.mean(v_)) for kname, v_ in per_kernel.items()}
    dominant = max(avg_ms, key=avg_ms.get)
    dom_flops = KERNEL_FLOPS_PER_PAIR[dominant] * w.d * pairs
    achieved = dom_flops / (avg_ms[dominant] / 1e3) / 1e12
    kernels = {kname: {"ms": avg_ms[kname],
                       "tflops": KERNEL_FLOPS_PER_PAIR[kname] * w.d * pairs / (avg_ms[kname] / 1e3) / 1e12,
                       "flops_per_valid_pair": f"{KERNEL_FLOPS_PER_PAIR[kname]}*d"} for kname in avg_ms}
    clk = clocks.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_s * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**w.describe(), "layout": args.layout, "valid_pairs_per_head": pairs / w.H,
                   "step": ("sigattn_fwd_varlen + sigattn_bwd_dq_varlen + sigattn_bwd_dkdv_varlen "
                            "(each: plan + compute kernel)") if packed else
                           ("sigattn_fwd + sigattn_bwd_dq + sigattn_bwd_dkdv "
                            "(each: plan + compute kernel; zero-fill kernel beside the forward)"),
                   "flops": "valid pairs only: 4*d fwd + 10*d bwd per pair",
                   "parallelism": f"replica per GPU x{world} (independent batches)",
                   "l2": ("flushed between steps (footprint %.0f MB)" % (footprint / 1e6)) if flush else
                         ("no flush: inputs+outputs %.0f MB > 126 MB L2" % (footprint / 1e6))},
        "fwd_tflops": fwd_tflops, "bwd_tflops": bwd_tflops,
        "fwd_frac_of_peak": fwd_tflops / peak, "bwd_frac_of_peak": bwd_tflops / peak,
        "frac_of_spec_2250": {"fwd": fwd_tflops / 2250.0, "bwd": bwd_tflops / 2250.0},
        "kernels": kernels,
        "step_fused": step_fused,
        "roofline": {"bound": "tensor", "kernel": dominant, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_source": f"bf16_tflops ({peaks['source']}, burst)",
                     "traffic": _traffic(dominant, w.name)},
        "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "schedule": f"{len(rows)} chunks of whole sequences; host-to-device copies, the calls "
                            f"({'sigattn_fwd_varlen + sigattn_bwd_varlen' if packed else 'sigattn_fwd + sigattn_bwd'}) and "
                            "device-to-host copies on three streams",
                "pcie_gbs": pcie, "bound": e2e_bound, "frac_of_bound": e2e_value / e2e_bound,
                "bound_source": "larger copy direction per step at the measured both-ways pinned copy rate"},
        "e2e_serial": {"value": e2e_serial, "unit": "TFLOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "steps": e2e_steps, "schedule": "copy in, three calls, copy out, one stream"},
        # Device-timed steps only: per call the plan and compute kernels, plus (padded
        # layout) the zero-fill kernel beside the forward kernel.
        "gpu_launches": (6 if packed else 7) * args.steps,
        "clocks": clk,
    }
    if world == 1 and not args.no_extras:
        # Same run, same box: the padding ratio and the short-sequence workloads
        # (device-timed), and the unfused PyTorch comparison on this workload.
        side = [n_ for n_ in ("pad_sweep_p00", "pad_sweep_p75", "scrna_ragged", "long_8k") if n_ != w.name]
        line["other_workloads"] = side_workloads(side, dev, steps=10, warmup=3)
        line["softmax_counterpart"] = softmax_comparison("pad_sweep_p25", dev)
        if w.name in ("pad_sweep_p00", "pad_sweep_p75"):
            mine = {"value": value, "fwd_tflops": fwd_tflops, "bwd_tflops": bwd_tflops}
            other = line["other_workloads"].get("pad_sweep_p75" if w.name == "pad_sweep_p00" else "pad_sweep_p00")
            p00, p75 = (mine, other) if w.name == "pad_sweep_p00" else (other, mine)
            line["other_workloads"]["p75_over_p00"] = p75["value"] / p00["value"]
        if not packed:
            u = unfused_torch(w, q, k, v, dout, lengths, dev)
            u["fused_speedup"] = {"fwd": fwd_tflops / u["fwd_tflops"], "bwd": bwd_tflops / u["bwd_tflops"]}
            line["unfused_torch"] = u
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def spawn_ranks(n: int, argv: list, timeout_s: float = 3600.0) -> int:
    """Run this script as n ranks (one process per GPU) under
    torch.distributed.run on this node, rendezvous on 127.0.0.1, and return
    the launcher's exit code. The launcher and its ranks form one process
    group, which is ended as a whole if it outlives `timeout_s`."""
    import signal
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE")}
    proc = subprocess.Popen(cmd, env=env, start_new_session=True)
    try:
        return proc.wait(timeout=timeout_s)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGTERM)
        try:
            proc.wait(timeout=60)
        except subprocess.TimeoutExpired:
            os.killpg(proc.pid, signal.SIGKILL)
            proc.wait()
        print(f"bench.py: {n}-rank run exceeded {timeout_s:.0f} s", file=sys.stderr)
        return 1


def main(argv=None):
    from sigmoid_attention_b200 import workloads

    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="dense_d128", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--layout", default="padded", choices=["padded", "packed"],
                    help="padded [B,H,Lmax,d] tensors, or the workload's valid tokens packed as [total,H,d]")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads and the unfused PyTorch comparison (1-GPU runs only)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = workloads.WORKLOADS[args.workload]
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # Not started by a launcher: start one process per GPU ourselves.
        return spawn_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv))
    world, _, _ = _dist_env()
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but the launcher started WORLD_SIZE={world} ranks")
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
