#!/usr/bin/env python
"""Benchmark of the Naju scan hot path (fwd + bwd) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one forward (fused conv + scan + readout + SiLU(z) modulation) and
one backward over one batch of the workload's synthetic inputs, all resident
in HBM.  With the decode workload (`--workload throughput_decode`) one step is
one decode token for the whole batch (conv state + scan state updated in
place).  Prints one JSON line (rank 0).  Under torchrun each rank runs its own
replica of the workload (batch elements are independent; weak scaling, no
collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from discrete_selective_ssm_b200.parallel import max_over_ranks  # noqa: E402
from discrete_selective_ssm_b200.workloads import (WORKLOADS, decode_D, decode_state0,  # noqa: E402
                                                   decode_step_inputs, make_inputs, scaled)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def alg_bytes(w, E):
    """Algorithmic HBM bytes of one fwd and one bwd over workload w with
    activation element size E (inputs read once, outputs written once)."""
    T = w.batch * w.seqlen
    d, N = w.d_inner, w.d_state
    fwd = T * (5 * E * d + 2 * E * N) + w.batch * d * N * 4
    bwd = T * (9 * E * d + 4 * E * N) + w.batch * d * N * 4
    return fwd, bwd


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_oracle_step(w, t, n_batch=1):
    """One fwd + bwd of the fp64 oracle over the first n_batch batch elements
    of the workload.  Returns (seconds, tokens, threads)."""
    import oracle
    sl = {k: (v[:n_batch] if k in ("u", "a", "b", "B", "C", "z", "dout") else v)
          for k, v in t.items()}
    t0 = time.perf_counter()
    oracle.block_fwd(sl["u"], sl["conv_w"], sl["conv_b"], sl["a"], sl["b"], sl["B"], sl["C"],
                     sl["z"], sl["D"])
    oracle.block_bwd(sl["u"], sl["conv_w"], sl["conv_b"], sl["a"], sl["b"], sl["B"], sl["C"],
                     sl["z"], sl["D"], None, sl["dout"])
    return time.perf_counter() - t0, n_batch * w.seqlen, oracle.num_threads()


def cpu_sample_workload(w):
    """Bounded CPU sample: one batch element, the sequence cut to keep the
    oracle's fwd+bwd around 10-20 s on a few host cores."""
    per_tok = w.d_inner * w.d_state  # state updates per token
    L = max(64, min(w.seqlen, int(6e8 / per_tok)))
    return scaled(w, batch=1, seqlen=L)


def run_reference(args, w, rank, world):
    """The oracle as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    ws = cpu_sample_workload(w)
    t = make_inputs(ws, which=("u", "a", "b", "B", "C", "z", "D", "conv_w", "conv_b", "dout"))
    for _ in range(max(0, min(args.warmup, 1))):
        cpu_oracle_step(ws, t)
    times = []
    for _ in range(args.steps):
        dt, toks, thr = cpu_oracle_step(ws, t)
        times.append(dt)
    ms = 1e3 * statistics.mean(times)
    val = ws.batch * ws.seqlen / (ms / 1e3)
    sample = (f"oracle fwd+bwd on batch 1 x L={ws.seqlen} x d_inner={ws.d_inner} x "
              f"d_state={ws.d_state} (slice of {w.name})")
    print(json.dumps({
        "metric": "naju_scan_fwd_bwd_tokens_per_s", "value": val, "unit": "tokens/s",
        "impl": "reference", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                   "d_inner": w.d_inner, "d_state": w.d_state, "dtype_inputs": w.dtype},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def decode_bytes(w, E):
    """Algorithmic HBM bytes of one decode token for the whole batch: inputs
    u, a, b, z and output y (5 E d), B, C (2 E N), fp32 state read + write
    (2 d N 4) and conv state read + write (2 d 3 4), per batch element."""
    d, N = w.d_inner, w.d_state
    return w.batch * (5 * E * d + 2 * E * N + 2 * d * N * 4 + 2 * d * 3 * 4)


def decode_cpu_sample(w, n_batch=8):
    import oracle
    st = decode_state0(w)[:n_batch].double().numpy()
    cs = np.zeros((n_batch, w.d_inner, 3))
    conv = make_inputs(w, which=("conv_w", "conv_b"))
    D = decode_D(w)
    dt, toks, k = 0.0, 0, 0
    while dt < 10.0 and k < w.decode_steps:
        s_in = decode_step_inputs(w, k)
        sl = {kk: v[:n_batch] for kk, v in s_in.items()}
        t0 = time.perf_counter()
        _, st, cs = oracle.block_step(st, cs, sl["h"], conv["conv_w"], conv["conv_b"], sl["a"],
                                      sl["b"], sl["B"], sl["C"], sl["z"], D)
        dt += time.perf_counter() - t0
        toks += n_batch
        k += 1
    return toks / dt, oracle.num_threads(), f"oracle decode steps, {k} x batch {n_batch} slice of {w.name}, {dt:.1f} s"


def run_reference_decode(args, w, rank):
    if rank != 0:
        return
    val, thr, sample = decode_cpu_sample(w)
    print(json.dumps({
        "metric": "naju_decode_step_tokens_per_s", "value": val, "unit": "tokens/s",
        "impl": "reference", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "d_inner": w.d_inner,
                   "d_state": w.d_state, "conv_state": True},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_decode(args, w, rank, world, local):
    """Decode-step bench: one step = one token (conv + scan step) for the batch."""
    import discrete_selective_ssm_b200 as naju
    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # A pool of distinct per-token inputs (larger than L2 together), cycled.
    pool = 64
    host = [decode_step_inputs(w, k) for k in range(pool)]
    inp = {k: torch.stack([h[k] for h in host]).to(dev) for k in host[0]}
    state = decode_state0(w).to(dev)
    cs = torch.zeros(w.batch, w.d_inner, 3, device=dev)
    conv = {k: v.to(dev) for k, v in make_inputs(w, which=("conv_w", "conv_b")).items()}
    D = decode_D(w).to(dev)
    y = torch.empty((w.batch, w.d_inner), dtype=w.torch_dtype, device=dev)
    stream = torch.cuda.current_stream()

    def step(k, src=None):
        src = src if src is not None else {kk: v[k % pool] for kk, v in inp.items()}
        naju.scan_step_conv(state, cs, src["h"], src["a"], src["b"], src["B"], src["C"],
                            conv["conv_w"], conv["conv_b"], src["z"], D, y=y)

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    # The K timed steps are captured once in a CUDA graph and replayed: one
    # launch per step from Python leaves the GPU waiting on the host between
    # steps (a step is ~50 us of device work).  The first replay uploads the
    # graph and is not timed.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for k in range(args.steps):
            step(args.warmup + k)
    graph.replay()
    torch.cuda.synchronize()
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = clk.stop()
    ms_total = e0.elapsed_time(e1)
    if dist is not None:
        ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps
    value = world * w.batch / (ms_step / 1e3)

    # e2e: the token's inputs H2D from pinned memory, y D2H, every step.
    pinned = {k: v.pin_memory() for k, v in host[0].items()}
    dev_in = {k: torch.empty_like(v[0]) for k, v in inp.items()}
    y_host = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y.numel() * y.element_size()

    def e2e_step(k):
        for kk, v in pinned.items():
            dev_in[kk].copy_(v, non_blocking=True)
        step(k, dev_in)
        y_host.copy_(y, non_blocking=True)

    e2e_step(0)
    torch.cuda.synchronize()
    s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for k in range(args.steps):
        e2e_step(k)
    t2.record(stream)
    torch.cuda.synchronize()
    e2e_ms = s2.elapsed_time(t2) / args.steps
    if dist is not None:
        e2e_ms = max_over_ranks(e2e_ms, dev)

    pk, pk_kind = peaks()
    E = 2 if w.dtype == "bf16" else 4
    nb = decode_bytes(w, E)
    achieved = nb / (ms_step / 1e3) / 1e9
    peak = float(pk["hbm_gbs"])
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, thr, sample = decode_cpu_sample(w)
        cpu = {"value": val, "unit": "tokens/s", "cores": thr, "kind": "oracle",
               "sample": sample}
    if rank == 0:
        print(json.dumps({
            "metric": "naju_decode_step_tokens_per_s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "d_inner": w.d_inner,
                       "d_state": w.d_state, "conv_state": True, "gating": True,
                       "parallelism": f"replicas{world}", "cuda_graph": True,
                       "l2": "state (134 MB) and input pool larger than L2 (no flush)"},
            "roofline": {"bound": "hbm", "kernel": "naju_scan_step_conv: step_kernel",
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "alg_bytes": nb,
                         "peak_kind": pk_kind},
            "cpu_baseline": cpu,
            "e2e": {"value": world * w.batch / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clocks,
        }), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_block(args, w, rank, world, local):
    """Full-block bench: one step = block forward + backward over the batch."""
    from discrete_selective_ssm_b200.block import NajuBlock
    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dm = w.d_inner // 2
    blk = NajuBlock(dm, w.d_inner, w.d_state, dev, dtype=w.torch_dtype, seed=1,
                    coupled=args.coupled)
    gen = torch.Generator().manual_seed(2)
    x = torch.randn(w.batch, w.seqlen, dm, generator=gen).to(dev, w.torch_dtype)
    dout = torch.randn(w.batch, w.seqlen, dm, generator=gen).to(dev, w.torch_dtype)
    stream = torch.cuda.current_stream()

    def step():
        out, ctx = blk.forward(x)
        blk.backward(ctx, dout)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = clk.stop()
    ms = e0.elapsed_time(e1) / args.steps
    if dist is not None:
        ms = max_over_ranks(ms, dev)
    di, N = w.d_inner, w.d_state
    gemm_flop = 2 * w.batch * w.seqlen * (dm * 2 * di + 2 * di * di + 2 * di * N + di * dm) * 3
    if rank == 0:
        print(json.dumps({
            "metric": "naju_block_fwd_bwd_tokens_per_s", "value": world * w.batch * w.seqlen /
            (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name + "_block", "batch": w.batch, "seqlen": w.seqlen,
                       "d_model": dm, "d_inner": di, "d_state": N, "coupled": args.coupled,
                       "gemm_tflop_per_step": gemm_flop / 1e12,
                       "parallelism": f"replicas{world}"},
            "roofline": None, "cpu_baseline": None, "e2e": None,
            "gpu_launches": None, "clocks": clocks,
        }), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="throughput_train", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--block", action="store_true",
                    help="time the full Naju block (norm, projections, conv, scan, residual) "
                         "with d_model = d_inner / 2 instead of the scan alone")
    ap.add_argument("--coupled", action="store_true",
                    help="coupled single gate i = 1 - f (no b input)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (a smaller case of the same kernels, "
                         "for profiling; the JSON line's config shows the sizes)")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="override the workload's sequence length (as --batch)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]
    if args.batch or args.seqlen:
        w = scaled(w, batch=args.batch or w.batch, seqlen=args.seqlen or w.seqlen)
    if w.decode_steps:
        if args.impl == "reference":
            run_reference_decode(args, w, rank)
        else:
            run_decode(args, w, rank, world, local)
        return

    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if args.block:
        run_block(args, w, rank, world, local)
        return

    import discrete_selective_ssm_b200 as naju

    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    t_host = make_inputs(w, which=("u", "a", "b", "B", "C", "z", "D", "conv_w", "conv_b", "dout"))
    t = {k: v.to(dev) for k, v in t_host.items()}
    E = 2 if w.dtype == "bf16" else 4
    out_dt = naju.BF16 if w.dtype == "bf16" else naju.F32
    dims = naju.make_dims(w.batch, w.seqlen, w.d_inner, w.d_state,
                          naju.BF16 if w.dtype == "bf16" else naju.F32, out_dt)
    ws = naju.alloc_workspace(dims, dev)
    y = torch.empty((w.batch, w.seqlen, w.d_inner), dtype=w.torch_dtype, device=dev)
    ot = w.torch_dtype
    shp = (w.batch, w.seqlen, w.d_inner)
    grads = {"dhu": torch.empty(shp, dtype=ot, device=dev),
             "da": torch.empty(shp, dtype=ot, device=dev),
             "db": torch.empty(shp, dtype=ot, device=dev),
             "dz": torch.empty(shp, dtype=ot, device=dev),
             "dB": torch.empty((w.batch, w.seqlen, w.d_state), dtype=ot, device=dev),
             "dC": torch.empty((w.batch, w.seqlen, w.d_state), dtype=ot, device=dev),
             "dD": torch.empty(w.d_inner, dtype=torch.float32, device=dev),
             "dconv_w": torch.empty_like(t["conv_w"]),
             "dconv_b": torch.empty(w.d_inner, dtype=torch.float32, device=dev),
             "dx0": None}
    stream = torch.cuda.current_stream()

    def step(inp, ev=None, y_out=None, g_out=None):
        y_out = y if y_out is None else y_out
        g_out = grads if g_out is None else g_out
        if ev is not None:
            ev[0].record(stream)
        naju.scan_fwd(inp["u"], inp["a"], None if args.coupled else inp["b"], inp["B"], inp["C"],
                      conv_w=inp["conv_w"],
                      conv_b=inp["conv_b"], z=inp["z"], D=inp["D"], out_dtype=out_dt,
                      workspace=ws, want_final=False, y=y_out)
        if ev is not None:
            ev[1].record(stream)
        naju.scan_bwd(inp["dout"], inp["u"], inp["a"], None if args.coupled else inp["b"],
                      inp["B"], inp["C"], ws,
                      conv_w=inp["conv_w"], conv_b=inp["conv_b"], z=inp["z"], D=inp["D"],
                      out_dtype=out_dt, grads=g_out)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step(t)
    torch.cuda.synchronize()
    if naju.last_device_status(ws) != 0:
        raise SystemExit("device status not OK after warm-up")

    # Kernels of one step: the forward kernel; the backward kernel, the dB/dC
    # and channel reductions, and the conv fixup across sequence-group edges or
    # piece-mode cuts when the backward splits the sequence.
    launches_per_step = 1 + 3 + (1 if naju.testing_bwd_groups(dims) > 1 else 0)

    # ---------------------------------------------------------- timed region
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(t, evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = clk.stop()
    ms_total = start.elapsed_time(end)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    if naju.last_device_status(ws) != 0:
        raise SystemExit("device status not OK after the timed region")
    if dist is not None:
        ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps
    tokens = w.batch * w.seqlen
    value = world * tokens / (ms_step / 1e3)

    # -------------------------------------------------------------- e2e leg
    # Every step copies its inputs host -> device (pinned) and all its outputs
    # device -> host inside the timed region.  Copies run on their own streams
    # with double-buffered device inputs and outputs, so step i's compute
    # overlaps step i+1's upload and step i-1's download (separate copy
    # engines); the timed region spans the first upload to the last download.
    pinned = {k: v.pin_memory() for k, v in t_host.items()}
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    dev_in = [{k: torch.empty_like(v) for k, v in t.items()} for _ in range(2)]
    y2 = [y, torch.empty_like(y)]
    g2 = [grads, {k: (torch.empty_like(v) if v is not None else None) for k, v in grads.items()}]
    outs2 = [[y2[i]] + [v for v in g2[i].values() if v is not None] for i in range(2)]
    host_outs = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs2[i]]
                 for i in range(2)]
    d2h = sum(o.numel() * o.element_size() for o in outs2[0])
    s_up, s_down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    n_e2e = max(args.e2e_steps, 1)

    def e2e_run(n):
        up_done = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        down_done = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_up)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(comp_done[i - 2])  # inputs buffer b free again
                for k, v in pinned.items():
                    dev_in[b][k].copy_(v, non_blocking=True)
                up_done[i].record(s_up)
            stream.wait_event(up_done[i])
            if i >= 2:
                stream.wait_event(down_done[i - 2])  # outputs buffer b copied out
            step(dev_in[b], y_out=y2[b], g_out=g2[b])
            comp_done[i].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(comp_done[i])
                for ho, o in zip(host_outs[b], outs2[b]):
                    ho.copy_(o, non_blocking=True)
                down_done[i].record(s_down)
        stream.wait_event(down_done[n - 1])
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n

    e2e_run(2)
    if dist is not None:
        dist.barrier()
    e2e_ms = e2e_run(n_e2e)
    if dist is not None:
        e2e_ms = max_over_ranks(e2e_ms, dev)
    e2e_val = world * tokens / (e2e_ms / 1e3)

    # ---------------------------------------------------------------- roofline
    pk, pk_kind = peaks()
    fwd_b, bwd_b = alg_bytes(w, E)
    dom_is_bwd = bwd_ms >= fwd_ms
    dom_ms = bwd_ms if dom_is_bwd else fwd_ms
    dom_b = bwd_b if dom_is_bwd else fwd_b
    achieved = dom_b / (dom_ms / 1e3) / 1e9
    peak = float(pk["hbm_gbs"])
    traffic = None  # measured for the named workload as benched by default only
    prof = os.path.join(ROOT, "profiles", f"traffic_{w.name}.json")
    if not (args.batch or args.seqlen or args.coupled) and os.path.exists(prof):
        with open(prof) as fh:
            tr = json.load(fh)
        traffic = tr.get("bwd" if dom_is_bwd else "fwd")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ws_cpu = cpu_sample_workload(w)
        tc = make_inputs(ws_cpu, which=("u", "a", "b", "B", "C", "z", "D", "conv_w", "conv_b",
                                        "dout"))
        dt_sum, toks_sum, reps = 0.0, 0, 0
        while dt_sum < 10.0 and reps < 64:  # about 10 s of host work
            dt, toks, thr = cpu_oracle_step(ws_cpu, tc)
            dt_sum += dt
            toks_sum += toks
            reps += 1
        cpu = {"value": toks_sum / dt_sum, "unit": "tokens/s", "cores": thr, "kind": "oracle",
               "sample": f"oracle fwd+bwd, {reps} x (batch 1 x L={ws_cpu.seqlen}) slice of "
                         f"{w.name}, {dt_sum:.1f} s"}

    if rank == 0:
        print(json.dumps({
            "metric": "naju_scan_fwd_bwd_tokens_per_s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                       "d_inner": w.d_inner, "d_state": w.d_state, "conv_width": 4,
                       "fused_conv": True, "gating": True, "coupled_gate": args.coupled,
                       "parallelism": f"replicas{world}",
                       "l2": "inputs larger than L2 (no flush)",
                       "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
                       "fwd_gbs": fwd_b / (fwd_ms / 1e3) / 1e9,
                       "bwd_gbs": bwd_b / (bwd_ms / 1e3) / 1e9,
                       "fwd_frac_hbm": fwd_b / (fwd_ms / 1e3) / 1e9 / peak,
                       "bwd_frac_hbm": bwd_b / (bwd_ms / 1e3) / 1e9 / peak},
            "roofline": {"bound": "hbm",
                         "kernel": ("naju_scan_bwd: scan_bwd_blk_kernel + finish_dBC + reductions"
                                    if dom_is_bwd else "naju_scan_fwd: scan_fwd_blk_kernel"),
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "alg_bytes": dom_b, "peak_kind": pk_kind},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
