#!/usr/bin/env python
"""Throughput of the PRISM sequence-mixer scan forward on B200.

One step = one prism_scan_fwd call (ShortConv anchor, residual chain, rank-(L-1)
residual write, gated-delta chunk scan, readout) over one batch of synthetic
inputs already resident in HBM.  Default workload: one 130M-LM-shaped layer
(B=16, T=2048, H=6, d_k=d_v=128, L=4, chunk=64, ShortConv width 4, bf16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

N > 1 runs under torchrun, one process per GPU; every rank scans its own batch
(independent replicas sharded by batch, no collective on the data path:
weak scaling).  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the slow, obviously correct
definition) on the host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "PRISM scan fwd tokens/s on 1 B200; achieved fraction of TC/HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "chunk_scan": "linear_attention_sequence_shortconv_b200/csrc/chunk_scan_kernel.cu",
    "prism_scan_kernel": "linear_attention_sequence_shortconv_b200/csrc/chunk_scan_kernel.cu",
    "residual_write_kernel": "linear_attention_sequence_shortconv_b200/csrc/chunk_scan_kernel.cu",
    "recurrent": "linear_attention_sequence_shortconv_b200/csrc/recurrent_kernel.cu",
}


# ---------------------------------------------------------------- workload arithmetic
def algorithmic_work(w, lengths=None):
    """Algorithmic bytes and FLOPs of one scan over workload ``w``.

    Per token-head: bytes = q,k,v,o (4 d elements) + u, gain (2 m d elements) in the
    I/O dtype, plus gamma, beta (fp32) and alpha (m fp32); per sequence-head the
    final state (d_v d_k fp32) and S0 if given.  FLOPs (chunk form, dense C x C
    blocks): 10 C d + 8 C m d + 6 d^2 + 2 m d^2 per token-head (d = d_k = d_v).
    Only valid tokens count for right-padded batches.
    """
    es = 2 if w.dtype == "bf16" else 4
    d, m, C = w.d_k, w.m, w.chunk
    valid_tokens = int(lengths.sum()) if lengths is not None else w.B * w.T
    token_heads = valid_tokens * w.H
    per_th = es * (2 * w.d_k + 2 * w.d_v) + es * m * (w.d_k + w.d_v) + 4 * (2 + m)
    state = w.B * w.H * w.d_v * w.d_k * 4 * (2 if w.with_s0 else 1)
    flops_th = 10 * C * d + 8 * C * m * d + 6 * d * d + 2 * m * d * d
    return {"tokens": valid_tokens, "token_heads": token_heads,
            "bytes": token_heads * per_th + state, "flops": token_heads * flops_th}


def algorithmic_work_split(w, lengths=None):
    """Bytes each launch of the tensor-core path must move, per token-head (valid
    tokens): the residual-write launch reads v and gain (I/O dtype) and gamma and
    alpha (fp32) and writes P~ (bf16, m d_v); the scan reads q, k, v, u (I/O dtype),
    P~ (bf16) and gamma, beta (fp32), writes o, and reads S0 / writes the final
    state per sequence-head."""
    es = 2 if w.dtype == "bf16" else 4
    m = w.m
    valid_tokens = int(lengths.sum()) if lengths is not None else w.B * w.T
    th = valid_tokens * w.H
    state = w.B * w.H * w.d_v * w.d_k * 4 * (2 if w.with_s0 else 1)
    prep = th * (es * w.d_v + es * m * w.d_v + 4 * (1 + m) + 2 * m * w.d_v)
    scan = th * (es * (2 * w.d_k + 2 * w.d_v) + es * m * w.d_k + 2 * m * w.d_v + 8) + state
    return {"residual_write": prep, "scan": scan}


def algorithmic_work_bwd(w, lengths=None):
    """Algorithmic bytes of one backward pass over workload ``w``: the forward's
    inputs and dO read once (as the forward's bytes with dO in place of o), the
    gradients written once in fp32 (dq, dk, dv, dgamma, dbeta, du, dalpha, dgain per
    token-head; dS0 per sequence-head; dS_final read per sequence-head)."""
    es = 2 if w.dtype == "bf16" else 4
    m = w.m
    valid_tokens = int(lengths.sum()) if lengths is not None else w.B * w.T
    token_heads = valid_tokens * w.H
    reads = es * (2 * w.d_k + 2 * w.d_v) + es * m * (w.d_k + w.d_v) + 4 * (2 + m)
    writes = 4 * (2 * w.d_k + w.d_v) + 4 * m * (w.d_k + w.d_v) + 4 * (2 + m)
    state = w.B * w.H * w.d_v * w.d_k * 4 * (3 if w.with_s0 else 2)
    return {"tokens": valid_tokens, "token_heads": token_heads, "bytes": token_heads * (reads + writes) + state}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def sha256_of(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of ``kernel`` and this workload; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    e = rec.get(kernel, {}).get(workload)
    if not e or e.get("source_sha256") != sha256_of(KERNEL_SOURCES[kernel]):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- multi-rank plumbing
def rank_workload(w, rank):
    """The batch rank ``rank`` scans: same shape, its own seed (independent
    replicas sharded by batch; no data crosses ranks)."""
    return w.replace(seed=w.seed + rank)


def max_over_ranks(x, dist, device):
    """Max of a per-rank float over all ranks (the job's time is its slowest rank)."""
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(tokens_per_rank, world, ms_per_step):
    """Whole-job tokens/s: the tokens every rank processed per step over the
    slowest rank's time per step."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r for r in csv.reader(io.StringIO(f.read())) if len(r) >= 9]
        os.unlink(self.file.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle (reference arm / baseline)
def time_oracle(w, budget_s, rows=None, tokens=None):
    """Time the fp64 oracle on a bounded sample of workload ``w``: the first
    ``tokens`` steps of the first ``rows`` batch rows, all heads."""
    from linear_attention_sequence_shortconv_b200 import synth
    from oracle import prism_seq

    rows = rows or 1
    tokens = tokens or w.T
    sample = w.replace(B=rows, T=tokens, lengths_lo=None)
    x = synth.to_float64_numpy(synth.make_inputs(sample))
    if w.L == 1:
        x["u"] = x["alpha"] = x["gain"] = None
    # every core this process may run on is offered to the BLAS and torch thread pools
    import torch

    avail = len(os.sched_getaffinity(0))
    torch.set_num_threads(avail)
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=avail):
        wall0, cpu0 = time.perf_counter(), time.process_time()
        prism_seq(**x)
        wall = time.perf_counter() - wall0
        cpu = time.process_time() - cpu0
    used = max(1, round(cpu / wall)) if wall > 0 else 1  # cores the oracle actually kept busy
    return {"tokens": rows * tokens, "seconds": wall, "cores": used, "cores_available": avail,
            "threads": avail, "sample": f"first {tokens} steps of {rows} batch row(s) x {w.H} heads of {w.name}"}


def calibrate_oracle_tokens(w, target_s):
    probe = time_oracle(w, 0, rows=1, tokens=min(w.T, 64))
    per_tok = probe["seconds"] / probe["tokens"]
    return max(8, min(w.T, int(target_s / max(per_tok, 1e-9))))


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    budget = 120.0
    tokens = calibrate_oracle_tokens(w, budget / max(1, steps + warmup))
    for _ in range(warmup):
        time_oracle(w, 0, rows=1, tokens=tokens)
    times, cores, sample, avail = [], 1, "", 1
    for _ in range(steps):
        r = time_oracle(w, 0, rows=1, tokens=tokens)
        times.append(r["seconds"])
        cores = max(cores, r["cores"])
        sample, avail = r["sample"], r["cores_available"]
    ms = 1e3 * sum(times) / len(times)
    value = tokens / (ms / 1e3)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": steps, "warmup": warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cores_available": avail, "threads": avail,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, n):
    return {"workload": f"{w.name}: B={w.B} T={w.T} H={w.H} d_k={w.d_k} d_v={w.d_v} L={w.L} chunk={w.chunk} "
                        f"W={w.W} {w.dtype}" + (f" lengths~U{{{w.lengths_lo}..{w.T}}}" if w.lengths_lo else ""),
            "B": w.B, "T": w.T, "H": w.H, "d_k": w.d_k, "d_v": w.d_v, "L": w.L, "chunk": w.chunk, "W": w.W,
            "parallelism": f"dp{n} (independent replicas, batch-sharded; no collective)",
            "l2": "flushed between timed steps (256 MiB write); inputs also exceed L2"}


# ---------------------------------------------------------------- our arm
def run_ours_bwd(args, w):
    """The training pass: prism_scan_bwd (gradients of every input) on workload ``w``."""
    import numpy as np
    import torch

    import linear_attention_sequence_shortconv_b200 as prism
    from linear_attention_sequence_shortconv_b200 import synth

    if int(os.environ.get("WORLD_SIZE", "1")) != 1:
        raise SystemExit("--pass bwd runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    host_inputs = synth.make_inputs(w)
    d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in host_inputs.items()}
    gen = torch.Generator().manual_seed(w.seed + 7)
    io_dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dO = torch.randn((w.B, w.T, w.H, w.d_v), generator=gen).to(io_dtype).to(dev)
    dSf = torch.randn((w.B, w.H, w.d_v, w.d_k), generator=gen).to(dev)
    code = prism.PRISM_BF16 if w.dtype == "bf16" else prism.PRISM_FP32
    ws = torch.empty(int(prism.lib().prism_scan_bwd_workspace_size(w.B, w.T, w.H, w.d_k, w.d_v, w.L, w.W, code)),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        return prism.scan_bwd(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"],
                              d["conv_w"], dO, L=w.L, S0=d["S0"], lengths=d["lengths"], dS_final=dSf,
                              workspace=ws, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if prism.stream_status() != 0:
        raise SystemExit("device status word reports an error after warm-up")
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clocks:
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / K
    work = algorithmic_work_bwd(w, host_inputs["lengths"].numpy() if host_inputs["lengths"] is not None else None)
    # d_k = d_v in {64, 128}, L <= 4: the chunked backward; otherwise the token-by-token one
    chunked = w.d_k == w.d_v and w.d_k in (64, 128) and w.L <= 4
    bwd_kernel = "chunk_grad" if chunked else "scan_bwd"
    bwd_timed = ("step = forward recording chunk-boundary states + adjoint pass + per-chunk gradients "
                 "+ dconv_w reduction" if chunked else "step = recording forward + reverse kernel + two reductions")
    peaks, peak_kind = load_peaks()
    achieved = work["bytes"] / (ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel": bwd_kernel,
                "timed": bwd_timed,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS hbm_gbs burst copy)" if peak_kind == "measured" else "fallback 6.65 TB/s",
                "algorithmic_bytes_per_launch": work["bytes"]}
    cpu_baseline = None
    if not args.no_cpu_baseline:
        from oracle.prism_grad import prism_seq_grad

        tokens = min(w.T, 128)
        sample = w.replace(B=1, T=tokens, lengths_lo=None)
        xs = synth.to_float64_numpy(synth.make_inputs(sample))
        if w.L == 1:
            xs["u"] = xs["alpha"] = xs["gain"] = None
        avail = len(os.sched_getaffinity(0))
        torch.set_num_threads(avail)
        t0, c0 = time.perf_counter(), time.process_time()
        prism_seq_grad(**xs, dO=np.ones((1, tokens, w.H, w.d_v)), dS_final=None)
        sec = time.perf_counter() - t0
        used = max(1, round((time.process_time() - c0) / sec)) if sec > 0 else 1
        cpu_baseline = {"value": tokens / sec, "unit": UNIT, "cores": used, "cores_available": avail,
                        "threads": avail, "kind": "oracle",
                        "sample": f"autograd of the first {tokens} steps of 1 batch row x {w.H} heads of {w.name}",
                        "seconds": sec}
    line = {"metric": "PRISM scan bwd (all input gradients) tokens/s on 1 B200", "value": work["tokens"] / (ms / 1e3),
            "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded)",
            "config": workload_config(w, 1), "roofline": roofline, "cpu_baseline": cpu_baseline, "e2e": None,
            "gpu_launches": 4 * K, "clocks": clocks.summary(), "impl": "ours", "pass": "bwd"}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import linear_attention_sequence_shortconv_b200 as prism
    from linear_attention_sequence_shortconv_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wr = rank_workload(w, rank)   # each rank scans its own batch
    host_inputs = synth.make_inputs(wr)
    d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in host_inputs.items()}
    io_dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    o = torch.empty((w.B, w.T, w.H, w.d_v), dtype=io_dtype, device=dev)
    S = torch.empty((w.B, w.H, w.d_v, w.d_k), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    dtype_code = prism.PRISM_BF16 if w.dtype == "bf16" else prism.PRISM_FP32
    ws_bytes = prism.workspace_size(w.B, w.T, w.H, w.d_k, w.d_v, w.L, w.W, w.chunk, dtype_code)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None

    def step():
        prism.scan_fwd(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"], d["conv_w"],
                       L=w.L, chunk=w.chunk, S0=d["S0"], lengths=d["lengths"], o=o, S_final=S, workspace=ws,
                       stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if prism.stream_status() != 0:
        raise SystemExit("device status word reports an error after warm-up")
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # the tensor-core path with residual writes is two launches (more for a cut sequence):
    # the library records mids[i] between the residual-write launch and the scan
    use_tc = prism.uses_tensor_cores(w.d_k, w.d_v, w.L, w.W, w.chunk, dtype_code)
    split = use_tc and w.L > 1
    launches_per_step = prism.scan_fwd_launches(w.B, w.T, w.H, w.d_k, w.d_v, w.L, w.W, w.chunk, dtype_code)
    first_chunks = prism.scan_fwd_split_chunks(w.B, w.T, w.H, w.d_k, w.d_v, w.L, w.W, w.chunk, dtype_code)
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(K)] if split else []
    for e in mids:
        e.record(stream)  # creates the event; the call below records it again
    with ClockSampler(local) as clocks:
        for i in range(K):
            flush.zero_()
            starts[i].record(stream)
            if split:
                prism.set_split_event(mids[i])
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
    prism.set_split_event(None)
    if world > 1:
        dist.barrier()
    if prism.stream_status() != 0:
        raise SystemExit("device status word reports an error in the timed region")
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = max_over_ranks(sum(per_step) / K, dist, dev)
    if split:
        prep_ms = max_over_ranks(sum(s.elapsed_time(m) for s, m in zip(starts, mids)) / K, dist, dev)
        scan_ms = max_over_ranks(sum(m.elapsed_time(e) for m, e in zip(mids, ends)) / K, dist, dev)
    work = algorithmic_work(w, host_inputs["lengths"].numpy() if host_inputs["lengths"] is not None else None)
    value = aggregate_throughput(work["tokens"], world, ms)

    # end to end through the host-buffer entry point: every step copies its inputs from
    # pinned host memory to HBM, scans, and copies o and S_final back.  Steps alternate
    # between two device buffer sets on two streams, so one step's scan and D2H copy
    # overlap the next step's H2D copy (PCIe is full duplex); each step still moves all
    # of its own bytes.
    e2e = None
    if not args.no_e2e:
        pinned_in = {n: (t.pin_memory() if isinstance(t, torch.Tensor) else None) for n, t in host_inputs.items()}
        slots = []
        for _ in range(2):
            pinned = dict(pinned_in)
            pinned["o"] = torch.empty(o.shape, dtype=io_dtype).pin_memory()
            pinned["S_final"] = torch.empty(S.shape, dtype=torch.float32).pin_memory()
            devbuf = {n: torch.empty_like(t, device=dev) for n, t in pinned.items() if t is not None}
            if ws_bytes:
                devbuf["workspace"] = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
            slots.append((pinned, devbuf, torch.cuda.Stream(device=dev)))
        K2 = max(1, min(K, args.e2e_steps))
        for pinned, devbuf, st in slots:
            prism.scan_fwd_host(pinned, devbuf, L=w.L, chunk=w.chunk, stream=st)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(slots[0][2])
        slots[1][2].wait_event(e0)
        for i in range(K2):
            pinned, devbuf, st = slots[i % 2]
            prism.scan_fwd_host(pinned, devbuf, L=w.L, chunk=w.chunk, stream=st)
        done1 = torch.cuda.Event()
        done1.record(slots[1][2])
        slots[0][2].wait_event(done1)
        e1.record(slots[0][2])
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1) / K2, dist, dev)
        h2d = sum(t.numel() * t.element_size() for n, t in pinned_in.items() if t is not None)
        d2h = slots[0][0]["o"].numel() * slots[0][0]["o"].element_size() + S.numel() * 4
        e2e = {"value": aggregate_throughput(work["tokens"], world, ems), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K2,
               "api": "prism_scan_fwd_host (C ABI, pinned host buffers; two buffer sets on two streams)"}

    # roofline against measured HBM bandwidth.  The dominant kernel is the scan, timed live
    # by CUDA events on the launching stream (the library records one between its two
    # launches); "path" is the whole step against the forward's algorithmic bytes
    # (q, k, v, u, gain, gates read once, o written once), the fraction of the method's
    # roofline that the step reaches.
    kernel = "chunk_scan" if use_tc else "recurrent"
    peaks, peak_kind = load_peaks()
    hbm = peaks["hbm_gbs"]
    peak_src = f"{peak_kind} (MEASURED_PEAKS hbm_gbs burst copy)" if peak_kind == "measured" else "fallback 6.65 TB/s"
    lens_np = host_inputs["lengths"].numpy() if host_inputs["lengths"] is not None else None
    t_s = ms / 1e3
    path = {"us": ms * 1e3, "algorithmic_bytes": work["bytes"], "achieved_gbs": work["bytes"] / t_s / 1e9,
            "frac": work["bytes"] / t_s / 1e9 / hbm, "algorithmic_flops": work["flops"],
            "tensor_frac_of_peak": work["flops"] / t_s / 1e12 / peaks["bf16_tflops"],
            "roofline_time_us": 1e6 * max(work["bytes"] / (hbm * 1e9), work["flops"] / (peaks["bf16_tflops"] * 1e12))}
    path["roofline_frac"] = path["roofline_time_us"] / path["us"]
    if split:
        # with the scan in two halves (four launches) the first residual-write launch covers
        # the first launch's chunks (first_chunks of nc), and the second half's residual
        # write runs beside the first scan launch: its bytes count in the scan's window
        sw = algorithmic_work_split(w, lens_np)
        nc = -(-w.T // w.chunk)
        halves = launches_per_step == 4
        f_first = first_chunks / nc if halves else 1.0
        rw_first = sw["residual_write"] * f_first
        scan_bytes = sw["scan"] + sw["residual_write"] * (1.0 - f_first)
        scan_gbs = scan_bytes / (scan_ms / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": scan_gbs, "peak": hbm, "unit": "GB/s", "frac": scan_gbs / hbm,
                    "traffic": recorded_traffic("prism_scan_kernel", w.name), "kernel": "prism_scan_kernel",
                    "timed": ("scan launches of each step (two halves, the second half's residual write "
                              "beside the first), CUDA events on the call's stream" if halves else
                              "scan launch(es) of each step, CUDA events on the launching stream"),
                    "kernel_us": scan_ms * 1e3, "algorithmic_bytes_per_launch": scan_bytes, "peak_source": peak_src,
                    "residual_write": {"kernel": "residual_write_kernel" + (
                                           f" (chunks 0-{first_chunks - 1}, first launch)" if halves else ""),
                                       "us": prep_ms * 1e3, "algorithmic_bytes": rw_first,
                                       "achieved_gbs": rw_first / (prep_ms / 1e3) / 1e9,
                                       "frac": rw_first / (prep_ms / 1e3) / 1e9 / hbm,
                                       "traffic": recorded_traffic("residual_write_kernel", w.name)},
                    "path": path}
    else:
        roofline = {"bound": "hbm", "achieved": path["achieved_gbs"], "peak": hbm, "unit": "GB/s",
                    "frac": path["frac"], "traffic": recorded_traffic(kernel, w.name), "kernel": kernel,
                    "timed": "step = one launch", "kernel_us": ms * 1e3,
                    "algorithmic_bytes_per_launch": work["bytes"], "peak_source": peak_src, "path": path}

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = 4 if w.T >= 1024 else 16
        r = time_oracle(w, 0, rows=min(rows, w.B), tokens=min(w.T, 2048))
        cpu_baseline = {"value": r["tokens"] / r["seconds"], "unit": UNIT, "cores": r["cores"],
                        "cores_available": r["cores_available"], "threads": r["threads"], "kind": "oracle",
                        "sample": r["sample"], "seconds": r["seconds"]}

    clk = clocks.summary()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded; shapes and distributions of the method's workloads)",
            "config": workload_config(w, world), "roofline": roofline, "cpu_baseline": cpu_baseline,
            "e2e": e2e, "gpu_launches": K * launches_per_step, "clocks": clk,
            "tokens_per_step_per_gpu": work["tokens"],
        }
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="lm_130m")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (smaller profiling captures)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="pass_", choices=("fwd", "bwd"), default="fwd",
                    help="fwd: the scan (the headline); bwd: prism_scan_bwd, one GPU")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    from linear_attention_sequence_shortconv_b200 import synth

    w = synth.WORKLOADS[args.workload]
    if args.batch is not None:
        w = w.replace(B=args.batch, name=f"{w.name}_b{args.batch}")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.pass_ == "bwd":
        return run_ours_bwd(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
