#!/usr/bin/env python
"""Benchmark of the fused ELMO classifier-head training step on B200.

One step is one pass of the whole hot path (label preparation, X
quantisation, logits and gradient, input gradient, weight gradient fused with
the stochastic-rounding update) over one batch of synthetic input, through the
C ABI of libelmo.  Default workload: the 3M-label FP8 head (L = 3,000,000,
d = 768, B = 256, chunk 131,072, lr 0.1), shaped like the Amazon-3M result of
"ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
Output Spaces"; the data are synthetic (the dataset is not available).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl elmo|reference]
                    [--workload NAME]

Prints one JSON line (rank 0).  For N > 1 the ranks hold one head of N * L
labels split by labels (rank r the rows [r L, (r + 1) L)): every rank runs the
fused step on its rows for the same batch and the ranks' input gradients are
summed by one all-reduce of dX per step (weak scaling: L labels per GPU); the
time is the max over ranks.  `--impl reference` times the CPU oracle (a deliberately
plain program) on a bounded sample of the same workload.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused XMC head train step: label-rows/s, TFLOP/s and % roofline (1×B200)"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="elmo", choices=["elmo", "reference"])
    p.add_argument("--workload", default="product3m_fp8")
    p.add_argument("--labels", type=int, default=0, help="override L (smaller cases for profiling)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target length of the oracle sample")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                "sm_max_mhz": pk.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        rows = []
        with open(self.f.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def step_costs(w):
    """Algorithmic work of one step: flops of the three contractions and the
    weight bytes that must cross HBM (read + write once)."""
    s_w = 2 if w.dtype == "bf16" else 1
    return {"flops": 6.0 * w.B * w.L * w.d, "w_bytes": 2.0 * w.L * w.d * s_w}


def tensor_peak_tflops(peaks, dtype, sustained=True):
    base = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    return base * (1.0 if dtype == "bf16" else 2.0)   # fp8 dense = 2 x bf16 dense (nominal ratio)


def alu_peak_tflops(peaks):
    # fp32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 flop x max SM clock
    return 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12


def max_over_ranks(ms, device=None):
    """The job's time: the largest of the ranks' device times (every rank calls
    this at the same point; one process: the value itself)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, labels, steps, ms):
    """Whole-job label-rows/s: every rank processes its L labels per step (its
    rows of the split head), so the job processes world * L * steps label-rows
    in the max time."""
    return world * labels * steps / (ms / 1e3)


def code_digest(path):
    """sha256 of a source file's code: comments removed and white space
    collapsed, so that an edit of the comments keeps the digest."""
    import hashlib
    import re
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()


def profiled_traffic(kernel, workload):
    """DRAM bytes (read + write) of one full launch of `kernel`, from the ncu
    summary committed under profiles/, with the labels that launch covered.
    None when there is no summary or when the kernel's code has changed since
    the counters were taken (the summary records code_digest of the source)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    try:
        # "path digest", or several such pairs separated by ";" (a kernel and its headers)
        for pair in fields["source"].split(";"):
            src, digest = pair.split()
            if code_digest(os.path.join(ROOT, src)) != digest:
                return None
        units = fields.get("labels per launch", fields.get("values per launch"))
        return {"bytes": float(fields["dram bytes per launch"]), "labels": int(units)}
    except (KeyError, ValueError, OSError):
        return None


def cpu_baseline(w, W_rows_host, X, rowptr, cols, target_s):
    """The oracle as it stands, on a bounded label sample of the same workload."""
    import oracle
    oracle.build()
    nthreads = os.cpu_count() or 1
    probe = min(w.L, W_rows_host.shape[0], 2048)      # enough labels that fixed costs do not dominate the rate
    t = time.perf_counter()
    oracle.train_step(W_rows_host[:probe], X, rowptr, cols, w.lr, 0, 0, w.dtype, 0, probe, L=w.L, nthreads=nthreads)
    per = (time.perf_counter() - t) / probe
    n = int(max(probe, min(W_rows_host.shape[0], target_s / max(per, 1e-9))))
    t = time.perf_counter()
    oracle.train_step(W_rows_host[:n], X, rowptr, cols, w.lr, 0, 0, w.dtype, 0, n, L=w.L, nthreads=nthreads)
    dt = time.perf_counter() - t
    return {"value": n / dt, "unit": "label-rows/s", "cores": nthreads, "kind": "oracle",
            "sample": f"labels [0, {n}) of the {w.L}-label step (full B={w.B}, d={w.d}), {dt:.1f} s",
            "tflops": 6.0 * w.B * n * w.d / dt / 1e12}


def run_reference(args, w):
    import oracle
    from synthetic import make_labels, make_W_bf16, make_W_f32, make_X
    oracle.build()
    nthreads = os.cpu_count() or 1
    X = make_X(w, 0)
    rowptr, cols = make_labels(w, 0)
    # sample size: about 120 s of oracle work for the whole run (warm-up steps included)
    probe = min(w.L, 2048)      # enough labels that fixed costs do not dominate the rate
    Wp = make_W_f32(w, rows=probe)
    wgrid = {"bf16": "bf16", "fp8": "fp8", "fp8_ge5m2": "fp8", "e5m2": "e5m2"}[w.dtype]
    Wq = oracle.sr_round(Wp, wgrid, 0, 2**64 - 1) if w.dtype != "bf16" else make_W_bf16(w)[:probe]
    t = time.perf_counter()
    oracle.train_step(Wq, X, rowptr, cols, w.lr, 0, 0, w.dtype, 0, probe, L=w.L, nthreads=nthreads)
    per = (time.perf_counter() - t) / probe
    per_step_s = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(probe, min(w.L, per_step_s / max(per, 1e-9))))
    Wf = make_W_f32(w, rows=n)
    Wq = oracle.sr_round(Wf, wgrid, 0, 2**64 - 1) if w.dtype != "bf16" else oracle.rne_bf16(Wf)
    for s in range(args.warmup):
        oracle.train_step(Wq, make_X(w, s), *make_labels(w, s), w.lr, 0, s, w.dtype, 0, n, L=w.L, nthreads=nthreads)
    t = time.perf_counter()
    for s in range(args.warmup, args.warmup + args.steps):
        oracle.train_step(Wq, make_X(w, s), *make_labels(w, s), w.lr, 0, s, w.dtype, 0, n, L=w.L, nthreads=nthreads)
    dt = time.perf_counter() - t
    value = n * args.steps / dt
    line = {
        "metric": METRIC, "value": value, "unit": "label-rows/s", "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "L": w.L, "d": w.d, "B": w.B, "w_dtype": w.dtype, "chunk": w.chunk,
                   "sample_labels": n},
        "cpu_baseline": {"value": value, "unit": "label-rows/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"labels [0, {n}) of each {w.L}-label step (full B={w.B}, d={w.d})"},
        "e2e": {"value": value, "unit": "label-rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _time_reference(args, fn):
    """Warm-up calls, then the mean seconds per timed call of fn(step)."""
    for s in range(args.warmup):
        fn(s)
    t = time.perf_counter()
    for s in range(args.warmup, args.warmup + args.steps):
        fn(s)
    return (time.perf_counter() - t) / args.steps


def run_reference_other(args, w):
    """--impl reference for the workloads other than the training step: the
    oracle as it stands, timed on a bounded sample (about 60 s for the run)."""
    import oracle
    from synthetic import make_X
    oracle.build()
    nthreads = os.cpu_count() or 1
    per_step_s = 60.0 / max(1, args.steps + args.warmup)
    rng = np.random.default_rng(0)
    if args.workload == "sr_round":
        metric, unit, cores = "standalone SR: values/s", "values/s", 1
        probe = (rng.standard_normal(1 << 16) * 0.02).astype(np.float32)
        t = time.perf_counter()
        oracle.sr_round(probe, "fp8", 0, 0)
        n = int(min(1 << 28, max(probe.size, per_step_s * probe.size / (time.perf_counter() - t))))
        x = (rng.standard_normal(n) * 0.02).astype(np.float32)
        sec = _time_reference(args, lambda s: oracle.sr_round(x, "fp8", 0, s))
        units, sample, config = n, f"{n} fp32 values to E4M3 per step", {"workload": "sr_round", "n": n}
    elif args.workload == "kahan_sgd":
        metric, unit, cores = "Kahan-compensated bf16 SGD: params/s", "params/s", 1
        bits = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)   # noqa: E731
        probe = 1 << 16
        p0, g0 = bits(rng.standard_normal(probe) * 0.05), bits(rng.standard_normal(probe) * 1e-2)
        t = time.perf_counter()
        oracle.kahan_sgd(p0, np.zeros(probe, np.uint16), g0, 1e-3)
        n = int(min(110_000_000, max(probe, per_step_s * probe / (time.perf_counter() - t))))
        p, c, g = bits(rng.standard_normal(n) * 0.05), np.zeros(n, np.uint16), bits(rng.standard_normal(n) * 1e-2)
        sec = _time_reference(args, lambda s: oracle.kahan_sgd(p, c, g, 1e-3))
        units, sample, config = n, f"{n} parameters per step", {"workload": "kahan_sgd", "n": n}
    else:                                   # top-k prediction
        metric, unit, cores = "chunked top-k predict: query-labels/s", "query-labels/s", nthreads
        import torch                        # W codes of N(0, 0.02^2), made block by block (timing only)
        gen = torch.Generator().manual_seed(0)
        fp8 = w.dtype != "bf16"
        Wq = np.empty((w.L, w.d), np.uint8 if fp8 else np.uint16)
        for r0 in range(0, w.L, 1 << 17):
            blk = torch.randn(min(1 << 17, w.L - r0), w.d, generator=gen) * 0.02
            Wq[r0:r0 + blk.shape[0]] = (blk.to(torch.float8_e4m3fn).view(torch.uint8) if fp8
                                         else blk.to(torch.bfloat16).view(torch.int16)).numpy().view(Wq.dtype)
        X = make_X(w, 0)
        t = time.perf_counter()
        oracle.topk(Wq, X, w.topk, w.dtype, rows=[0], nthreads=nthreads)
        rows = int(min(w.B, max(1, per_step_s / (time.perf_counter() - t))))
        sec = _time_reference(args, lambda s: oracle.topk(Wq, X, w.topk, w.dtype, rows=list(range(rows)),
                                                          nthreads=nthreads))
        units = rows * w.L
        sample = f"query rows [0, {rows}) against all {w.L} labels per step"
        config = {"workload": w.name, "L": w.L, "d": w.d, "B": w.B, "w_dtype": w.dtype, "k": w.topk}
    value = units / sec
    print(json.dumps({
        "metric": metric, "value": value, "unit": unit, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config,
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_topk(args, w, rank, world, local):
    """Chunked top-k prediction (X [B x d] bf16 against the whole head): one
    step is one elmo_topk_predict call over all L labels.  N > 1: a head of
    N * L labels split by labels; each rank ranks its L rows, the ranks' lists
    are gathered and merged on the device."""
    import torch
    import torch.distributed as dist
    import precision_label_chunk_b200 as elmo
    from precision_label_chunk_b200.sharded import ShardedHead
    from synthetic import make_X
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    wdt = torch.int16 if w.dtype == "bf16" else torch.uint8
    W = torch.empty(w.L, w.d, dtype=wdt, device=dev)
    labels_total = world * w.L
    sharded = ShardedHead(W, labels_total, w.dtype, fill=True, init_std=0.02, seed=0, label_base=rank * w.L)
    head = sharded.head
    nsteps = args.warmup + args.steps
    Xh = [make_X(w, s) for s in range(nsteps)]
    Xd = [torch.from_numpy(x.view(np.int16)).to(dev) for x in Xh]
    idx = torch.empty(w.B, w.topk, dtype=torch.int32, device=dev)
    sc = torch.empty(w.B, w.topk, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    predict = lambda X: sharded.topk_predict(X, w.topk, w.chunk, idx, sc)   # noqa: E731
    for s in range(args.warmup):
        predict(Xd[s])
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    launches0 = elmo.elmo_launch_count(head)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for s in range(args.warmup, nsteps):
        predict(Xd[s])
    ev1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    # the head's kernels, plus one merge launch per step when split
    gpu_launches = elmo.elmo_launch_count(head) - launches0 + (args.steps if world > 1 else 0)
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev) / args.steps
    # per-kernel pass (events around every launch, outside the timed region)
    elmo.elmo_profile_reset(head)
    elmo.elmo_profile_enable(head, True)
    for s in range(args.warmup, nsteps):
        predict(Xd[s])
    torch.cuda.synchronize()
    elmo.elmo_profile_enable(head, False)
    classes = {}
    for name in elmo.KERNEL_CLASSES:
        t_ms, n = elmo.elmo_profile_read(head, name)
        if n:
            classes[name] = {"ms": t_ms, "launches": n}
    flops = 2.0 * w.B * w.L * w.d
    dominant = max(classes, key=lambda k: classes[k]["ms"]) if classes else None
    roof = None
    if dominant == "topk_score":
        t_k = classes[dominant]["ms"] / 1e3 / args.steps
        if os.environ.get("ELMO_TOPK_SIMT", "0") == "1":
            peak, bound, src = alu_peak_tflops(peaks), "alu", "derived: 148 SM x 128 FMA x 2 x max clock"
        else:
            # tensor-core screening: the algorithmic 2 B L d flops against the dense
            # peak of the operand type (E4M3 heads issue the contraction twice, for
            # the two E4M3 parts of the bf16 queries, so their ceiling is frac = 0.5)
            peak, bound = tensor_peak_tflops(peaks, w.dtype), "tensor"
            src = (f"{peaks['source']} bf16 sustained" + (" x 2 (fp8/bf16 nominal ratio)" if w.dtype != "bf16" else ""))
        tr = profiled_traffic("topk_screen_tc", w.name) if bound == "tensor" else None
        roof = {"kernel": dominant, "bound": bound, "achieved": flops / t_k / 1e12, "peak": peak, "unit": "TFLOP/s",
                "frac": flops / t_k / 1e12 / peak,
                "traffic": None if tr is None else tr["bytes"] * w.L / tr["labels"], "peak_source": src,
                "mma_passes": 2 if (w.dtype != "bf16" and bound == "tensor") else 1}
    # end to end: X from pinned host memory, indices and scores back every step
    pin = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in Xh]
    idx_h = torch.empty(w.B, w.topk, dtype=torch.int32).pin_memory()
    sc_h = torch.empty(w.B, w.topk, dtype=torch.float32).pin_memory()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for s in range(args.warmup, nsteps):
        predict(pin[s].to(dev, non_blocking=True))
        idx_h.copy_(idx, non_blocking=True)
        sc_h.copy_(sc, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), dev) / args.steps
    # rows of the last call whose screening could not certify the top-k and
    # that took the exact CUDA-core path
    uncertified = elmo.elmo_topk_uncertified_rows(head, w.B, w.topk)
    # P@1, P@3, P@5 of the last predictions against the queries' synthetic labels
    # (random weights: near zero; the point is that the metric runs on the device)
    from synthetic import make_labels, workload
    rp, cl = make_labels(w if world == 1 else workload(w.name, L=labels_total), nsteps - 1)
    kk = min(5, w.topk)
    pk = torch.empty(kk, dtype=torch.float32, device=dev)
    elmo.elmo_precision_at_k(idx[:, :kk].contiguous(), torch.from_numpy(rp).to(dev), torch.from_numpy(cl).to(dev), pk)
    p_at_k = {f"P@{j}": float(pk[j - 1]) for j in (1, 3, 5) if j <= kk}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        Wh = W.cpu().numpy().view(np.uint8 if w.dtype != "bf16" else np.uint16)
        nthreads = os.cpu_count() or 1
        t = time.perf_counter()
        oracle.topk(Wh, Xh[0], w.topk, w.dtype, rows=[0], nthreads=nthreads)
        dt = time.perf_counter() - t
        cpu = {"value": w.L / dt, "unit": "query-labels/s", "cores": nthreads, "kind": "oracle",
               "sample": f"query row 0 against all {w.L} labels, {dt:.1f} s"}
    if rank == 0:
        line = {
            "metric": "chunked top-k predict: query-labels/s", "value": world * w.B * w.L / (ms / 1e3),
            "unit": "query-labels/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "L": w.L, "d": w.d, "B": w.B, "w_dtype": w.dtype, "k": w.topk,
                       "chunk": w.chunk, "l2": f"inputs larger than L2 (W = {w.L * w.d / 1e9:.2f} GB per GPU)",
                       "labels_total": labels_total,
                       "parallelism": f"label-shards{world} (gather + merge of top-k)" if world > 1 else "single"},
            "tflops": flops / (ms / 1e3) / 1e12, "roofline": roof, "kernels": classes,
            "gpu_launches": gpu_launches,
            "e2e": {"value": world * w.B * w.L / (ms_e2e / 1e3), "unit": "query-labels/s",
                    "h2d_bytes_per_step": w.B * w.d * 2, "d2h_bytes_per_step": w.B * w.topk * 8},
            "cpu_baseline": cpu, "clocks": clocks, "p_at_k": p_at_k,
            "uncertified_rows": {"rows": uncertified, "of": w.B},
        }
        print(json.dumps(line), flush=True)
    head.close()
    if world > 1:
        dist.destroy_process_group()


def run_sr(args, local):
    """Standalone stochastic rounding of 2^28 fp32 values to E4M3, bf16 and E5M2:
    an HBM-bound pass (4 bytes read and 1 or 2 bytes written per value)."""
    import torch
    import precision_label_chunk_b200 as elmo
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    n = 1 << 28
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    x = torch.randn(n, generator=g, device=dev) * 0.02
    res = {}
    for dt, odt, ob in (("fp8", torch.uint8, 1), ("bf16", torch.int16, 2), ("e5m2", torch.uint8, 1)):
        out = torch.empty(n, dtype=odt, device=dev)
        for s in range(args.warmup):
            elmo.elmo_sr_round(x, out, dt, 0, s)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s in range(args.steps):
            elmo.elmo_sr_round(x, out, dt, 0, args.warmup + s)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        gbs = n * (4 + ob) / (ms / 1e3) / 1e9
        res[dt] = {"ms": ms, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]}
    line = {"metric": "standalone SR: values/s", "value": n / (res["fp8"]["ms"] / 1e3), "unit": "values/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["fp8"]["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "sr_round", "n": n, "l2": "inputs larger than L2 (1 GiB fp32)"},
            "roofline": {"kernel": "sr_round", "bound": "hbm", "achieved": res["fp8"]["GB/s"],
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": res["fp8"]["frac"],
                         "traffic": (lambda tr: None if tr is None else tr["bytes"] * n / tr["labels"])(
                             profiled_traffic("sr_round_vec", "sr_round")),
                         "peak_source": f"{peaks['source']} copy bandwidth"},
            "per_dtype": res}
    print(json.dumps(line), flush=True)


def run_kahan(args, local):
    """Kahan-compensated SGD of an encoder-sized BF16 parameter vector (110M
    parameters, a BERT-base-sized encoder): bf16 p, c, g read and p, c written,
    10 bytes per parameter, HBM-bound.  One step is one update of all
    parameters; the fp32 dX of the head (B = 256, d = 768) handed over in
    bf16 is timed beside it."""
    import torch
    import precision_label_chunk_b200 as elmo
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    n = 110_000_000
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    P = (torch.randn(n, generator=gen, device=dev) * 0.05).to(torch.bfloat16)
    C = torch.zeros(n, dtype=torch.bfloat16, device=dev)
    G = (torch.randn(n, generator=gen, device=dev) * 1e-2).to(torch.bfloat16)
    lr = 1e-3
    for _ in range(args.warmup):
        elmo.elmo_kahan_sgd(P, C, G, lr)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        elmo.elmo_kahan_sgd(P, C, G, lr)
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    gbs = n * 10 / (ms / 1e3) / 1e9
    # dX of the head to bf16 (small: launch-bound, reported for completeness)
    dX = torch.randn(256 * 768, generator=gen, device=dev)
    dXb = torch.empty(256 * 768, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        elmo.elmo_round_bf16(dX, dXb)
    torch.cuda.synchronize()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record()
    for _ in range(100):
        elmo.elmo_round_bf16(dX, dXb)
    r1.record()
    torch.cuda.synchronize()
    # end to end: the gradient from pinned host memory, the parameters back to the host
    Gh = G.cpu().pin_memory()
    Ph = torch.empty(n, dtype=torch.bfloat16).pin_memory()
    torch.cuda.synchronize()
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record()
    for _ in range(args.steps):
        elmo.elmo_kahan_sgd(P, C, Gh.to(dev, non_blocking=True), lr)
        Ph.copy_(P, non_blocking=True)
    h1.record()
    torch.cuda.synchronize()
    ms_e2e = h0.elapsed_time(h1) / args.steps
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        oracle.build()
        ps, cs, gs = (t.view(torch.int16).cpu().numpy().view(np.uint16) for t in (P, C, G))
        t, k = time.perf_counter(), 0
        while k < 3 and time.perf_counter() - t < args.cpu_seconds:     # bounded: at most 3 steps
            ps, cs = oracle.kahan_sgd(ps, cs, gs, lr)
            k += 1
        dt = time.perf_counter() - t
        cpu = {"value": k * n / dt, "unit": "params/s", "cores": 1, "kind": "oracle",
               "sample": f"all {n} parameters, {k} step(s), {dt:.1f} s"}
    tr = profiled_traffic("kahan_sgd_vec", "kahan_sgd")
    line = {"metric": "Kahan-compensated bf16 SGD: params/s", "value": n / (ms / 1e3), "unit": "params/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (fp32 arithmetic)",
            "data": "synthetic",
            "config": {"workload": "kahan_sgd", "n": n, "lr": lr,
                       "l2": "inputs larger than L2 (660 MB of bf16 p, c, g)"},
            "roofline": {"kernel": "kahan_sgd_vec", "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "traffic": None if tr is None else tr["bytes"] * n / tr["labels"],
                         "bytes_per_param": 10, "peak_source": f"{peaks['source']} copy bandwidth"},
            "round_bf16_dx_us": r0.elapsed_time(r1) / 100 * 1e3,
            "gpu_launches": args.steps,
            "e2e": {"value": n / (ms_e2e / 1e3), "unit": "params/s", "h2d_bytes_per_step": n * 2,
                    "d2h_bytes_per_step": n * 2},
            "cpu_baseline": cpu, "clocks": clocks}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":            # the oracle on the host cores, rank 0 only
        if int(os.environ.get("RANK", "0")) == 0:
            from synthetic import workload
            if args.workload in ("sr_round", "kahan_sgd"):
                run_reference_other(args, None)
            else:
                w = workload(args.workload, **({"L": args.labels} if args.labels else {}))
                (run_reference_other if w.topk > 0 else run_reference)(args, w)
        return
    if args.workload in ("sr_round", "kahan_sgd"):
        if int(os.environ.get("RANK", "0")) == 0:
            (run_sr if args.workload == "sr_round" else run_kahan)(args, int(os.environ.get("LOCAL_RANK", "0")))
        return
    from synthetic import workload
    w = workload(args.workload, **({"L": args.labels} if args.labels else {}))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if w.topk > 0:
        run_topk(args, w, rank, world, local)
        return

    import torch
    import torch.distributed as dist

    import precision_label_chunk_b200 as elmo
    from precision_label_chunk_b200.sharded import ShardedHead
    from synthetic import make_labels, make_X

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    costs = step_costs(w)

    # model state: W resident in HBM, filled on the device (SR of N(0, 0.02^2)).
    # N > 1: this rank's L rows of a head of N * L labels; the labels of a
    # batch are drawn over the whole head
    wdt = torch.int16 if w.dtype == "bf16" else torch.uint8
    W = torch.empty(w.L, w.d, dtype=wdt, device=dev)
    labels_total = world * w.L
    sharded = ShardedHead(W, labels_total, w.dtype, fill=True, init_std=0.02, seed=0, label_base=rank * w.L)
    head = sharded.head
    w_labels = w if world == 1 else workload(args.workload, L=labels_total)
    nsteps = args.warmup + args.steps
    host_batches = []
    for s in range(nsteps):
        X = make_X(w, s)
        rowptr, cols = make_labels(w_labels, s)
        host_batches.append((X, rowptr, cols))
    dev_batches = [(torch.from_numpy(X.view(np.int16)).to(dev), torch.from_numpy(rp).to(dev),
                    torch.from_numpy(cl).to(dev)) for X, rp, cl in host_batches]
    dX = torch.empty(w.B, w.d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(s, batch):
        Xd, rp, cl = batch
        sharded.train_step(Xd, rp, cl, w.lr, w.chunk, 0, s, dX)     # + all-reduce of dX when N > 1

    for s in range(args.warmup):
        step(s, dev_batches[s])
    elmo.elmo_sync_status(head)
    torch.cuda.synchronize()

    # ---------------------------------------------------------------- timed region
    sampler = ClockSampler(local)
    launches0 = elmo.elmo_launch_count(head)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for s in range(args.warmup, nsteps):
        step(s, dev_batches[s])
    ev1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    elmo.elmo_sync_status(head)
    gpu_launches = elmo.elmo_launch_count(head) - launches0
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    ms_per_step = ms / args.steps
    value = job_throughput(world, w.L, args.steps, ms)

    # ---------------------------------------------------------------- per-kernel pass
    # The same K steps again, with the library recording a CUDA event pair on
    # the launch stream around every kernel.  An event between two kernels
    # costs a few microseconds of device time (the next launch can no longer
    # be overlapped with the previous kernel's drain), so these events stay
    # out of the timed region above; `kernels_pass_ms_per_step` reports what
    # the pass itself took.
    elmo.elmo_profile_reset(head)
    elmo.elmo_profile_enable(head, True)
    torch.cuda.synchronize()
    pv0, pv1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pv0.record(stream)
    for s in range(args.warmup, nsteps):
        step(nsteps + s, dev_batches[s])
    pv1.record(stream)
    torch.cuda.synchronize()
    elmo.elmo_profile_enable(head, False)
    elmo.elmo_sync_status(head)
    classes = {}
    for name in elmo.KERNEL_CLASSES:
        t_ms, n = elmo.elmo_profile_read(head, name)
        if n:
            classes[name] = {"ms": t_ms, "launches": n}
    elmo.elmo_profile_reset(head)
    kernels_pass_ms = pv0.elapsed_time(pv1) / args.steps

    # roofline of the dominant kernel class: algorithmic flops of the
    # contractions it performs per step (2 B L d each) over its device time
    # (the persistent step kernel does all three; the range-by-range kernels one or two).
    # The kernel is timed inside a pass of tens of milliseconds: the burst peak applies.
    contractions = {"logits_grad": 1, "update": 2, "step": 3}
    dominant = max(classes, key=lambda k: classes[k]["ms"]) if classes else None
    roof = None
    if dominant in contractions:
        fl_per_step = contractions[dominant] * 2.0 * w.B * w.L * w.d
        achieved = fl_per_step * args.steps / (classes[dominant]["ms"] / 1e3) / 1e12
        peak, bound = tensor_peak_tflops(peaks, w.dtype, sustained=False), "tensor"
        src = (f"{peaks['source']} bf16 burst" + (" x 2 (fp8/bf16 nominal ratio)" if w.dtype != "bf16" else ""))
        # ncu DRAM bytes of one full launch, scaled to the mean launch of this
        # run by the labels it covers (the kernel's traffic is linear in them)
        tr = profiled_traffic({"update": "update_tc", "logits_grad": "logits_grad_xt", "step": "step_fused"}.get(
            dominant, dominant), w.name)
        traffic = None
        if tr is not None:
            traffic = tr["bytes"] * (w.L / (classes[dominant]["launches"] / args.steps)) / tr["labels"]
        roof = {"kernel": dominant, "bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "peak_source": src,
                "flops_per_launch": fl_per_step / (classes[dominant]["launches"] / args.steps),
                "launches_per_step": classes[dominant]["launches"] / args.steps}

    # the step against its own roofline (slower of tensor and HBM time)
    t_tensor = costs["flops"] / (tensor_peak_tflops(peaks, w.dtype) * 1e12)
    t_hbm = costs["w_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_tensor, t_hbm)
    t_roof_burst = max(costs["flops"] / (tensor_peak_tflops(peaks, w.dtype, sustained=False) * 1e12), t_hbm)
    step_roof = {"t_roof_ms": t_roof * 1e3, "bound": "tensor" if t_tensor >= t_hbm else "hbm",
                 "frac": t_roof / (ms_per_step / 1e3), "tflops": costs["flops"] / (ms_per_step / 1e3) / 1e12,
                 "peaks": f"{peaks['source']}: {tensor_peak_tflops(peaks, w.dtype):.0f} TFLOP/s "
                          f"({w.dtype}, sustained), {peaks['hbm_gbs']:.0f} GB/s",
                 "t_roof_burst_ms": t_roof_burst * 1e3, "frac_burst": t_roof_burst / (ms_per_step / 1e3)}

    # ---------------------------------------------------------------- end to end (host buffers)
    pin = [(torch.from_numpy(X.view(np.int16)).pin_memory(), torch.from_numpy(rp).pin_memory(),
            torch.from_numpy(cl).pin_memory()) for X, rp, cl in host_batches]
    dX_host = torch.empty(w.B, w.d, dtype=torch.float32).pin_memory()
    h2d = sum(X.numel() * 2 + rp.numel() * 4 + cl.numel() * 4 for X, rp, cl in pin[args.warmup:]) / args.steps
    d2h = dX_host.numel() * 4
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(args.warmup, nsteps):
        Xh, rph, clh = pin[s]
        batch = (Xh.to(dev, non_blocking=True), rph.to(dev, non_blocking=True), clh.to(dev, non_blocking=True))
        step(s, batch)
        dX_host.copy_(dX, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e = {"value": job_throughput(world, w.L, args.steps, ms_e2e), "unit": "label-rows/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    # ---------------------------------------------------------------- CPU oracle baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Wh = W[: 200_000].cpu().numpy()
        Wh = Wh.view(np.uint16) if w.dtype == "bf16" else Wh.view(np.uint8)
        X, rp, cl = host_batches[0]
        cpu = cpu_baseline(w, Wh, X, rp, cl, args.cpu_seconds)

    peak_mem = torch.cuda.max_memory_allocated(dev) + elmo.elmo_head_workspace_bytes(head)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "label-rows/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": {"bf16": "bf16", "fp8": "fp8-e4m3", "fp8_ge5m2": "fp8-e4m3 (e5m2 gradient operand)",
                                             "e5m2": "fp8-e5m2 weights, e4m3 operands"}[w.dtype], "data": "synthetic",
            "config": {"workload": w.name, "L": w.L, "d": w.d, "B": w.B, "w_dtype": w.dtype, "chunk": w.chunk,
                       "lr": w.lr, "positives_per_sample": f"1+Poisson({w.lam})", "zipf_s": w.zipf_s,
                       "l2": f"inputs larger than L2 (W = {costs['w_bytes'] / 2 / 1e9:.2f} GB per GPU)",
                       "labels_total": labels_total,
                       "parallelism": f"label-shards{world} (all-reduce of dX)" if world > 1 else "single"},
            "tflops": step_roof["tflops"], "step_roofline": step_roof, "roofline": roof,
            "kernels": classes, "kernels_pass_ms_per_step": kernels_pass_ms, "gpu_launches": gpu_launches, "e2e": e2e, "cpu_baseline": cpu,
            "clocks": clocks, "peak_device_bytes": int(peak_mem),
        }
        print(json.dumps(line), flush=True)
    head.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
