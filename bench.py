#!/usr/bin/env python
"""Throughput of exact attention forward + backward on B200, through the C ABI.

One step = one pass of the whole hot path over one batch: the forward kernel
(O, L) and the three backward kernels (preprocess, dK/dV with atomic dQ, dQ
conversion) on the workload B=2, H=32, N=8192, d=128, bf16, causal (the ~8k-token
case of 64 M scores per head). Inputs are seeded synthetic iid N(0,1) values already
resident in HBM when the timed region starts; Q, K, V, dO are 134 MB each, larger
than the 126 MB L2, so no flush is needed between steps.

Prints ONE JSON line on rank 0. --impl reference times the fp64 CPU oracle on a
bounded sample of the same workload instead (the oracle is the only reference this
method has).

Launch: python bench.py [--gpus N --steps K --warmup W]; for N > 1 under
torch.distributed.run (one process per GPU, each an independent replica: the
attention problems are independent, so there is no data-path collective).
"""

from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from exact_io_aware_69_b200.inputs import WORKLOADS, sweep_workloads  # noqa: E402

METRIC = "attention TFLOP/s fwd & fwd+bwd (bf16, causal/non) and % of tensor-core peak"
UNIT = "TFLOP/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c3", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads, the small-call latency and the memory fit")
    return ap.parse_args()


def flops(w):
    """(fwd, bwd) algorithmic FLOPs: fwd 4*B*H*N^2*d (halved for causal), bwd 2.5 x fwd."""
    f = w.fwd_flops()
    return f, 2.5 * f


def config_of(w):
    return {
        "workload": f"B{w.B} H{w.H} N{w.N} d{w.d} {w.dtype} {'causal' if w.causal else 'non-causal'}"
                    " exact attention fwd+bwd",
        "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "scale": "1/sqrt(d)",
        "l2": "inputs larger than L2 (Q, K, V, dO %.0f MB each > 126 MB), no flush"
              % (w.B * w.H * w.N * w.d * 2 / 1e6),
        "flop_convention": "fwd = 4*B*H*N^2*d, halved for causal; value = fwd+bwd counted as "
                           "2.5 x fwd as the target states; 'fwd_bwd_tflops_3p5x' counts the "
                           "five backward GEMMs too (3.5 x fwd)",
        "parallelism": "replicas (one independent problem per GPU)",
    }


def load_peaks():
    try:
        with open(PEAKS_FILE) as fh:
            p = json.load(fh)
        return p, "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "exact_io_aware_69_b200", "csrc", "*"))):
        with open(p, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches this source."""
    try:
        with open(TRAFFIC_FILE) as fh:
            t = json.load(fh)
    except OSError:
        return None
    e = t.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash() or e.get("workload") != workload:
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while the timed region runs. Every
    sample carries nvidia-smi's timestamp; only those between mark_start() and mark_end()
    (host times taken right after the synchronizes that open and close the timed region)
    enter the result, so that the idle moments around the region do not."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.window = None
        self.out = os.path.join("/tmp", f"fa_clocks_{os.getpid()}.csv")
        self.sel = []
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.fh = open(self.out, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def mark_start(self):
        self.window = [time.time(), None]

    def mark_end(self):
        if self.window is not None:
            self.window[1] = time.time()

    @staticmethod
    def parse(lines, window=None):
        """(seconds since the epoch, SM MHz, max SM MHz, active reasons) per sample line,
        keeping the samples inside `window` = (t0, t1) when one is given."""
        import datetime
        out = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            t = None
            for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
                try:
                    t = datetime.datetime.strptime(parts[0], fmt).timestamp()
                    break
                except ValueError:
                    pass
            if window is not None and (t is None or not window[0] <= t <= window[1]):
                continue
            out.append((t, sm, mx, [n for n, v in zip(ClockSampler.REASONS, parts[5:9])
                                    if v.lower().startswith("active")]))
        return out

    @staticmethod
    def summarise(samples, in_window):
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [x[1] for x in samples]
        # outside a marked window, the samples under load: the top part of the distribution
        hi = sm if in_window else [v for v in sm if v >= 0.5 * max(sm)]
        return {"sm_mhz": statistics.median(hi), "sm_min_mhz": min(hi),
                "sm_max_mhz": max(x[2] for x in samples),
                "reasons": sorted({r for x in samples for r in x[3]}), "samples": len(sm),
                "window": "timed region" if in_window else "whole sampling period"}

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        with open(self.out) as fh:
            lines = fh.readlines()
        os.unlink(self.out)
        if self.window is not None and self.window[1] is not None:
            inside = self.parse(lines, self.window)
            if inside:
                return self.summarise(inside, True)
        return self.summarise(self.parse(lines), False)


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(world, flops_per_rank_step, steps, max_ms):
    """Whole-job rate: the work of all ranks over the slowest rank's time (TFLOP/s)."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


def torch_inputs(w, dev, seed):
    """Seeded iid N(0,1) inputs of workload w drawn on the device, for the timing-only
    runs: torch's generator, rounded to the 16-bit type; w's large-logit rows (floor(
    frac * N) distinct rows per head, x8) are chosen with the same generator."""
    import torch
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    shape = (w.B, w.H, w.N, w.d)
    out = [torch.randn(shape, generator=g, device=dev, dtype=torch.float32) for _ in range(4)]
    if w.large_frac > 0:
        n_large = int(math.floor(w.large_frac * w.N))
        qf = out[0].view(w.B * w.H, w.N, w.d)
        for bh in range(w.B * w.H):
            rows = torch.randperm(w.N, generator=g, device=dev)[:n_large]
            qf[bh, rows] *= 8.0
    return [t.to(tdt) for t in out]


def visible_pairs(Nq, Nk, window):
    """(query, key) pairs inside the (left, right) key window (negative = unbounded),
    bottom-right aligned: the algorithmic FLOP count of a windowed pass is 4 d per pair
    forward."""
    off = Nk - Nq
    i = np.arange(Nq, dtype=np.int64)
    lo = np.zeros(Nq, np.int64) if window[0] < 0 else np.maximum(0, i + off - window[0])
    hi = np.full(Nq, Nk - 1, np.int64) if window[1] < 0 else np.minimum(Nk - 1, i + off + window[1])
    return int(np.maximum(0, hi - lo + 1).sum())


def time_workload(fa, w, dev, stream, steps, warmup, peak_burst, window=None, layout="bhnd",
                  deterministic=False):
    """Device time per step of the forward and the three backward kernels of workload
    w (CUDA events on the launching stream), and the rates they give. `window`
    replaces w's causal flag by a key window (FLOPs counted over the visible pairs)."""
    import torch
    q, k, v, do = torch_inputs(w, dev, w.seed)
    if layout == "bnhd":
        q, k, v, do = (t.transpose(1, 2).contiguous() for t in (q, k, v, do))
    o, o_res = torch.empty_like(q), torch.empty_like(q)
    L = torch.empty((w.B, w.H, w.N), device=dev, dtype=torch.float32)
    dq, dk, dvv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.workspace_size(w.B, w.H, w.N, w.d, deterministic=deterministic),
                     device=dev, dtype=torch.uint8)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    mask = dict(causal=w.causal, window=window, layout=layout)

    def step(rec):
        if rec:
            ev[0].record(stream)
        fa.forward(q, k, v, scale=w.scale, out=o, lse=L, out_res=o_res, stream=stream, **mask)
        if rec:
            ev[1].record(stream)
        fa.backward(q, k, v, o, L, do, scale=w.scale, o_res=o_res, workspace=ws, dq=dq, dk=dk,
                    dv=dvv, stream=stream, deterministic=deterministic, **mask)
        if rec:
            ev[2].record(stream)

    for _ in range(warmup):
        step(False)
    fwd_ms = bwd_ms = 0.0
    for _ in range(steps):
        step(True)
        ev[2].synchronize()
        fwd_ms += ev[0].elapsed_time(ev[1])
        bwd_ms += ev[1].elapsed_time(ev[2])
    st = fa.device_status()
    if st != fa.FA_OK:
        raise RuntimeError(f"device status {st} in {w.name}")
    fwd_ms /= steps
    bwd_ms /= steps
    f, b = flops(w)
    if window is not None:
        f = 4.0 * w.B * w.H * w.d * visible_pairs(w.N, w.N, window)
        b = 2.5 * f
    r = {"fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
         "fwd_tflops": round(f / fwd_ms / 1e9, 1), "bwd_tflops": round(b / bwd_ms / 1e9, 1),
         "fwd_bwd_tflops_2p5x": round(2.5 * f / (fwd_ms + bwd_ms) / 1e9, 1),
         "fwd_bwd_tflops_3p5x": round((f + b) / (fwd_ms + bwd_ms) / 1e9, 1)}
    r["frac_3p5x_of_burst"] = round(r["fwd_bwd_tflops_3p5x"] / peak_burst, 3)
    return r


def time_forward(fa, w, dev, stream, steps, warmup, peak_burst):
    """Device time per forward of workload w alone (for head dimensions the backward does
    not take), CUDA events on the launching stream."""
    import torch
    q, k, v, _ = torch_inputs(w, dev, w.seed)
    o, o_res = torch.empty_like(q), torch.empty_like(q)
    L = torch.empty((w.B, w.H, w.N), device=dev, dtype=torch.float32)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(warmup):
        fa.forward(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=L, out_res=o_res,
                   stream=stream)
    e0.record(stream)
    for _ in range(steps):
        fa.forward(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=L, out_res=o_res,
                   stream=stream)
    e1.record(stream)
    e1.synchronize()
    st = fa.device_status()
    if st != fa.FA_OK:
        raise RuntimeError(f"device status {st} in {w.name}")
    ms = e0.elapsed_time(e1) / steps
    f, _ = flops(w)
    return {"fwd_ms": round(ms, 4), "fwd_tflops": round(f / ms / 1e9, 1),
            "frac_of_burst": round(f / ms / 1e9 / peak_burst, 3)}


def time_decode(fa, B, H, Nq, Nk, d, dev, stream, steps, warmup, hbm_peak):
    """The split-KV decode path: Nq rows per head against Nk keys, causal. Its bound is
    HBM: K and V are read once (plus Q, O, L), so the rate is reported in GB/s."""
    import torch
    w = type(WORKLOADS["c4"])(f"decode Nq{Nq} Nk{Nk}", B, H, Nk, d, "bf16", True, 9000 + Nq)
    _, k, v, _ = torch_inputs(w, dev, w.seed)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 1)
    q = torch.randn((B, H, Nq, d), generator=g, device=dev).to(torch.bfloat16)
    o = torch.empty_like(q)
    L = torch.empty((B, H, Nq), device=dev, dtype=torch.float32)
    need = int(fa.load().fa_decode_workspace_size(B, H, Nq, Nk, d, -1, 0))
    ws = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(warmup):
        fa.decode(q, k, v, causal=True, out=o, lse=L, workspace=ws, stream=stream)
    e0.record(stream)
    for _ in range(steps):
        fa.decode(q, k, v, causal=True, out=o, lse=L, workspace=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    st = fa.device_status()
    if st != fa.FA_OK:
        raise RuntimeError(f"device status {st} in decode")
    ms = e0.elapsed_time(e1) / steps
    kv_bytes = 2 * B * H * Nk * d * 2
    all_bytes = kv_bytes + 2 * B * H * Nq * d * 2 + B * H * Nq * 4
    flops_ = 4.0 * B * H * d * visible_pairs(Nq, Nk, (-1, 0))
    return {"shape": f"B{B} H{H} Nq{Nq} Nk{Nk} d{d} bf16 causal", "ms": round(ms, 4),
            "kv_gbs": round(kv_bytes / ms / 1e6, 1), "hbm_gbs": round(all_bytes / ms / 1e6, 1),
            "frac_of_hbm_peak": round(all_bytes / ms / 1e6 / hbm_peak, 3),
            "tflops": round(flops_ / ms / 1e9, 2), "splits_workspace_bytes": need}


def small_call_latency(fa, dev, stream, iters=200):
    """Config 1 (B1 H1 N256 d64): device time and host wall time of one forward +
    backward through the binding, and the host cost of enqueueing each call."""
    import torch
    w = WORKLOADS["c1"]
    q, k, v, do = torch_inputs(w, dev, w.seed)
    o, o_res = torch.empty_like(q), torch.empty_like(q)
    L = torch.empty((w.B, w.H, w.N), device=dev, dtype=torch.float32)
    dq, dk, dvv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.workspace_size(w.B, w.H, w.N, w.d), device=dev, dtype=torch.uint8)

    def fwd():
        fa.forward(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=L, out_res=o_res,
                   stream=stream)

    def bwd():
        fa.backward(q, k, v, o, L, do, causal=w.causal, scale=w.scale, o_res=o_res,
                    workspace=ws, dq=dq, dk=dk, dv=dvv, stream=stream)

    for _ in range(20):
        fwd()
        bwd()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    e0.record(stream)
    for _ in range(iters):
        fwd()
        bwd()
    e1.record(stream)
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) / iters * 1e6
    dev_us = e0.elapsed_time(e1) / iters * 1e3
    enq_f, enq_b = [], []
    for _ in range(50):
        t = time.perf_counter()
        fwd()
        enq_f.append(time.perf_counter() - t)
        t = time.perf_counter()
        bwd()
        enq_b.append(time.perf_counter() - t)
        torch.cuda.synchronize()
    return {"workload": "c1 B1 H1 N256 d64 bf16 non-causal", "iters": iters,
            "device_us_per_fwd_bwd": round(dev_us, 2),
            "host_wall_us_per_fwd_bwd": round(wall, 2),
            "host_enqueue_us": {"forward": round(statistics.median(enq_f) * 1e6, 2),
                                "backward": round(statistics.median(enq_b) * 1e6, 2)},
            "note": "back-to-back calls through the Python binding; wall time includes the "
                    "binding's marshalling and the C ABI's argument checks and tensor maps"}


def linear_fit(xs, ys):
    """Least squares y = a + b x: (slope b, intercept a, R^2)."""
    x = np.asarray(xs, np.float64)
    y = np.asarray(ys, np.float64)
    b, a = np.polyfit(x, y, 1)
    res = y - (a + b * x)
    tot = y - y.mean()
    return float(b), float(a), float(1.0 - (res @ res) / (tot @ tot))


def peak_memory_vs_n(fa, dev, stream, ns=(1024, 2048, 4096, 8192, 16384, 32768, 65536)):
    """Peak device memory of one forward + backward (inputs, outputs, workspace) at
    B1 H16 d128 bf16 causal for each N, and a linear fit against N."""
    import torch
    peaks = []
    for N in ns:
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        base = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        w = type(WORKLOADS["c4"])(f"mem N{N}", 1, 16, N, 128, "bf16", True, 7000 + N)
        q, k, v, do = torch_inputs(w, dev, w.seed)
        o, L, o_res = fa.forward(q, k, v, causal=True, scale=w.scale, stream=stream)
        dq, dk, dvv = fa.backward(q, k, v, o, L, do, causal=True, scale=w.scale, o_res=o_res,
                                  stream=stream)
        torch.cuda.synchronize()
        peaks.append(int(torch.cuda.max_memory_allocated() - base))
        del q, k, v, do, o, L, o_res, dq, dk, dvv
    slope, icpt, r2 = linear_fit(ns, peaks)
    return {"shape": "B1 H16 d128 bf16 causal, fwd + bwd through the binding",
            "N": list(ns), "peak_bytes": peaks, "slope_bytes_per_N": round(slope, 1),
            "intercept_bytes": round(icpt, 1), "r2": r2}


def run_reference(args, w, rank):
    """The oracle as it stands, timed on this host's cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    inp = w.make()
    d = w.d
    BH = w.B * w.H
    sample_heads = [0]
    qf, kf, vf, df = (inp.widened(n).reshape(BH, w.N, d)[sample_heads].astype(np.float64)
                      for n in ("q", "k", "v", "do"))
    fwd_f, bwd_f = flops(w)
    step_flops = 2.5 * fwd_f / BH * len(sample_heads)
    for _ in range(args.warmup):
        oracle.attn_bwd(qf, kf, vf, df, w.causal, w.scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attn_bwd(qf, kf, vf, df, w.causal, w.scale)
    dt = time.perf_counter() - t0
    value = step_flops * args.steps / dt / 1e12
    cores = oracle.num_threads()
    sample = f"head 0 of {BH} (fwd+bwd, all {w.N} rows) per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded iid N(0,1), rounded to bf16)", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_and_parity(w, inp, outs, target_s):
    """Time the oracle on whole heads until ~target_s of CPU work; check the GPU's
    outputs for those heads against it."""
    import oracle
    BH, N, d = w.B * w.H, w.N, w.d
    fwd_f, bwd_f = flops(w)
    per_head = 2.5 * fwd_f / BH
    q, k, v, do = (inp.widened(n).reshape(BH, N, d) for n in ("q", "k", "v", "do"))
    heads, elapsed = [], 0.0
    worst = {}
    order = [0, BH - 1] + list(range(1, BH - 1))
    while elapsed < target_s and len(heads) < BH:
        h = order[len(heads)]
        args = [x[h:h + 1].astype(np.float64) for x in (q, k, v, do)]
        t0 = time.perf_counter()
        ref = oracle.attn_bwd(*args, w.causal, w.scale)
        elapsed += time.perf_counter() - t0
        heads.append(h)
        for name in ("o", "dq", "dk", "dv"):
            got = outs[name].reshape(BH, N, d)[h].astype(np.float64)
            diff = np.abs(got - ref[name][0])
            rel = float((diff / np.maximum(1.0, np.abs(ref[name][0]))).max())
            cur = worst.get(name, (0.0, 0.0, 0.0))
            worst[name] = (max(cur[0], float(diff.max())), max(cur[1], rel),
                           max(cur[2], float(diff.mean())))
        dl = float(np.abs(outs["L"].reshape(BH, N)[h] - ref["L"][0]).max())
        worst["L"] = (max(worst.get("L", (0.0,))[0], dl), 0.0, 0.0)
    tol_max, tol_mean = (2e-2, 2e-3) if w.dtype == "bf16" else (5e-3, 5e-4)
    # the literal max-abs bar; the relative reading (|got-ref|/max(1,|ref|)) only for the
    # large-logit workload, whose x8 rows have gradients of magnitude ~10
    relative = w.large_frac > 0
    kmax = 1 if relative else 0
    ok = all(worst[n][kmax] <= tol_max and worst[n][2] <= tol_mean for n in ("o", "dq", "dk", "dv"))
    ok = ok and worst["L"][0] <= 1e-3
    base = {"value": per_head * len(heads) / elapsed / 1e12, "unit": UNIT,
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(heads)} of {BH} heads (fwd+bwd, all {N} rows each), "
                      f"{elapsed:.1f} s of fp64 CPU work"}
    parity = {"heads_checked": heads, "ok": bool(ok),
              "max_abs_err": {n: round(worst[n][0], 6) for n in worst},
              "max_rel_err": {n: round(worst[n][1], 6) for n in ("o", "dq", "dk", "dv")},
              "mean_abs_err": {n: round(worst[n][2], 7) for n in ("o", "dq", "dk", "dv")},
              "reading": ("max |got-ref|/max(1,|ref|)" if relative else "max |got-ref|")
              + f" vs {tol_max:g}, mean |got-ref| vs {tol_mean:g}, L abs 1e-3"}
    return base, parity


def main():
    args = parse_args()
    w = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, w, rank)
        return

    import torch
    from exact_io_aware_69_b200 import fa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
        pg = dist

    fa.load()
    stream = torch.cuda.current_stream()
    B, H, N, d = w.B, w.H, w.N, w.d
    inp = w.make()
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16

    def pinned(bits):
        t = torch.from_numpy(bits.view(np.int16)).view(tdt)
        return t.pin_memory()

    h_in = {n: pinned(getattr(inp, n)) for n in ("q", "k", "v", "do")}
    dv_in = {n: t.to(dev) for n, t in h_in.items()}
    q, k, v, do = dv_in["q"], dv_in["k"], dv_in["v"], dv_in["do"]
    o = torch.empty_like(q)
    o_res = torch.empty_like(q)
    L = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    dq, dk, dvv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.workspace_size(B, H, N, d), device=dev, dtype=torch.uint8)
    scale = w.scale

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fa.forward(q, k, v, causal=w.causal, scale=scale, out=o, lse=L, out_res=o_res,
                   stream=stream)
        if ev is not None:
            ev[1].record(stream)
        fa.backward_stage("preprocess", q, k, v, o, L, do, dq, dk, dvv, ws, w.causal, scale,
                          o_res, stream)
        if ev is not None:
            ev[2].record(stream)
        fa.backward_stage("dkdv", q, k, v, o, L, do, dq, dk, dvv, ws, w.causal, scale, o_res,
                          stream)
        if ev is not None:
            ev[3].record(stream)
        fa.backward_stage("dq_convert", q, k, v, o, L, do, dq, dk, dvv, ws, w.causal, scale,
                          o_res, stream)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    st = fa.device_status()
    if st != fa.FA_OK:
        raise RuntimeError(f"device status {st} after warm-up")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    sampler.start()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    sampler.mark_start()
    t_start.record(stream)
    for s in range(args.steps):
        step(events[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark_end()
    if pg:
        pg.barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    per_kernel = {"fa_fwd_pp_kernel": 0.0, "fa_bwd_pre_kernel": 0.0, "fa_bwd_main_kernel": 0.0,
                  "fa_bwd_dq_kernel": 0.0}
    names = list(per_kernel)
    for ev in events:
        for i, n in enumerate(names):
            per_kernel[n] += ev[i].elapsed_time(ev[i + 1])
    red = max_over_ranks([total_ms] + [per_kernel[n] for n in names], pg, dev)
    total_ms = red[0]
    for i, n in enumerate(names):
        per_kernel[n] = red[1 + i]
    st = fa.device_status()
    if st != fa.FA_OK:
        raise RuntimeError(f"device status {st} after timing")

    fwd_f, bwd_f = flops(w)
    steps = args.steps
    ms_step = total_ms / steps
    # fwd+bwd counted as 2.5 x fwd, literally as the target states it
    value = job_throughput(world, 2.5 * fwd_f, steps, total_ms)
    fwd_ms = per_kernel["fa_fwd_pp_kernel"] / steps
    bwd_ms = sum(per_kernel[n] for n in names[1:]) / steps
    peaks, peak_kind = load_peaks()
    peak_burst = float(peaks["bf16_tflops"])
    peak_sus = float(peaks.get("bf16_tflops_sustained", peak_burst))

    # dominant kernel: the largest share of the step
    kflops = {"fa_fwd_pp_kernel": fwd_f, "fa_bwd_main_kernel": bwd_f}
    rows = B * H * N
    kbytes = {"fa_bwd_pre_kernel": rows * d * 2 * 3 + rows * 4 + rows * 8 + rows * d * 4,
              "fa_bwd_dq_kernel": rows * d * 4 + rows * d * 2}
    dom = max(per_kernel, key=per_kernel.get)
    dom_ms = per_kernel[dom] / steps
    # The timed region is a fraction of a second at full clock, so the denominator is
    # the burst peak (a kernel timed in a short loop); the sustained peak (seconds
    # under the power cap) is printed beside it for reference.
    if dom in kflops:
        achieved = kflops[dom] / (dom_ms * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak_burst,
                "unit": "TFLOP/s", "frac": achieved / peak_burst,
                "peak_kind": f"{peak_kind} bf16 burst (of measured cuBLAS; timed region "
                             f"{total_ms:.0f} ms)",
                "frac_of_sustained_peak": achieved / peak_sus,
                "algorithmic_per_launch": kflops[dom], "avg_launch_ms": dom_ms}
    else:
        achieved = kbytes[dom] / (dom_ms * 1e-3) / 1e9
        hbm = float(peaks["hbm_gbs"])
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_kind": f"{peak_kind} HBM copy",
                "algorithmic_per_launch": kbytes[dom], "avg_launch_ms": dom_ms}
    roof["traffic"] = recorded_traffic(dom, args.workload)

    kernels = {}
    for n in names:
        ms = per_kernel[n] / steps
        e = {"avg_ms": ms, "share": per_kernel[n] / sum(per_kernel.values())}
        if n in kflops:
            e["tflops"] = kflops[n] / (ms * 1e-3) / 1e12
            e["frac_of_burst_peak"] = e["tflops"] / peak_burst
        else:
            e["gbs"] = kbytes[n] / (ms * 1e-3) / 1e9
        kernels[n] = e

    # ---- end to end through the public API, host buffers, copies inside the timing.
    # Steps are pipelined the way a caller streaming batches would: step k+1's inputs go
    # up and step k-1's results come down while step k's kernels run (three streams,
    # device tensors double-buffered); every step's copies are inside the timed region.
    h_out = {n: torch.empty(q.shape, dtype=tdt).pin_memory() for n in ("o", "dq", "dk", "dv")}
    h_L = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = sum(t.numel() * t.element_size() for t in h_out.values()) + h_L.numel() * 4
    bufs = [dict(inp=dv_in, o=o, o_res=o_res, L=L, dq=dq, dk=dk, dv=dvv, ws=ws)]
    if args.e2e_steps > 1:
        bufs.append(dict(inp={n: torch.empty_like(t) for n, t in dv_in.items()},
                         o=torch.empty_like(q), o_res=torch.empty_like(q), L=torch.empty_like(L),
                         dq=torch.empty_like(q), dk=torch.empty_like(q), dv=torch.empty_like(q),
                         ws=torch.empty_like(ws)))
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in bufs]
    ev_comp = [torch.cuda.Event() for _ in bufs]
    ev_out = [torch.cuda.Event() for _ in bufs]
    used = [False] * len(bufs)

    def e2e_step(k):
        b = k % len(bufs)
        x = bufs[b]
        if used[b]:
            s_in.wait_event(ev_comp[b])    # step k-2's kernels have read these inputs
            s_comp.wait_event(ev_out[b])   # ... and its results have left the device
        with torch.cuda.stream(s_in):
            for n in ("q", "k", "v", "do"):
                x["inp"][n].copy_(h_in[n], non_blocking=True)
            ev_in[b].record(s_in)
        s_comp.wait_event(ev_in[b])
        qq, kk, vv, dd = (x["inp"][n] for n in ("q", "k", "v", "do"))
        fa.forward(qq, kk, vv, causal=w.causal, scale=scale, out=x["o"], lse=x["L"],
                   out_res=x["o_res"], stream=s_comp)
        fa.backward(qq, kk, vv, x["o"], x["L"], dd, causal=w.causal, scale=scale,
                    o_res=x["o_res"], workspace=x["ws"], dq=x["dq"], dk=x["dk"], dv=x["dv"],
                    stream=s_comp)
        ev_comp[b].record(s_comp)
        s_out.wait_event(ev_comp[b])
        with torch.cuda.stream(s_out):
            for n in ("o", "dq", "dk", "dv"):
                h_out[n].copy_(x[n], non_blocking=True)
            h_L.copy_(x["L"], non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    if args.e2e_steps <= 0:
        e2e_ms = float("nan")
    else:
        e2e_step(0)
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    if args.e2e_steps > 0:
        e0.record(s_in)
        for k in range(args.e2e_steps):
            e2e_step(k)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks([e2e_ms], pg, dev)[0]
    e2e_val = job_throughput(world, 2.5 * fwd_f, args.e2e_steps, e2e_ms)

    extras = {}
    if rank == 0 and not args.no_extras:
        # the metric's other named workloads (fwd and fwd+bwd, causal and not, fp16, d=64)
        by_w = {}
        for name in ("c2", "c2c", "c4"):
            by_w[WORKLOADS[name].name] = time_workload(fa, WORKLOADS[name], dev, stream, 5, 3,
                                                       peak_burst)
        for sw in sweep_workloads():
            by_w[sw.name] = time_workload(fa, sw, dev, stream, 5, 3, peak_burst)
        # the rows beyond the basic calls, on the headline shape
        c3 = WORKLOADS["c3"]
        by_w["c3 sliding window (1024, 0)"] = time_workload(fa, c3, dev, stream, 5, 3, peak_burst,
                                                            window=(1024, 0))
        by_w["c3 [B,N,H,d] layout"] = time_workload(fa, c3, dev, stream, 5, 3, peak_burst,
                                                    layout="bnhd")
        by_w["c3 deterministic backward"] = time_workload(fa, c3, dev, stream, 5, 3, peak_burst,
                                                          deterministic=True)
        # head dimension 256 (forward only)
        for causal in (True, False):
            w256 = type(c3)(f"B2 H16 N8192 d256 bf16 {'causal' if causal else 'non-causal'}, "
                            "forward only", 2, 16, 8192, 256, "bf16", causal, 8256 + causal)
            by_w[w256.name] = time_forward(fa, w256, dev, stream, 5, 3, peak_burst)
        extras["by_workload"] = by_w
        hbm = float(peaks["hbm_gbs"])
        extras["decode"] = [time_decode(fa, 4, 32, nq, 65536, 128, dev, stream, 10, 3, hbm)
                            for nq in (1, 2, 4, 8, 16)]
        extras["latency_small"] = small_call_latency(fa, dev, stream)
        extras["peak_memory"] = peak_memory_vs_n(fa, dev, stream)
        torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp16",
        "data": "synthetic (seeded iid N(0,1), rounded to 16 bit)", "config": config_of(w),
        "fwd_tflops": fwd_f / (fwd_ms * 1e-3) / 1e12,
        "bwd_tflops": bwd_f / (bwd_ms * 1e-3) / 1e12,
        "fwd_bwd_tflops_3p5x": job_throughput(world, fwd_f + bwd_f, steps, total_ms),
        "pct_of_peak": {"fwd": fwd_f / (fwd_ms * 1e-3) / 1e12 / peak_burst,
                        "fwd_bwd_2p5x": value / world / peak_burst,
                        "fwd_bwd_3p5x": (fwd_f + bwd_f) / (ms_step * 1e-3) / 1e12 / peak_burst,
                        "peak": peak_burst, "peak_kind": f"{peak_kind} bf16 burst",
                        "sustained_peak": peak_sus},
        "kernels": kernels,
        "roofline": roof,
        "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "api": "fa.forward + fa.backward (C ABI) with pinned host buffers; copies of "
                       "neighbouring steps overlap each step's kernels (3 streams, 2 device "
                       "buffer sets)"},
        "gpu_launches": 4 * steps,
        "clocks": clocks,
    }
    line.update(extras)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        outs = {"o": o.float().cpu().numpy(), "dq": dq.float().cpu().numpy(),
                "dk": dk.float().cpu().numpy(), "dv": dvv.float().cpu().numpy(),
                "L": L.cpu().numpy()}
        base, parity = cpu_baseline_and_parity(w, inp, outs, args.cpu_seconds)
        line["cpu_baseline"] = base
        line["parity"] = parity
        if not parity["ok"]:
            log(json.dumps(line))
            raise SystemExit("parity check of the timed outputs against the oracle FAILED")
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
