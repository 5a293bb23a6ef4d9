#!/usr/bin/env python
"""GCA hot-path benchmark: frames/sec per layer at T=10000 on the 518x378
workload (M=999 image + 6 summary tokens, n=3 anchors, k=64 window, H=16,
D=64, 24 layers, bf16), and the attention kernel's share of the bf16 tensor
peak.

One step = one new frame through the whole hot path: append its K/V for all
24 layers (one launch), evict the frame that left the window, then GCA
attention for each of the 24 layers.  Timed steps are frames 10000-K..9999, so
the last timed step is at T=10000.  Inputs (seeded synthetic streams) are
resident in HBM before timing; the end-to-end figure repeats steps with pinned
host buffers through the same C ABI.

--impl reference times the CPU oracle (oracle/) on the host cores on a bounded
sample of the same workload (rank 0 only).

Multi-GPU: one independent stream per rank (seeded by rank), no collective on
the data path (weak scaling); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from windowed_memory_attention_b200 import gca, inputs  # noqa: E402

METRIC = "GCA frames/sec per layer at T=10000 (M=999,n=3,k=64) and % of BF16 TC peak"
UNIT = "frames/s/layer"
ATTEND_SRC = os.path.join(ROOT, "windowed_memory_attention_b200", "csrc", "attend_sm100.cu")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the layer count (profiling captures of a smaller case)")
    ap.add_argument("--report", action="store_true",
                    help="instead of the bench line: per-layer attention / append timings of "
                         "the worked-example stream at T=100/1000/10000, the dense causal "
                         "limit at T=1000 and the whole windowed-VO stream, one JSON line each")
    ap.add_argument("--vo", action="store_true",
                    help="instead of the bench line: only the windowed-VO stream's frames/s")
    ap.add_argument("--report-oracle", action="store_true",
                    help="instead of the bench line: the CPU oracle's time per layer-step at the "
                         "report points (worked example and 518x378 at T=100/1000/10000, dense "
                         "limit at T=1000) on the host cores; no GPU work")
    ap.add_argument("--frame-probe", type=int, default=0, metavar="FRAMES",
                    help="instead of the bench line: intra-frame attention of the 518x378 workload, "
                         "FRAMES frames per gca_frame_attention_batch call, 5 calls; a small command "
                         "for profiler captures of the batched launch")
    ap.add_argument("--append-probe", type=int, default=0, metavar="FRAMES",
                    help="instead of the bench line: FRAMES appends of the 518x378 workload's 24 "
                         "layers into a small cache (window 4, about 1 GB of pools) with the append "
                         "timed; a small command for profiler captures of the append kernel")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"bf16": d["bf16_tflops"], "bf16_sustained": d.get("bf16_tflops_sustained"),
                "hbm": d["hbm_gbs"], "source": "measured"}
    except Exception:
        return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


def rank_workload(rank: int, layers=None):
    """The stream a rank runs: the metric workload seeded by the rank."""
    w = inputs.METRIC_518x378.with_(seed0=rank)
    if layers:
        w = w.with_(L=layers, name=f"{w.name}_layers{layers}")
    return w


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value over all ranks (time-like quantities: the job's time)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank: float, world: int, elapsed_ms: float) -> float:
    """Whole-job throughput: units all ranks processed / the max-over-ranks time."""
    return units_per_rank * world / (elapsed_ms / 1e3)


def lk_at(w, T):
    """Keys a single-frame query sees after T frames: M*min(T, n+k) + S*T."""
    return w.M * min(T, w.n + w.k) + w.S * T


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                self.samples.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4)
                          if s[4 + i].lower().startswith("active")})
        loaded = [x for x in sm if mx and x > 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples)}


def traffic_record():
    """dram bytes per attend launch from the committed ncu summary, if it was
    taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        src = hashlib.sha256(open(ATTEND_SRC, "rb").read()).hexdigest()
        if rec.get("source_sha256") == src:
            return rec
    except Exception:
        pass
    return None


# ----------------------------------------------------------------------------
# oracle sample (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------
class OracleSample:
    """Layer-0 keys of the step at T=10000, gathered for the CPU oracle."""

    def __init__(self, w):
        self.w = w
        self.summ_k, self.summ_v, self.full_k, self.full_v = {}, {}, {}, {}

    def keep_full(self, t, T):
        return t < self.w.n or t >= T - self.w.k

    def record(self, t, k, v, T):
        S = self.w.S
        self.summ_k[t] = k[0, :S].float().cpu().numpy()
        self.summ_v[t] = v[0, :S].float().cpu().numpy()
        if self.keep_full(t, T):
            self.full_k[t] = k[0].float().cpu().numpy()
            self.full_v[t] = v[0].float().cpu().numpy()

    def run(self, q0, last, rows):
        """Seconds of one oracle step on `rows`, and its estimate for all rows:
        (gather of the visible keys, attention of the sampled rows)."""
        from oracle import gca as ogca
        w = self.w

        def fkv(j, summary_only):
            if summary_only:
                return self.summ_k[j], self.summ_v[j]
            return self.full_k[j], self.full_v[j]
        t0 = time.perf_counter()
        kk, vv = ogca.gather_keys(last, fkv, n=w.n, k=w.k, S=w.S)
        t1 = time.perf_counter()
        self.last_out, _ = ogca.attention(q0[rows], kk, vv, w.softmax_scale)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1


# Query rows of layer 0 that one oracle sample computes: the same sample for the
# reference arm (once per step) and the repo arm's cpu_baseline (twice).
SAMPLE_ROWS = 384


def sample_rows(w):
    return list(range(min(SAMPLE_ROWS, w.Lq)))


# ----------------------------------------------------------------------------
def run_reference(args):
    """The CPU oracle as it stands, on the host cores (rank 0 only)."""
    from oracle import gca as ogca
    w = inputs.METRIC_518x378
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    T = w.T
    sample = OracleSample(w)
    # the synthetic stream is drawn on the GPU when there is one (data only)
    for t in range(T):
        k = inputs.draw(w, t, "k", dev)
        v = inputs.draw(w, t, "v", dev)
        sample.record(t, k, v, T)
    q0 = inputs.draw(w, T - 1, "q", dev)[0].float().cpu().numpy()
    rows = sample_rows(w)
    measured, full = [], []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        g, a = sample.run(q0, T - 1, rows)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            measured.append(dt)                        # wall time of the sample, as run
            full.append(g + a * w.Lq / len(rows))      # the same rate over all rows of the layer
    sample_s = sum(measured) / len(measured)
    layer_s = sum(full) / len(full)
    value = 1.0 / layer_s
    cores = ogca.core_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sample_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "S": w.S, "n": w.n, "k": w.k, "H": w.H,
                   "D": w.D, "layers": w.L, "T": T},
        "step": f"one oracle sample: key gather of layer 0 at T={T} + attention of {len(rows)} of "
                f"its {w.Lq} query rows x {w.H} heads; ms_per_step is its measured wall time",
        "extrapolated": {"ms_per_layer_step": layer_s * 1e3,
                         "ms_per_step_all_layers": layer_s * w.L * 1e3,
                         "note": "the sample's attention rate over all rows of one layer (the "
                                 "metric's unit, frames/s per layer) and over all layers"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{len(rows)} query rows x {w.H} heads of layer 0 at T={T} "
                                   f"(Lk={lk_at(w, T)}) per step: key gather + attention of "
                                   f"the sampled rows, scaled to all {w.Lq} rows"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    w = rank_workload(rank, args.layers)
    K, W = args.steps, args.warmup
    T_end = w.T
    n_pre = T_end - K - W
    assert n_pre > w.n + w.k, "too many steps for the stream length"
    E = max(0, args.e2e_steps)
    cache = gca.Cache.for_workload(w, max_frames=T_end + E + 2, device=local_rank)
    stream = torch.cuda.current_stream(dev)
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    sample = OracleSample(w) if want_cpu else None

    # ---- prefill (untimed): frames 0 .. n_pre-1
    for t in range(n_pre):
        k = inputs.draw(w, t, "k", dev)
        v = inputs.draw(w, t, "v", dev)
        cache.append(k, v)
        cache.evict()
        if sample:
            sample.record(t, k, v, T_end)
    # ---- inputs of the warm-up and timed steps, resident in HBM
    frames = []
    for t in range(n_pre, T_end):
        k = inputs.draw(w, t, "k", dev)
        v = inputs.draw(w, t, "v", dev)
        q = inputs.draw(w, t, "q", dev)
        frames.append((t, k, v, q))
        if sample:
            sample.record(t, k, v, T_end)
    out = torch.empty((w.L, 1, w.Lq, w.H, w.D), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize(dev)

    def ev():
        return torch.cuda.Event(enable_timing=True)
    att_ev = [[(ev(), ev()) for _ in range(w.L)] for _ in range(K)]
    app_ev = [(ev(), ev()) for _ in range(K)]

    def step(i, timed):
        t, k, v, q = frames[i]
        if timed:
            app_ev[i - W][0].record(stream)
        cache.append(k, v)
        if timed:
            app_ev[i - W][1].record(stream)
        cache.evict()
        for l in range(w.L):
            if timed:
                att_ev[i - W][l][0].record(stream)
            cache.attend(l, q[l:l + 1], out[l])
            if timed:
                att_ev[i - W][l][1].record(stream)

    for i in range(W):
        step(i, False)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local_rank)
    launches0 = cache.info().kernel_launches
    t0, t1 = ev(), ev()
    t0.record(stream)
    for i in range(W, W + K):
        step(i, True)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    launches = cache.info().kernel_launches - launches0
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = t0.elapsed_time(t1)
    if cache.status() != 0:
        raise RuntimeError(f"device status word raised: {cache.status()}")

    att_ms = [a.elapsed_time(b) for s in att_ev for (a, b) in s]
    app_ms = [a.elapsed_time(b) for (a, b) in app_ev]
    flops = sum(4.0 * w.Lq * lk_at(w, frames[i][0] + 1) * w.H * w.D
                for i in range(W, W + K)) * w.L
    att_total_s = sum(att_ms) / 1e3
    att_tflops = flops / att_total_s / 1e12
    app_bytes = 2 * 2 * w.L * w.Lq * w.H * w.D * 2     # K and V, read + write
    app_gbs = app_bytes / (statistics.mean(app_ms) / 1e3) / 1e9

    # ---- end-to-end: host (pinned) buffers through the same C ABI.  Every step
    # uploads its K/V (all layers) and q, and reads every layer's output back;
    # three pinned input sets are cycled (the copies do not depend on the values)
    e2e = None
    if E > 0:
        host = []
        for t in range(T_end, T_end + 3):
            host.append(tuple(inputs.draw(w, t, x, dev).cpu().pin_memory() for x in "kvq"))
        out_h = torch.empty((w.L, 1, w.Lq, w.H, w.D), dtype=torch.bfloat16).pin_memory()

        def hstep(j):
            k, v, q = host[j % len(host)]
            cache.append(k, v)
            cache.evict()
            for l in range(w.L):
                cache.attend(l, q[l:l + 1], out_h[l])

        hstep(0)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = ev(), ev()
        e0.record(stream)
        for j in range(1, E + 1):
            hstep(j)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        fb = w.L * w.Lq * w.H * w.D * 2
        e2e = {"value": job_value(E * w.L, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": 3 * fb, "d2h_bytes_per_step": fb}

    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)

    # ---- non-keyframe step (untimed above): the frame reads the cache and its
    # own tokens through gca_attend_transient and nothing is kept
    qn, kn, vn = (inputs.draw(w, T_end + E + 7, x, dev) for x in "qkv")
    outn = torch.empty((w.Lq, w.H, w.D), dtype=torch.bfloat16, device=dev)
    for l in range(w.L):
        cache.attend_transient(l, qn[l], kn[l], vn[l], outn)
    torch.cuda.synchronize(dev)
    nk_ev = [(ev(), ev()) for _ in range(w.L)]
    for l in range(w.L):
        nk_ev[l][0].record(stream)
        cache.attend_transient(l, qn[l], kn[l], vn[l], outn)
        nk_ev[l][1].record(stream)
    torch.cuda.synchronize(dev)
    nk_ms = statistics.mean(a.elapsed_time(b) for (a, b) in nk_ev)
    nk_keys = lk_at(w, cache.info().frames) + w.Lq
    nonkey = {"ms_per_layer": nk_ms, "frames_per_s_per_layer": 1e3 / nk_ms, "keys": nk_keys,
              "tflops": 4.0 * w.Lq * nk_keys * w.H * w.D / nk_ms / 1e9,
              "note": "gca_attend_transient per layer: the frame's K/V into transient pages, then "
                      "attention over the cache and the frame; page table unchanged"}
    if cache.status() != 0:
        raise RuntimeError(f"device status word raised: {cache.status()}")

    if rank != 0:
        return
    pk = peaks()
    tr = traffic_record()
    value = job_value(K * w.L, world, elapsed_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "S": w.S, "n": w.n, "k": w.k, "H": w.H,
                   "D": w.D, "layers": w.L, "T": T_end,
                   "step": "append all layers + evict + attend per layer",
                   "parallelism": f"independent stream per GPU x{world}",
                   "l2": "no flush: per-layer KV is 520 MB and one step reads 12.5 GB, both "
                         "larger than the 126 MB L2"},
        "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": pk["bf16"],
                     "unit": "TFLOP/s", "frac": att_tflops / pk["bf16"],
                     "traffic": tr["dram_bytes_per_launch"] if tr else None,
                     "kernel": "gca attend (tcgen05, split heads merged in the kernel), per layer launch",
                     "peak_source": f"{pk['source']} bf16 burst; sustained {pk['bf16_sustained']}",
                     "frac_of_sustained": att_tflops / pk["bf16_sustained"] if pk["bf16_sustained"] else None,
                     "algorithmic_flop_per_launch": flops / (K * w.L),
                     "avg_launch_ms": statistics.mean(att_ms)},
        "append_roofline": {"bound": "hbm", "achieved": app_gbs, "peak": pk["hbm"],
                            "unit": "GB/s", "frac": app_gbs / pk["hbm"],
                            "bytes_per_launch": app_bytes, "avg_launch_ms": statistics.mean(app_ms)},
        "nonkey_step": nonkey,
        "gpu_launches": int(launches),
        "clocks": clk,
        "e2e": e2e,
    }
    if sample:
        q0 = frames[-1][3][0].float().cpu().numpy()
        rows = sample_rows(w)
        runs = [sample.run(q0, T_end - 1, rows) for _ in range(2)]
        g = sum(r[0] for r in runs) / len(runs)
        a = sum(r[1] for r in runs) / len(runs)
        step_s = g + a * w.Lq / len(rows)
        # the same sample checks the timed step's output: layer 0 of frame T-1
        got = out[0, 0].double().cpu().numpy()[rows]
        line["parity"] = {"max_abs_err": float(np.abs(got - sample.last_out).max()), "tolerance": 2e-2,
                          "rows": len(rows), "heads": w.H, "layer": 0, "frame": T_end - 1,
                          "against": "CPU oracle (fp64) on the sampled rows"}
        from oracle import gca as ogca
        line["cpu_baseline"] = {
            "value": 1.0 / step_s, "unit": UNIT, "cores": ogca.core_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} query rows x {w.H} heads of layer 0 at T={T_end} "
                      f"(Lk={lk_at(w, T_end)}), run twice: key gather {g:.2f} s + attention "
                      f"{a:.2f} s per run, attention scaled to all {w.Lq} rows"}
    print(json.dumps(line), flush=True)
    cache.close()


def _time_ms(fn, reps=20, warm=3):
    """Device time per call: the calls are queued behind a ~5 ms spin kernel,
    so they run back to back however long the host takes to issue them (a
    microsecond-scale launch would otherwise time the host's call overhead)."""
    for _ in range(warm):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    torch.cuda._sleep(10_000_000)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def run_append_probe(args):
    """Append launches of the full 24-layer frame into a cache with a short window:
    the append's work per launch does not depend on the window, the pools do."""
    pk = peaks()
    dev = torch.device("cuda", 0)
    w = inputs.METRIC_518x378.with_(k=4)
    cache = gca.Cache.for_workload(w, max_frames=args.append_probe + 1)
    kv = [(inputs.draw(w, t, "k", dev), inputs.draw(w, t, "v", dev)) for t in range(4)]
    # back-to-back launches between two events: the host runs ahead of the GPU,
    # so the per-launch figure is the kernels' own time plus the launch gaps
    half = args.append_probe // 2
    for t in range(half):
        cache.append(*kv[t % 4])
        cache.evict()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for t in range(half, args.append_probe):
        cache.append(*kv[t % 4])
        cache.evict()
    e1.record()
    torch.cuda.synchronize()
    if cache.status() != 0:
        raise RuntimeError("device status word raised")
    med = e0.elapsed_time(e1) / (args.append_probe - half)
    b = 2 * 2 * w.L * w.Lq * w.H * w.D * 2
    print(json.dumps({"append_probe": w.name + " (window 4)", "frames": args.append_probe,
                      "us_per_launch": med * 1e3, "bytes_per_launch": b, "GBs": b / (med / 1e3) / 1e9,
                      "frac_hbm": b / (med / 1e3) / 1e9 / pk["hbm"]}), flush=True)


def run_frame_probe(args):
    """Batched intra-frame attention: 5 calls of FRAMES frames of one layer."""
    dev = torch.device("cuda", 0)
    w = inputs.METRIC_518x378.with_(L=1)
    F = args.frame_probe
    cache = gca.Cache.for_workload(w, max_frames=4)
    q, k, v = (torch.stack([inputs.draw(w, f, x, dev)[0] for f in range(F)]) for x in "qkv")
    out = torch.empty_like(q)
    ms = _time_ms(lambda: cache.frame_attention_batch(0, q, k, v, out), reps=2, warm=3)
    if cache.status() != 0:
        raise RuntimeError("device status word raised")
    fl = 4.0 * w.Lq * w.Lq * w.H * w.D * F
    print(json.dumps({"frame_probe": w.name, "frames": F, "ms_per_call": ms, "ms_per_frame": ms / F,
                      "tflops": fl / ms / 1e9}), flush=True)
    cache.close()


def run_oracle_report(args):
    """cpu_baseline of the report points: the oracle's attention core as it stands, on a bounded
    sample (64 query rows of one head) of each point's shape, scaled to all rows and heads.  The
    inputs are seeded random arrays of the point's shape: the core's time does not depend on the
    values.  The key gather of the bench line's cpu_baseline is not included."""
    from oracle import gca as ogca
    import numpy as np
    points = [(inputs.WORKED_EXAMPLE, T) for T in (100, 1000, 10000)] + \
             [(inputs.METRIC_518x378, T) for T in (100, 1000, 10000)] + [(inputs.DENSE_CAUSAL, 1000)]
    rows, heads = 64, 1
    cores = ogca.core_threads()
    rng = np.random.default_rng(0)
    for w, T in points:
        lk = lk_at(w, T)
        q = rng.standard_normal((rows, heads, w.D), dtype=np.float32)
        k = rng.standard_normal((lk, heads, w.D), dtype=np.float32)
        v = rng.standard_normal((lk, heads, w.D), dtype=np.float32)
        ogca.attention_c(q[:4], k, v, w.softmax_scale)          # warm the core once
        t0 = time.perf_counter()
        ogca.attention_c(q, k, v, w.softmax_scale)
        dt = time.perf_counter() - t0
        step_s = dt * (w.Lq / rows) * (w.H / heads)
        print(json.dumps({"workload": w.name, "T": T, "Lq": w.Lq, "Lk": lk,
                          "cpu_baseline": {"value": 1.0 / step_s, "unit": UNIT, "cores": cores,
                                           "kind": "oracle", "ms_per_layer": step_s * 1e3,
                                           "sample": f"{rows} query rows x {heads} head against all "
                                                     f"{lk} keys, seeded random inputs of the point's "
                                                     f"shape, scaled to {w.Lq} rows x {w.H} heads; "
                                                     f"key gather not included"}}), flush=True)


def run_report(args):
    """Attention and append timings per layer on the other workloads."""
    pk = peaks()
    dev = torch.device("cuda", 0)

    def emit(w, T, attend_ms, append_ms, note=""):
        lk = lk_at(w, T)
        fl = 4.0 * w.Lq * lk * w.H * w.D
        print(json.dumps({"workload": w.name, "T": T, "Lq": w.Lq, "Lk": lk,
                          "attend_ms": attend_ms, "append_ms_per_layer": append_ms,
                          "tflops": fl / attend_ms / 1e9, "frac_bf16_peak": fl / attend_ms / 1e9 / pk["bf16"],
                          "frames_per_s_per_layer": 1e3 / (attend_ms + append_ms), "note": note}),
              flush=True)

    def stream(w, T_points, max_frames):
        cache = gca.Cache.for_workload(w, max_frames=max_frames)
        out = torch.empty((1, w.Lq, w.H, w.D), dtype=torch.bfloat16, device=dev)
        for t in range(max(T_points)):
            k = inputs.draw(w, t, "k", dev)
            v = inputs.draw(w, t, "v", dev)
            if t + 1 in T_points:
                q = inputs.draw(w, t, "q", dev)
                # append time of this frame (one layer), then attention at T = t+1
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                torch.cuda._sleep(2_000_000)          # the append is queued before it runs
                e0.record()
                cache.append(k, v)
                e1.record()
                cache.evict()
                torch.cuda.synchronize()
                app = e0.elapsed_time(e1)
                att = _time_ms(lambda: cache.attend(0, q, out))
                emit(w, t + 1, att, app)
                # a non-keyframe at the same state: reads the cache and its own tokens
                qn, kn, vn = (inputs.draw(w, 10 ** 6 + t, x, dev)[0] for x in "qkv")
                outn = torch.empty((w.Lq, w.H, w.D), dtype=torch.bfloat16, device=dev)
                att_n = _time_ms(lambda: cache.attend_transient(0, qn, kn, vn, outn))
                lk = lk_at(w, t + 1) + w.Lq
                fl = 4.0 * w.Lq * lk * w.H * w.D
                print(json.dumps({"workload": w.name, "T": t + 1, "step": "non-keyframe",
                                  "Lk": lk, "ms_per_layer": att_n, "tflops": fl / att_n / 1e9,
                                  "frames_per_s_per_layer": 1e3 / att_n}), flush=True)
            else:
                cache.append(k, v)
                cache.evict()
        cache.close()

    # intra-frame attention of one 518x378 frame (the layers that alternate with GCA)
    w = inputs.METRIC_518x378.with_(L=1)
    cache = gca.Cache.for_workload(w, max_frames=4)
    qf, kf, vf = (inputs.draw(w, 3, x, dev)[0] for x in "qkv")
    outf = torch.empty_like(qf)
    att = _time_ms(lambda: cache.frame_attention(0, qf, kf, vf, outf))
    fl = 4.0 * w.Lq * w.Lq * w.H * w.D
    print(json.dumps({"workload": w.name + " (one frame)", "step": "intra-frame attention",
                      "Lq": w.Lq, "Lk": w.Lq, "ms_per_layer": att, "tflops": fl / att / 1e9,
                      "note": "one launch: the frame's K/V read in place by the attention kernel "
                              "(bf16, no RoPE); 4.1 GFLOP per layer"}),
          flush=True)
    # the same layer over 16 frames in one call (one launch: a CTA per frame, tile pair and head)
    Fb = 16
    qb, kb, vb = (torch.stack([inputs.draw(w, 3 + f, x, dev)[0] for f in range(Fb)]) for x in "qkv")
    outb = torch.empty_like(qb)
    att_b = _time_ms(lambda: cache.frame_attention_batch(0, qb, kb, vb, outb))
    print(json.dumps({"workload": w.name + f" ({Fb} frames, one call)", "step": "intra-frame attention, batched",
                      "frames": Fb, "ms_per_call": att_b, "ms_per_frame": att_b / Fb,
                      "tflops": Fb * fl / att_b / 1e9}), flush=True)
    cache.close()

    # trajectory-memory variants on the 518x378 workload (one layer) at T=10000
    for label, mode, n in (("camera token only", gca.GCA_MEMORY_CAMERA, None),
                           ("sliding window (no memory, no anchors)", gca.GCA_MEMORY_NONE, 0)):
        w = inputs.METRIC_518x378.with_(L=1) if n is None else inputs.METRIC_518x378.with_(L=1, n=n)
        cache = gca.Cache.for_workload(w, max_frames=w.T, trajectory_memory=mode)
        out = torch.empty((1, w.Lq, w.H, w.D), dtype=torch.bfloat16, device=dev)
        for t in range(w.T):
            cache.append(inputs.draw(w, t, "k", dev), inputs.draw(w, t, "v", dev))
            cache.evict()
        q = inputs.draw(w, w.T - 1, "q", dev)
        att = _time_ms(lambda: cache.attend(0, q, out))
        keys = cache.info().resident_tokens
        fl = 4.0 * w.Lq * keys * w.H * w.D
        print(json.dumps({"workload": w.name + " (layer 0 only)", "memory": label, "n": w.n, "T": w.T, "Lk": keys,
                          "attend_ms": att, "tflops": fl / att / 1e9,
                          "frac_bf16_peak": fl / att / 1e9 / pk["bf16"]}), flush=True)
        cache.close()

    stream(inputs.WORKED_EXAMPLE, {100, 1000, 10000}, 10000)
    # the 518x378 workload's layer at the same points (the bench line is its 24-layer T=10000 step)
    stream(inputs.METRIC_518x378.with_(L=1), {100, 1000, 10000}, 10000)
    stream(inputs.DENSE_CAUSAL, {1000}, 1000)
    run_vo_stream(dev)


def run_vo_stream(dev):
    """The windowed (VO) workload as defined: 179 windows of 128 frames
    overlapping by 16 over 20,000 frames, 22,848 frames processed, a reset at
    each window start; one layer.  Every frame is appended, the window's old
    frame evicted and the frame attended; the whole stream is timed with CUDA
    events.  Inputs cycle through 160 pre-drawn frames resident in HBM (the
    kernels' time does not depend on the values)."""
    vo = inputs.WINDOWED_VO
    wins = vo.windows()
    pool = [tuple(inputs.draw(vo, f, x, dev) for x in "kvq") for f in range(160)]
    cache = gca.Cache.for_workload(vo)
    out = torch.empty((1, vo.Lq, vo.H, vo.D), dtype=torch.bfloat16, device=dev)

    def window(start, ln):
        cache.reset()
        for t in range(ln):
            k, v, q = pool[(start + t) % len(pool)]
            cache.append(k, v)
            cache.evict()
            cache.attend(0, q, out)

    window(*wins[0])                                   # warm-up
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    frames = 0
    keys = 0
    for start, ln in wins:
        window(start, ln)
        frames += ln
        keys += sum(lk_at(vo, t + 1) for t in range(ln))
    e1.record()
    torch.cuda.synchronize()
    if cache.status() != 0:
        raise RuntimeError("device status word raised")
    ms = e0.elapsed_time(e1)
    fl = 4.0 * vo.Lq * keys * vo.H * vo.D
    print(json.dumps({"workload": vo.name, "windows": len(wins), "frames_processed": frames,
                      "ms_total": ms, "frames_per_s_per_layer": frames / (ms / 1e3),
                      "tflops_attention_incl_append": fl / ms / 1e9,
                      "note": "append + evict + attend per frame, one layer, reset at each window "
                              "start; CUDA events around the whole stream"}), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return
    if args.report_oracle:
        run_oracle_report(args)
        return
    torch.cuda.set_device(local_rank)
    if args.report:
        run_report(args)
        return
    if args.vo:
        run_vo_stream(torch.device("cuda", local_rank))
        return
    if args.frame_probe:
        run_frame_probe(args)
        return
    if args.append_probe:
        run_append_probe(args)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
