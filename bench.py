#!/usr/bin/env python
"""Benchmark of the Longformer sparse self-attention forward on B200.

One step = one full forward (prep, band rows, global rows) of the workload
on inputs already resident in HBM.  Steps are replayed from CUDA graphs over
rotating input sets whose total size exceeds twice the L2 cache, so every
step reads its q/k/v from DRAM.  Rank 0 prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (weak scaling): one process per GPU under torchrun; each rank runs
its own copy of the workload (every (b, h) is independent: no collective on
the data path); the time is the max over ranks (all_reduce MAX of the CUDA
event time), and the value is the work of all ranks over that time.

The reference arm (--impl reference) is the fp64 CPU oracle (oracle/), timed
on the host cores on a bounded sample of rows of the same workload.
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

from sparse_long_sequence_fwd_b200 import flops as flops_mod  # noqa: E402
from sparse_long_sequence_fwd_b200 import sharding, workloads  # noqa: E402

METRIC = "useful sparse-attn TFLOP/s & tokens/s at T=4096,w=513; % of bf16 TC peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=workloads.BASE.name, choices=sorted(workloads.BY_NAME))
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--backward-only", action="store_true",
                    help="time only lf_attn_bwd on --workload and print that entry (for profiling the backward)")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the QA, dilated, large, f16 base, d = 128 and BigBird workload entries")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(
        os.environ.get("LOCAL_RANK", "0"))


def workload_config(w, extra=None):
    cfg = {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "r": w.r, "w": w.w,
           "dil": sorted(set(int(x) for x in w.dil)), "scale": w.softmax_scale}
    if w.globals_per_b is not None:
        gl = sorted(set(w.globals_per_b[0]))
        cfg["global"] = gl if len(gl) <= 8 else "%d positions" % len(gl)
    if w.n_random_globals:
        cfg["global"] = "%d seeded positions incl. 0" % w.n_random_globals
    if w.pad_from is not None:
        cfg["pad_from"] = list(w.pad_from)
    if extra:
        cfg.update(extra)
    return cfg


def band_row_mask(w, inp):
    """Per (b, i): True where row i is not a global row (written by the band kernel)."""
    G = inp["global_idx"]
    m = np.ones((w.B, w.T), dtype=bool)
    if G is not None:
        for b in range(w.B):
            for g in set(G[b].tolist()):
                if 0 <= g < w.T:
                    m[b, g] = False
    return m


def split_flops(w, inp):
    """(total useful FLOPs, band-kernel FLOPs, global-row FLOPs, global-row algorithmic bytes)."""
    G = inp["global_idx"]
    pad = inp["key_pad_mask"]
    keep = band_row_mask(w, inp)
    total = band = 0
    gr_bytes = 0
    for b in range(w.B):
        Gb = None if G is None else G[b].numpy()
        pb = None if pad is None else pad[b].numpy()
        n_valid = w.T if pb is None else int((pb == 0).sum())
        n_gq = int((~keep[b]).sum())
        for h in range(w.H):
            cnt = flops_mod.row_key_counts(w.T, w.r, int(w.dil[h]), Gb, pb)
            if inp.get("rand_blocks") is not None:  # the BigBird variant's random keys
                cnt = cnt + flops_mod.rand_extra_counts(w.T, w.r, Gb, pb, inp["rand_blocks"][b, h].numpy())
            total += int(cnt.sum())
            band += int(cnt[keep[b]].sum())
            if n_gq:
                gr_bytes += 2 * n_valid * w.d * 2 + 2 * n_gq * w.d * 2
    f = 4.0 * w.d
    return f * total, f * band, f * (total - band), gr_bytes


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.rows = []
        self.proc = None
        self.gpu = gpu_index
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 10:
                self.rows.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=2)

    def summary(self, t0=None, t1=None):
        rows = self.rows
        inside = [r for r in rows if t0 is not None and t0 <= r[0] <= t1]
        use = inside if inside else rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1][2]) for r in use if num(r[1][2]) is not None]
        smax = [num(r[1][3]) for r in use if num(r[1][3]) is not None]
        power = [num(r[1][4]) for r in use if num(r[1][4]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in use for k in range(4) if r[1][6 + k].lower().startswith("active")})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None, "reasons": reasons, "samples": len(use),
                "window": "timed region" if inside else "whole measurement (timed region shorter than a sample)"}


def traffic_from_profile(kernel_file: str):
    """dram read+write bytes per launch of the band kernel from the committed ncu summary, if the kernel
    source still matches the hash recorded with it; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    src = open(os.path.join(ROOT, "sparse_long_sequence_fwd_b200", "csrc", kernel_file), "rb").read()
    if d.get("source_sha1") != hashlib.sha1(src).hexdigest():
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------- ours
class WorkloadRun:
    """One workload on one GPU: rotating input sets (together more than twice
    the L2 size, so every step reads q/k/v from DRAM), CUDA graphs of steps
    and of single stages, timed with CUDA events on the launching stream."""

    def __init__(self, w, torch, lf_attn, dev, stream, warmup):
        self.w, self.torch, self.lf_attn, self.stream = w, torch, lf_attn, stream
        self.inp = inp = workloads.make_inputs(w)
        self.total_f, self.band_f, self.gr_f, self.gr_bytes = split_flops(w, inp)
        props = torch.cuda.get_device_properties(dev)
        self.l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20)
        es = 4 if w.dtype == "f32" else 2
        self.set_bytes = 4 * w.B * w.H * w.T * w.d * es
        self.n_sets = max(2, math.ceil(2 * self.l2 / self.set_bytes) + 1)
        q0, k0, v0 = (inp[x].to(dev) for x in ("q", "k", "v"))
        self.sets = [(q0, k0, v0, torch.empty_like(q0))]
        for _ in range(self.n_sets - 1):
            self.sets.append((q0.clone(), k0.clone(), v0.clone(), torch.empty_like(q0)))
        self.gidx = inp["global_idx"].to(dev) if inp["global_idx"] is not None else None
        self.pad = inp["key_pad_mask"].to(dev) if inp["key_pad_mask"] is not None else None
        self.rnd = inp["rand_blocks"].to(dev) if inp.get("rand_blocks") is not None else None
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for i in range(max(warmup, 0)):
                self.call(i)
            self.launches_per_step = lf_attn.last_launch_count()
        torch.cuda.synchronize()

    def call(self, i, stages=7):
        q, k, v, o = self.sets[i % self.n_sets]
        self.lf_attn.fwd(q, k, v, self.w.r, dil=self.inp["dil"], global_idx=self.gidx, key_pad_mask=self.pad,
                         scale=self.w.softmax_scale, out=o, stages=stages, stream=self.stream,
                         rand_blocks=self.rnd)

    def capture(self, n, stages=7):
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g, stream=self.stream):
            for i in range(n):
                self.call(i, stages)
        return g

    def graphs(self, K, stages=7):
        S = min(self.n_sets, K) if K > 0 else self.n_sets
        return S, self.capture(S, stages), (self.capture(K % S, stages) if K % S else None)

    def replay(self, K, S, g_main, g_rem):
        for _ in range(K // S):
            g_main.replay()
        if g_rem is not None:
            g_rem.replay()

    def time_steps(self, K, stages=7, before=None, after=None):
        """ms for exactly K steps (one CUDA-event pair around them)."""
        torch = self.torch
        S, g_main, g_rem = self.graphs(K, stages)
        with torch.cuda.stream(self.stream):
            g_main.replay()
        torch.cuda.synchronize()
        if before:
            before()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            e0.record()
            self.replay(K, S, g_main, g_rem)
            e1.record()
        torch.cuda.synchronize()
        if after:
            after()
        return e0.elapsed_time(e1)

    def stage_us(self, stages, budget_s=0.3):
        """Mean µs of one stage of the forward alone (graph replays over the rotating sets)."""
        torch = self.torch
        with torch.cuda.stream(self.stream):
            self.call(0)  # prep state for the band / global-row stages
        torch.cuda.synchronize()
        one = self.time_steps(self.n_sets, stages) / self.n_sets
        reps = max(self.n_sets, int(budget_s / max(one * 1e-3, 1e-6)))
        return 1e3 * self.time_steps(reps, stages) / reps

    def summary(self, ms_per_step, peaks, world=1):
        w = self.w
        out = {"value": round(sharding.job_rate(self.total_f, world, ms_per_step * 1e-3) / 1e12, 3),
               "unit": "TFLOP/s", "ms_per_step": round(ms_per_step, 6),
               "tokens_per_s": round(sharding.job_rate(w.B * w.T, world, ms_per_step * 1e-3), 1),
               "useful_gflop_per_step": round(self.total_f / 1e9, 4)}
        if self.rnd is not None:  # the per-stage entry point has no random-block form: the step only
            out["stages"] = "not timed separately (random key blocks)"
            out["l2"] = "rotating %d input sets, %.0f MB > 2x L2 (%.0f MB)" % (
                self.n_sets, self.n_sets * self.set_bytes / 1e6, self.l2 / 1e6)
            return out
        band_us = self.stage_us(2)
        out.update({"band_tc_us": round(band_us, 2),
               "band_frac": round(self.band_f / (band_us * 1e-6) / 1e12 / peaks["bf16_tflops"], 4),
               "prep_us": round(self.stage_us(1), 2)})
        if self.gidx is not None:
            gr_us = self.stage_us(4)
            out["global_rows_us"] = round(gr_us, 2)
            out["global_rows_hbm_frac"] = round(self.gr_bytes / (gr_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)
        out["l2"] = "rotating %d input sets, %.0f MB > 2x L2 (%.0f MB)" % (
            self.n_sets, self.n_sets * self.set_bytes / 1e6, self.l2 / 1e6)
        return out


def backward_entry(w, torch, lf_attn, dev, stream, calls=5):
    """lf_attn_bwd on one workload: its time per call (CUDA events, after a warm-up call) and
    useful TFLOP/s counted as 2.5x the forward's useful FLOPs (dS recomputed from Q K^T: five
    products of 2 d FLOPs per kept (query, key) pair against the forward's two)."""
    inp = workloads.make_inputs(w)
    total_f = split_flops(w, inp)[0]
    g = torch.Generator().manual_seed(w.seed + 1)
    dy = torch.randn(inp["q"].shape, generator=g).to(inp["q"].dtype).to(dev)
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    G = inp["global_idx"].to(dev) if inp["global_idx"] is not None else None
    pad = inp["key_pad_mask"].to(dev) if inp["key_pad_mask"] is not None else None
    with torch.cuda.stream(stream):
        y = lf_attn.fwd(q, k, v, w.r, dil=inp["dil"], global_idx=G, key_pad_mask=pad, scale=w.softmax_scale,
                        stream=stream)
        call = lambda: lf_attn.bwd(q, k, v, y, dy, w.r, dil=inp["dil"], global_idx=G, key_pad_mask=pad,
                                   scale=w.softmax_scale, stream=stream)
        call()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(calls):
            call()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / calls
    return {"value": round(2.5 * total_f / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_call": round(ms, 4),
            "useful_gflop_per_call": round(2.5 * total_f / 1e9, 4), "calls": calls,
            "kernels": "prep + row statistics + dq + dk/dv, CUDA cores, fp32 gradients"}


def copy_bandwidth(torch, dev, nbytes):
    """Pinned host <-> device copy bandwidth (GB/s) for nbytes, CUDA events."""
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for _ in range(3):
        d.copy_(h, non_blocking=True)
        h.copy_(d, non_blocking=True)
    torch.cuda.synchronize()
    res = {}
    for name, fn in (("h2d", lambda: d.copy_(h, non_blocking=True)), ("d2h", lambda: h.copy_(d, non_blocking=True))):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            fn()
        e1.record()
        torch.cuda.synchronize()
        res[name] = 10 * nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    from sparse_long_sequence_fwd_b200 import build, lf_attn

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    lf_attn.load()
    peaks, peak_src = load_peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)

    w = workloads.BY_NAME[args.workload]
    if args.backward_only:
        print(json.dumps({"backward_" + w.name: backward_entry(w, torch, lf_attn, dev, stream)}))
        return
    run = WorkloadRun(w, torch, lf_attn, dev, stream, args.warmup)
    launches_per_step = run.launches_per_step
    K = args.steps

    # ---- the timed steps; clocks are sampled during them and over a replay window of
    #      about a second around them (the steps alone can be shorter than a sample)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    one_ms = run.time_steps(run.n_sets) / run.n_sets
    pad_steps = max(run.n_sets, int(0.5 / max(one_ms * 1e-3, 1e-6)))
    run.time_steps(pad_steps)  # half a second of steps before the timed ones (clock window)
    marks = {}
    if world > 1:
        dist.barrier()
    ms = run.time_steps(K, before=lambda: marks.__setitem__("t0", time.time()),
                        after=lambda: marks.__setitem__("t1", time.time()))
    run.time_steps(pad_steps)  # and after them
    t_win1 = time.time()
    if world > 1:
        dist.barrier()
    ms = sharding.max_over_ranks(ms, device=dev)
    ms_per_step = ms / K
    sampler.stop()
    clocks = sampler.summary(marks["t0"], marks["t1"])
    if clocks.get("window") != "timed region":
        clocks = sampler.summary(marks["t0"] - 0.6, t_win1)
        clocks["window"] = "replay window of about 1 s around the %d timed steps (they take %.1f ms)" % (K, ms)

    base = run.summary(ms_per_step, peaks, world)
    band_tflops = run.band_f / (base["band_tc_us"] * 1e-6) / 1e12
    roofline = {"kernel": "band_tc_kernel", "bound": "tensor", "achieved": round(band_tflops, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(band_tflops / peaks["bf16_tflops"], 4),
                "peak_source": "%s bf16 burst (kernel timed alone)" % peak_src,
                "algorithmic": "4*d*|N(i)| summed over the %d non-global rows, per launch" % int(
                    band_row_mask(w, run.inp).sum() * w.H),
                "traffic": traffic_from_profile("band_tc.cuh")}
    kernels = {k: base[k] for k in ("band_tc_us", "prep_us") if k in base}
    if "global_rows_us" in base:
        gbw = run.gr_bytes / (base["global_rows_us"] * 1e-6) / 1e9
        kernels["global_rows_us"] = base["global_rows_us"]
        kernels["global_rows_hbm"] = {"achieved": round(gbw, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                      "frac": round(gbw / peaks["hbm_gbs"], 4),
                                      "algorithmic": "K,V of the non-padded keys + q,out of the global rows"}

    # ---- one call including its launch (no graph), host wall clock around launch + completion
    single = []
    for i in range(20):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            run.call(i)
        torch.cuda.synchronize()
        single.append(1e3 * (time.perf_counter() - t0))
    single_call_ms = float(np.median(single))

    # ---- the other workloads (each its own rotating inputs), rank 0 only
    others = {}
    if rank == 0 and world == 1 and not args.no_others:
        for name in ("qa_B2_T4096_g64_pad", "dilated_T8192_r128", "large_T16384_g32", "base_T4096_w513_f16",
                     "d128_H8_T4096_w513", "bigbird_T4096_w513_rand3"):
            if name == w.name:
                continue
            ow = workloads.BY_NAME[name]
            orun = WorkloadRun(ow, torch, lf_attn, dev, stream, args.warmup)
            o_one = orun.time_steps(orun.n_sets) / orun.n_sets
            oK = max(orun.n_sets, int(0.4 / max(o_one * 1e-3, 1e-6)))
            o_ms = orun.time_steps(oK) / oK
            others[name] = orun.summary(o_ms, peaks)
            del orun
            torch.cuda.empty_cache()
        others["backward_" + w.name] = backward_entry(w, torch, lf_attn, dev, stream)

    # ---- end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if args.e2e_steps > 0:
        inp = run.inp
        hq, hk, hv = (inp[x].pin_memory() for x in ("q", "k", "v"))
        hout = torch.empty_like(hq).pin_memory()
        hg = inp["global_idx"].pin_memory() if inp["global_idx"] is not None else None
        hp = inp["key_pad_mask"].pin_memory() if inp["key_pad_mask"] is not None else None
        dil = inp["dil"]
        with torch.cuda.stream(stream):
            for _ in range(3):
                lf_attn.fwd_host(hq, hk, hv, w.r, dil=dil, global_idx=hg, key_pad_mask=hp,
                                 scale=w.softmax_scale, out=hout, stream=stream)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(args.e2e_steps):
                lf_attn.fwd_host(hq, hk, hv, w.r, dil=dil, global_idx=hg, key_pad_mask=hp,
                                 scale=w.softmax_scale, out=hout, stream=stream)
            b.record()
        torch.cuda.synchronize()
        e2e_ms = sharding.max_over_ranks(a.elapsed_time(b) / args.e2e_steps, device=dev)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv) + tuple(x for x in (hg, hp) if x is not None))
        d2h = int(hout.numel() * hout.element_size())
        bw = copy_bandwidth(torch, dev, h2d)
        bound_ms = 1e3 * (h2d / (bw["h2d"] * 1e9) + d2h / (bw["d2h"] * 1e9))
        e2e = {"value": round(sharding.job_rate(run.total_f, world, e2e_ms * 1e-3) / 1e12, 4), "unit": "TFLOP/s",
               "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": d2h,
               "api": "lf_attn_fwd_host (pinned host buffers, copies inside the timed region)",
               "copy_bound": {"h2d_gbs": round(bw["h2d"], 2), "d2h_gbs": round(bw["d2h"], 2),
                              "serial_copy_ms": round(bound_ms, 4),
                              "frac": round(bound_ms / e2e_ms, 4),
                              "note": "plain pinned copies of the same bytes on this box, one after the other; "
                                      "frac = their time / the e2e step (the entry point overlaps copies of one "
                                      "slice with kernels of another, so frac can exceed 1)"}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, run.inp, args.cpu_seconds)

    tflops = sharding.job_rate(run.total_f, world, ms_per_step * 1e-3) / 1e12
    tokens = sharding.job_rate(w.B * w.T, world, ms_per_step * 1e-3)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(tflops, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic: seeded iid N(0,1) q/k/v rounded to %s" % w.dtype,
            "config": workload_config(w, {"parallelism": "replicas (one workload per GPU)" if world > 1 else "1 GPU",
                                          "l2": base["l2"],
                                          "timing": "CUDA graphs of %d steps, CUDA events on the launch stream"
                                                    % min(run.n_sets, K)}),
            "tokens_per_s": round(tokens, 1),
            "pct_of_bf16_peak": round(100.0 * tflops / world / peaks["bf16_tflops"], 2),
            "useful_gflop_per_step": round(run.total_f / 1e9, 4),
            "roofline": roofline, "kernels": kernels, "single_call_ms": round(single_call_ms, 4),
            "workloads": others, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(K * launches_per_step), "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------- CPU oracle
def oracle_sample_rate(w, inp, seconds, seed=0, nthreads=0):
    """Times the oracle on seeded random rows for about `seconds` (nthreads 0: every host core); returns
    (useful FLOPs, seconds, rows, threads)."""
    import oracle

    rng = np.random.default_rng(seed)
    pad = inp["key_pad_mask"]
    G = inp["global_idx"]
    counts = {}

    def row_flops(rows):
        f = 0
        for b, h, i in rows:
            key = (b, int(w.dil[h]))
            if key not in counts:
                counts[key] = flops_mod.row_key_counts(
                    w.T, w.r, key[1], None if G is None else G[b].numpy(), None if pad is None else pad[b].numpy())
            f += int(counts[key][i])
        return 4.0 * w.d * f

    def draw(n):
        return np.stack([rng.integers(0, w.B, n), rng.integers(0, w.H, n), rng.integers(0, w.T, n)], 1).astype(
            np.int32)

    def run(rows):
        t0 = time.perf_counter()
        oracle.rows(inp["q"], inp["k"], inp["v"], w.r, rows, dil=inp["dil"], global_idx=G, key_pad_mask=pad,
                    scale=w.softmax_scale, nthreads=nthreads)
        return time.perf_counter() - t0

    # calibrate: grow the probe until it runs long enough to measure the rate
    n = 256
    while True:
        dt = run(draw(n))
        if dt >= min(0.5, seconds / 8) or n >= 64 * w.B * w.H * w.T:
            break
        n *= 4
    # rows are drawn with replacement, so a cheap workload is sampled several times over
    n = int(min(max(256, n * seconds / max(dt, 1e-4)), 64 * w.B * w.H * w.T))
    rows = draw(n)
    dt = run(rows)
    return row_flops(rows.tolist()), dt, n, (nthreads if nthreads > 0 else oracle.max_threads())


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, inp, seconds):
    f, dt, n, threads = oracle_sample_rate(w, inp, seconds)
    f1, dt1, n1, _ = oracle_sample_rate(w, inp, seconds, seed=1, nthreads=1)
    return {"value": round(f / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": "%d seeded random rows of %s (%.1f s, fp64 C oracle, OpenMP %d threads, %s)" % (
                n, w.name, dt, threads, cpu_model()),
            "single_thread": {"value": round(f1 / dt1 / 1e12, 6), "unit": "TFLOP/s", "cores": 1,
                              "sample": "%d seeded random rows of %s (%.1f s, one thread)" % (n1, w.name, dt1)}}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = workloads.BY_NAME[args.workload]
    inp = workloads.make_inputs(w)
    steps = max(args.steps, 1)
    per_step = max(0.002, min(2.0, 60.0 / (steps + max(args.warmup, 0))))
    for _ in range(max(args.warmup, 0)):
        oracle_sample_rate(w, inp, per_step / 4, seed=1)
    tot_f = tot_t = 0.0
    rows = 0
    threads = 1
    for s in range(steps):
        f, dt, n, threads = oracle_sample_rate(w, inp, per_step / 2, seed=100 + s)
        tot_f += f
        tot_t += dt
        rows += n
    value = tot_f / tot_t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_t / steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: seeded iid N(0,1) q/k/v rounded to %s, widened to fp64" % w.dtype,
            "config": workload_config(w, {"sample": "per step: seeded random rows"}),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": "%d rows over %d steps of %s (%s)" % (rows, steps, w.name, cpu_model())},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
