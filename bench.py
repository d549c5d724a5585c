#!/usr/bin/env python
"""Benchmark of the B200 exact attention forward.

One step = one attention forward (one kernel launch) over the whole workload,
inputs resident in HBM.  Default workload: the sequence-length sweep point
N=4096, B=4, H=16, d=128, bf16, non-causal -- the smallest N at which the
throughput target (>= 60% of the dense bf16 tensor-core peak) applies.
FLOPs per step = 4*B*H*N^2*d (halved when causal).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores
  python bench.py --sweep                 # one JSON line per benchmark workload

Prints one JSON line (rank 0).  Under torchrun each rank runs its own copy of
the workload (independent (b, h) problems, no collective on the data path:
weak scaling); the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_attention_154_b200 import dist as fdist  # noqa: E402
from exact_attention_154_b200 import fa, synth  # noqa: E402

METRIC = "attention fwd TFLOP/s (bf16, 1×B200) and % of dense tensor-core peak"
METRIC_BWD = "attention bwd TFLOP/s (bf16, 1×B200), 10·N²·d per head (5·N²·d causal)"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "fa_fwd_sm100_traffic.md")
# The sources each direction's kernels are built from: the forward kernel from
# its header, the PTX wrappers and the host file; the backward kernels from
# those and their own header.
KERNEL_SOURCES = {"fwd": ["exact_attention_154_b200/csrc/fa_fwd_sm100.cuh",
                          "exact_attention_154_b200/csrc/sm100_ptx.cuh",
                          "exact_attention_154_b200/csrc/fa_api.cu"]}
KERNEL_SOURCES["bwd"] = KERNEL_SOURCES["fwd"] + ["exact_attention_154_b200/csrc/fa_bwd_sm100.cuh"]


def workloads_by_key():
    table = {
        "single-head-n256": synth.single_head_n256(),
        "packed-b2-n256-h12": synth.packed_qkv_b2_n256_h12(),
        "causal-h128-n2048": synth.many_heads_causal_n2048(),
        "hd256-causal-n8192": synth.headdim256_causal(),
        "window256-causal-n4096": synth.window_causal_n4096(),
        "alibi-causal-n4096": synth.alibi_causal_n4096(),
        "varlen-mix-causal": synth.varlen_mix_causal(),
        "fp8-n4096": synth.fp8_sweep_n4096(False),
        "fp8-n4096-causal": synth.fp8_sweep_n4096(True),
    }
    for n in synth.SWEEP_N:
        table[f"sweep-n{n}"] = synth.seqlen_sweep(n, False)
        table[f"sweep-n{n}-causal"] = synth.seqlen_sweep(n, True)
    return table


DEFAULT_WORKLOAD = "sweep-n4096"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# A timed region at least this long runs the GPU at its power cap, where the
# kernel is compared with the sustained GEMM peak (cuBLAS back to back for
# 4 s); shorter regions with the burst peak.
SUSTAINED_REGION_S = 0.5


def pick_peak(peaks, peak_src, region_s, ratio=1.0):
    """(peak TFLOP/s, note) for a timed region of region_s seconds; ratio scales
    the bf16 peak to the MMA type (2 for e4m3)."""
    sustained = region_s >= SUSTAINED_REGION_S
    if peak_src != "measured":
        note = "fallback 1.4 PFLOP/s sustained" if sustained else "fallback 1.59 PFLOP/s"
    else:
        note = (f"measured dense bf16 {'sustained' if sustained else 'burst'} (MEASURED_PEAKS.json; "
                f"timed region {region_s:.2f} s {'>=' if sustained else '<'} {SUSTAINED_REGION_S} s)")
    if ratio != 1.0:
        note += " x 2 (nominal fp8 / bf16 dense ratio, 4.5 / 2.25 PFLOP/s)"
    return peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"] * ratio, note


def kernel_source_hash(direction="fwd"):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[direction]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of that direction's kernels ("bwd:" keys: the backward)
    and this workload; else None."""
    try:
        text = open(PROFILE_TRAFFIC).read()
    except OSError:
        return None
    direction = "bwd" if workload_key.startswith("bwd:") else "fwd"
    src = re.search(rf"source_sha256_{direction}:\s*([0-9a-f]+)", text)
    if not src or src.group(1) != kernel_source_hash(direction):
        return None
    m = re.search(rf"traffic_bytes_per_launch\[{re.escape(workload_key)}\]:\s*([0-9.eE+]+)", text)
    return float(m.group(1)) if m else None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        # samples under load: the upper half of the SM clocks seen
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def dist_max(x: float, world: int) -> float:
    return fdist.max_over_ranks(x, world, device="cuda")


def dist_barrier(world):
    fdist.barrier(world)


def device_inputs(w):
    if w.layout == "packed":
        (qkv,) = synth.make_inputs(w)
        return (qkv.cuda(),)
    return tuple(t.cuda() for t in synth.make_inputs(w))


def tokens(w):
    return int(sum(w.lengths)) if w.layout == "varlen" else w.B * w.N


def launcher(w, dev_inputs):
    """Returns a zero-argument callable issuing one forward on the current stream."""
    lib = fa.load()
    slopes = synth.alibi_slopes(w.H).cuda() if w.alibi else None
    sp = None if slopes is None else slopes.data_ptr()
    if w.dtype == synth.E4M3:
        q, k, v = dev_inputs
        out = torch.empty(q.shape, device="cuda", dtype=torch.bfloat16)
        lse = torch.empty((w.B, w.H, w.N), device="cuda", dtype=torch.float32)
        dq, dk, dv = synth.fp8_factors(w)
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B,
                w.H, w.N, w.d, 0.0, dq, dk, dv, int(w.causal))

        def go():
            rc = lib.fa_fwd_fp8(*args, torch.cuda.current_stream().cuda_stream)
            if rc:
                raise fa.FaError(rc, "fa_fwd_fp8")
        return go, (out, lse)
    if w.layout == "varlen":
        q, k, v, cu = dev_inputs
        out = torch.empty_like(q)
        lse = torch.empty((w.H, q.shape[0]), device="cuda", dtype=torch.float32)
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                cu.data_ptr(), w.B, w.N, q.shape[0], w.H, w.d, 0.0, int(w.causal), w.window[0],
                w.window[1], sp, w.dtype)

        def go():
            rc = lib.fa_fwd_varlen(*args, torch.cuda.current_stream().cuda_stream)
            if rc:
                raise fa.FaError(rc, "fa_fwd_varlen")
        return go, (out, lse, slopes)
    if w.masked and w.layout == "bhnd":
        q, k, v = dev_inputs
        out = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N), device="cuda", dtype=torch.float32)
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B,
                w.H, w.N, w.d, 0.0, int(w.causal), w.window[0], w.window[1], sp, w.dtype)

        def go():
            rc = lib.fa_fwd_ext(*args, torch.cuda.current_stream().cuda_stream)
            if rc:
                raise fa.FaError(rc, "fa_fwd_ext")
        return go, (out, lse, slopes)
    if w.layout == "packed":
        (qkv,) = dev_inputs
        out = torch.empty((w.B, w.N, w.H, w.d), device="cuda", dtype=qkv.dtype)
        lse = torch.empty((w.B, w.H, w.N), device="cuda", dtype=torch.float32)
        lib = fa.load()
        args = (qkv.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B, w.N, w.H, w.d, 0.0,
                int(w.causal), 0.0, w.dtype)

        def go():
            rc = lib.fa_fwd_qkvpacked(*args, torch.cuda.current_stream().cuda_stream)
            if rc:
                raise fa.FaError(rc, "fa_fwd_qkvpacked")
        return go, (out, lse)
    q, k, v = dev_inputs
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), device="cuda", dtype=torch.float32)
    lib = fa.load()
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B, w.H,
            w.N, w.d, 0.0, int(w.causal), w.dtype)

    def go():
        rc = lib.fa_fwd(*args, torch.cuda.current_stream().cuda_stream)
        if rc:
            raise fa.FaError(rc, "fa_fwd")
    return go, (out, lse)


def time_device(go, steps, warmup, world):
    for _ in range(warmup):
        go()
    dist_barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    t0 = time.perf_counter()
    for _ in range(steps):
        go()
    host_ms = (time.perf_counter() - t0) * 1e3 / steps
    end.record(stream)
    torch.cuda.synchronize()
    dist_barrier(world)
    ms = start.elapsed_time(end) / steps
    time_device.host_ms = host_ms  # enqueue time per step (Python + C ABI + launch)
    return dist_max(ms, world)


def pipelined_e2e(host, run, outs_host, steps, warmup, world, nbuf=2):
    """End-to-end steps through the public API: every step copies its inputs
    from pinned host memory (``host``), runs ``run(device_inputs)`` on the
    current stream and copies the returned tensors back into ``outs_host``.
    The copies run on their own streams against ``nbuf`` device buffer sets,
    so step k+1's upload and step k-1's download overlap step k's compute
    (a buffer set is reused only after its compute and download are done).
    Returns ms per step (max over ranks), measured from the first upload to
    the last download with CUDA events."""
    dev = [[torch.empty_like(t, device="cuda") for t in host] for _ in range(nbuf)]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_done = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]

    def step(i):
        b = i % nbuf
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_done[b])  # the last compute on this set has read it
            for h, d in zip(host, dev[b]):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        comp.wait_event(ev_out[b])  # this set's previous outputs are downloaded
        outs = run(dev[b])
        ev_done[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            for o, h in zip(outs, outs_host):
                h.copy_(o, non_blocking=True)
                o.record_stream(s_out)
            ev_out[b].record(s_out)

    for i in range(warmup):
        step(i)
    dist_barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(steps):
        step(i)
    s_out.wait_stream(comp)
    end.record(s_out)
    torch.cuda.synchronize()
    dist_barrier(world)
    return dist_max(start.elapsed_time(end) / steps, world)


def time_e2e(w, steps, warmup, world):
    """Same metric through the public Python API with pinned host inputs:
    H2D of q, k, v (or qkv), the forward, D2H of O and LSE, every step
    (pipelined across steps, see pipelined_e2e)."""
    host = [t.pin_memory() for t in synth.make_inputs(w)]
    if w.layout == "packed":
        o_host = torch.empty((w.B, w.N, w.H, w.d), dtype=host[0].dtype).pin_memory()
    elif w.dtype == synth.E4M3:
        o_host = torch.empty(host[0].shape, dtype=torch.bfloat16).pin_memory()
        factors = synth.fp8_factors(w)
    else:
        o_host = torch.empty_like(host[0]).pin_memory()
    lse_host = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    slopes = synth.alibi_slopes(w.H).cuda() if w.alibi else None
    if w.layout == "varlen":
        lse_host = torch.empty((w.H, host[0].shape[0]), dtype=torch.float32).pin_memory()

    def run(dev):
        if w.layout == "packed":
            return fa.fwd_qkvpacked(dev[0], causal=w.causal)
        if w.dtype == synth.E4M3:
            return fa.fwd_fp8(dev[0], dev[1], dev[2], *factors, causal=w.causal)
        if w.layout == "varlen":
            return fa.fwd_varlen(dev[0], dev[1], dev[2], dev[3], w.N, causal=w.causal,
                                 window_size=w.window, alibi_slopes=slopes)
        return fa.fwd(dev[0], dev[1], dev[2], causal=w.causal, window_size=w.window,
                      alibi_slopes=slopes)

    ms = pipelined_e2e(host, run, [o_host, lse_host], steps, warmup, world)
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = o_host.numel() * o_host.element_size() + lse_host.numel() * 4
    return ms, h2d, d2h


def row_flops(w, rows):
    """Algorithmic FLOPs of the given query rows (4*d per visible key)."""
    if w.window != (-1, -1):
        left, right = w.window
        right = 0 if w.causal else right
        r = np.asarray(rows, dtype=np.int64)
        lo = np.zeros_like(r) if left < 0 else np.maximum(r - left, 0)
        hi = np.full_like(r, w.N - 1) if right < 0 else np.minimum(r + right, w.N - 1)
        return float(4.0 * w.d * (hi - lo + 1).sum())
    if w.causal:
        return float(sum(4.0 * w.d * (int(r) + 1) for r in rows))
    return 4.0 * w.d * w.N * len(rows)


class OracleSampler:
    """Times the fp64 oracle, as it stands, on bounded samples of the
    workload's query rows (the same rows in every (b, h)), on all host cores.
    The sample size is calibrated once so one timed call takes ~target_s."""

    def __init__(self, w, target_s):
        import oracle
        oracle.build()
        self.oracle, self.w = oracle, w
        if w.layout == "packed":
            q, k, v = synth.unpack_qkv(synth.make_inputs(w)[0])
        elif w.layout == "varlen":
            q, k, v, cu = synth.make_inputs(w)
            self.cu = cu.numpy()
        elif w.dtype == synth.E4M3:
            (q, k, v), f = synth.fp8_inputs(w.B, w.H, w.N, w.d, w.seed, w.sigma_qk, w.sigma_v)
            q, k, v = (torch.from_numpy(fi * oracle.decode_e4m3(t.view(torch.uint8).numpy()))
                       for t, fi in zip((q, k, v), f))
        else:
            q, k, v = synth.make_inputs(w)
        self.qkv = tuple(t.double().numpy() for t in (q, k, v))
        self.rng = np.random.default_rng(w.seed + 2000)
        self.scale = fa.default_scale(w.d)
        self.slopes = synth.alibi_slopes(w.H).double().numpy() if w.alibi else None
        if w.layout == "varlen":
            # whole sequences, shortest first, until about target_s of work
            dt, fl, _ = self.run(1)
            self.nseq = max(1, min(w.B, int(max(target_s, 1e-3) / max(dt, 1e-4))))
            return
        n0 = min(w.N, 2)
        dt, _, _ = self.run(n0)
        self.nrows = max(1, min(w.N, int(n0 * max(target_s, 1e-3) / max(dt, 1e-4))))

    def run(self, n):
        w = self.w
        if w.layout == "varlen":
            order = np.argsort(np.diff(self.cu), kind="stable")[:n]
            t0 = time.perf_counter()
            fl = 0.0
            for b in order:
                s0, s1 = int(self.cu[b]), int(self.cu[b + 1])
                self.oracle.attention_varlen(*(t[s0:s1] for t in self.qkv), [0, s1 - s0],
                                             scale=self.scale, causal=w.causal, window=w.window,
                                             alibi_slopes=self.slopes)
                fl += 4.0 * w.d * w.H * synth.visible_pairs(s1 - s0, w.causal, w.window)
            return time.perf_counter() - t0, fl, n
        rows = np.sort(self.rng.choice(w.N, size=n, replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        if w.masked:
            self.oracle.attention_masked(*self.qkv, scale=self.scale, causal=w.causal, rows=rows,
                                         window=w.window, alibi_slopes=self.slopes)
        else:
            self.oracle.attention(*self.qkv, scale=self.scale, causal=w.causal, rows=rows)
        return time.perf_counter() - t0, row_flops(w, rows) * w.B * w.H, n

    def step(self):
        w = self.w
        if w.layout == "varlen":
            dt, fl, n = self.run(self.nseq)
            sample = (f"the {n} shortest of the {w.B} sequences of the workload, whole, "
                      f"fp64 oracle, all host threads")
        else:
            dt, fl, n = self.run(self.nrows)
            sample = (f"{n} seeded query rows in each of the {w.B * w.H} (b, h) heads of "
                      f"the workload (of N={w.N}), fp64 oracle, all host threads")
        return {"value": fl / dt / 1e12, "unit": UNIT, "cores": self.oracle.num_threads(),
                "kind": "oracle", "seconds": round(dt, 4), "sample": sample}


def cpu_oracle_sample(w, target_s=12.0):
    return OracleSampler(w, target_s).step()


def clocks_ok(c):
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    return not (bad & set(c.get("reasons", [])))


def bench_gpu(args, w, key, world, rank, local):
    w = fdist.shard_workload(w, world, rank)
    dev_in = device_inputs(w)
    go, _ = launcher(w, dev_in)
    flops = w.flops
    steps = args.steps
    with ClockSampler(local) as clk:
        ms = time_device(go, steps, args.warmup, world)
    clocks = clk.summary()
    e2e_steps = max(3, min(steps, 50))
    e2e_ms, h2d, d2h = time_e2e(w, e2e_steps, min(args.warmup, 3), world)
    rc, detail = fa.device_status(clear=True)
    if rc != fa.FA_OK:
        raise RuntimeError(f"kernel watchdog fired ({detail:#x})")
    peaks, peak_src = load_peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    value = world * flops / (ms * 1e-3) / 1e12
    # e4m3 MMAs: the measured bf16 peak times the nominal fp8 / bf16 ratio (2)
    ratio = 2.0 if w.dtype == synth.E4M3 else 1.0
    peak, peak_note = pick_peak(peaks, peak_src, ms * steps * 1e-3, ratio)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": synth.DTYPE_NAME[w.dtype], "data": DATA,
        "config": run_config(w, key, world),
        "pct_of_peak": {
            "measured_burst": round(100 * achieved / peak, 2),
            "measured_sustained": round(100 * achieved / (peaks["bf16_tflops_sustained"] * ratio), 2),
            "nvidia_dense_datasheet": round(100 * achieved / (2250.0 * ratio), 2),
            "peaks_source": peak_src},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2),
                     "peak": round(peak, 2), "unit": UNIT,
                     "frac": round(achieved / peak, 4),
                     "peak_note": peak_note,
                     "traffic": profiled_traffic(key),
                     "algorithmic_bytes": algorithmic_bytes(w),
                     "kernel": "fa_fwd_kernel", "launches_per_step": 1},
        "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps},
        "gpu_launches": steps,
        "host_ms_per_step": round(time_device.host_ms, 5),
        "clocks": clocks,
    }
    if not clocks_ok(clocks):
        line["clocks_rejected"] = True
    return line


def bwd_inputs(w):
    """q, k, v and a seeded upstream gradient dO, all [B, H, N, d], on the host."""
    q, k, v = synth.make_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 500)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    return q, k, v, dout


def bench_gpu_bwd(args, w, key, world, rank, local):
    """One step = one fa_bwd call (row statistic, dK/dV and dQ kernels) on
    inputs resident in HBM; O and LSE come from one forward beforehand."""
    if w.layout != "bhnd" or w.d not in (64, 128):
        raise SystemExit(f"--direction bwd needs a [B,H,N,d] workload with d in (64, 128): {key}")
    w = fdist.shard_workload(w, world, rank)
    host = bwd_inputs(w)
    q, k, v, dout = (t.cuda() for t in host)
    o, lse = fa.fwd(q, k, v, causal=w.causal)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    work = torch.empty((w.B, w.H, w.N), device="cuda", dtype=torch.float32)
    lib = fa.load()
    cargs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
             dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), work.data_ptr(), w.B, w.H, w.N, w.d, 0.0,
             int(w.causal), w.dtype)

    def go():
        rc = lib.fa_bwd(*cargs, torch.cuda.current_stream().cuda_stream)
        if rc:
            raise fa.FaError(rc, "fa_bwd")

    flops = 2.5 * w.flops
    with ClockSampler(local) as clk:
        ms = time_device(go, args.steps, args.warmup, world)
    clocks = clk.summary()
    # end to end: host q, k, v, O, LSE, dO in; dQ, dK, dV out, every step
    pinned = [t.pin_memory() for t in host] + [o.cpu().pin_memory(), lse.cpu().pin_memory()]
    outs = [torch.empty_like(t).pin_memory() for t in host[:3]]
    e2e_steps = max(3, min(args.steps, 30))
    e2e_ms = pipelined_e2e(
        pinned, lambda d: fa.bwd(d[0], d[1], d[2], d[4], d[5], d[3], causal=w.causal), outs,
        e2e_steps, 3, world)
    rc, detail = fa.device_status(clear=True)
    if rc != fa.FA_OK:
        raise RuntimeError(f"kernel watchdog fired ({detail:#x})")
    peaks, peak_src = load_peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    bpeak, bpeak_note = pick_peak(peaks, peak_src, ms * args.steps * 1e-3)
    e = 2
    nd = w.B * w.H * w.N * w.d
    line = {
        "metric": METRIC_BWD, "value": round(world * achieved, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": synth.DTYPE_NAME[w.dtype], "data": DATA,
        "config": dict(w.describe(), workload_key=key, direction="bwd",
                       parallelism=f"replicas{world}" if world > 1 else "single-gpu",
                       global_batch=w.B * world, seq_len=w.N,
                       l2="inputs larger than L2" if 8 * nd * e > (126 << 20) else "inputs fit in L2"),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2),
                     "peak": round(bpeak, 2), "unit": UNIT,
                     "frac": round(achieved / bpeak, 4),
                     "peak_note": bpeak_note,
                     # DRAM bytes of all three kernels of one step (ncu)
                     "traffic": profiled_traffic("bwd:" + key),
                     "algorithmic_bytes": 8 * nd * e + 12 * w.B * w.H * w.N,
                     "kernel": "fa_bwd_kernel", "launches_per_step": 3},
        "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pinned),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs),
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if not clocks_ok(clocks):
        line["clocks_rejected"] = True
    return line, host


def cpu_oracle_bwd_sample(w, host, target_s=12.0):
    """The fp64 gradient oracle, as it stands, on the first heads of the
    workload (it runs one (b, h) per host thread), sized to ~target_s."""
    import oracle
    oracle.build()
    q, k, v, g = (t.double().numpy().reshape(w.B * w.H, w.N, w.d) for t in host)
    scale = fa.default_scale(w.d)
    t0 = time.perf_counter()
    oracle.attention_bwd(q[:1], k[:1], v[:1], g[:1], scale=scale, causal=w.causal)
    dt1 = max(time.perf_counter() - t0, 1e-4)
    threads = oracle.num_threads()
    heads = max(1, min(w.B * w.H, threads * max(1, int(target_s / dt1))))
    t0 = time.perf_counter()
    oracle.attention_bwd(q[:heads], k[:heads], v[:heads], g[:heads], scale=scale, causal=w.causal)
    dt = time.perf_counter() - t0
    fl = 2.5 * w.flops / (w.B * w.H) * heads
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "seconds": round(dt, 4),
            "sample": f"{heads} of the {w.B * w.H} (b, h) heads of the workload, whole heads, "
                      f"fp64 gradient oracle, one head per host thread"}


L2_BYTES = 126 * 10 ** 6
DATA = "synthetic: seeded CPU torch randn (fp32) x sigma, rounded once to the compute dtype"


def run_config(w, key, world):
    """The ``config`` object of a forward line; both arms print the same one."""
    return dict(w.describe(), workload_key=key,
                parallelism=f"replicas{world}" if world > 1 else "single-gpu",
                global_batch=w.B * world, seq_len=w.N,
                l2=l2_note(algorithmic_bytes(w)))


def l2_note(step_bytes):
    """How the timed steps relate to the 126 MB L2 (no flush is done)."""
    if step_bytes > L2_BYTES:
        return "inputs larger than L2 (q,k,v,o = %d MiB per step)" % (step_bytes >> 20)
    return "inputs fit in L2 (q,k,v,o = %d KiB per step; no flush between steps)" % (
        step_bytes >> 10)


def algorithmic_bytes(w):
    e = 1 if w.dtype == synth.E4M3 else 2
    # q, k, v read and o written once (o is bf16 for e4m3 inputs), fp32 LSE
    return (3 * e + 2) * tokens(w) * w.H * w.d + 4 * tokens(w) * w.H


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads_by_key()))
    ap.add_argument("--sweep", action="store_true", help="one line per benchmark workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--direction", choices=["fwd", "bwd"], default="fwd",
                    help="fwd: the forward (default); bwd: the gradient (fa_bwd)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    table = workloads_by_key()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        w = table[args.workload]
        # the whole --steps K --warmup W run stays within about two minutes
        sampler = OracleSampler(w, target_s=min(10.0, 120.0 / max(1, args.steps + args.warmup)))
        for _ in range(args.warmup):
            sampler.step()
        per_step = [sampler.step() for _ in range(args.steps)]
        info = per_step[-1]
        value = statistics.median(x["value"] for x in per_step)
        line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": DATA,
                "config": run_config(w, args.workload, args.gpus),
                "cpu_baseline": dict(info, value=round(value, 6)),
                "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "gpu_launches": 0}
        print(json.dumps(line))
        return 0

    world, rank, local = dist_setup()
    keys = list(table) if args.sweep else [args.workload]
    for key in keys:
        w = table[key]
        if args.direction == "bwd":
            if args.sweep and (w.layout != "bhnd" or w.d not in (64, 128)):
                continue
            line, host = bench_gpu_bwd(args, w, key, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.sweep:
                line["cpu_baseline"] = cpu_oracle_bwd_sample(w, host)
        else:
            line = bench_gpu(args, w, key, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.sweep:
                line["cpu_baseline"] = cpu_oracle_sample(w)
        if rank == 0:
            print(json.dumps(line), flush=True)
        torch.cuda.empty_cache()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
