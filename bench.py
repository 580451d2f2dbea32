"""Benchmark: exact attention forward + backward on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole hot path over one batch of synthetic input:
the forward (O, lse) and then the backward (dQ, dK, dV from dO and the
forward's O and lse), causal, B=2, H=16, S=8192, D=128, bf16 (the causal
forward workload and the backward workload share these shapes).  FLOPs
follow the convention 4*B*H*S_q*S_k*D for the forward, 2.5x that for the
backward, halved for causal.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream; L2 is flushed (a 256 MiB write, then a read of another
256 MiB that evicts the written lines) before every timed
step, outside the events.  For N > 1 (torchrun, one process per GPU) every
rank runs the same workload independently (replicas: the path has no
exchange step), steps are bracketed by barriers and the slowest rank's time
is reported; value = all ranks' FLOPs / that time.

The e2e figure times the same steps from pinned host buffers through
attn.FwdBwdPipeline (every step's inputs go up and its results come down inside
the timed region; copies overlap the neighbouring steps' kernels).

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the one other use of oracle/ here, besides the
cpu_baseline leg).  --profile fwd|bwd launches one pass repeatedly (the driver
for ncu captures); --variants prints timed side measurements (e4m3 Q/K forward,
decode shapes, deterministic backward) instead of the JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "attention fwd/bwd TFLOPS (bf16, D=128) and % of B200 dense BF16 peak"
SPEC_PEAK_TFLOPS = 2250.0  # dense bf16 tensor peak the pages quote for B200
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}

WORKLOADS = {
    "causal8k": (workloads.FWD_CAUSAL, workloads.BWD_CAUSAL),
}


def captured_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from profiles/roofline_traffic.txt, or None
    when the kernel sources changed since that capture (sha1 mismatch)."""
    import glob
    import hashlib

    h = hashlib.sha1()
    for f in sorted(glob.glob(os.path.join(ROOT, "attention_attn_fwd_10_b200", "csrc", "*.cuh"))):
        with open(f, "rb") as fh:
            h.update(fh.read())
    try:
        with open(os.path.join(ROOT, "profiles", "roofline_traffic.txt")) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 3 and not line.startswith("#") and parts[0] == kernel:
                    return int(parts[1]) if parts[2] == h.hexdigest() else None
    except OSError:
        pass
    return None


def frac_key(peaks_src: str, suffix: str = "") -> str:
    """Name of a fraction-of-peak key: of the measured peaks when MEASURED_PEAKS.json
    was read, else of the recipe's fallback figures."""
    return ("frac_of_measured" if peaks_src == "measured" else "frac_of_fallback") + suffix


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 20):
        self.gpu = gpu_index
        self.interval_ms = interval_ms
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.interval_ms)], stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)  # nvidia-smi starts sampling only after it has initialised
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r.strip().split(", ") for r in f if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons)}


# --------------------------------------------------------------------------- L2 flush

class L2Flush:
    """Empties L2 (126 MB) before a timed call: a 256 MiB write, then one pass over a
    second 256 MiB buffer with the library's read probe.  The read evicts the
    written lines, so their write-back to DRAM happens here and not inside the timed
    region that follows (a write alone leaves up to 126 MB of dirty lines that the
    next kernel's reads would have to make room for)."""

    def __init__(self, attn, dev):
        import torch

        self.wbuf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.rbuf = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
        self.sink = torch.zeros(1, dtype=torch.int64, device=dev)
        self.lib = attn.load()

    def __call__(self):
        import torch

        self.wbuf.fill_(1)
        code = self.lib.attn_read_probe(self.rbuf.data_ptr(), self.rbuf.numel(), self.sink.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)
        if code != 0:
            raise RuntimeError(f"attn_read_probe failed: {code}")


# --------------------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus: int):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    if world != n_gpus and rank == 0:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE={world}", file=sys.stderr)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(world, x: float, device: str = "cuda") -> float:
    """The slowest rank's value (every rank takes part; NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, flops_per_rank_step: float, step_ms_max: float) -> float:
    """Whole-job TFLOPS of N independent replicas: all ranks' work / slowest rank's time."""
    return world * flops_per_rank_step / (step_ms_max * 1e-3) / 1e12


# --------------------------------------------------------------------------- oracle (CPU) timing

def oracle_sample_time(wf, wb, budget_s: float = 15.0):
    """Time the fp64 oracle's forward+backward on whole (b, h) heads of the workload
    until about budget_s of CPU time; returns (TFLOPS by convention, sample text, cores)."""
    import numpy as np

    from oracle import reference as ref

    x = workloads.make_inputs(wb)
    cores = len(os.sched_getaffinity(0))
    per_head_flops = (wf.fwd_flops() + wb.bwd_flops()) / (wf.B * wf.H_q)
    done, t0 = 0, time.perf_counter()
    heads = [(b, h) for b in range(wf.B) for h in range(wf.H_q)]
    for (b, h) in heads:
        qh = x["q"][b:b + 1, :, h:h + 1]
        kh = x["k"][b:b + 1, :, h:h + 1]
        vh = x["v"][b:b + 1, :, h:h + 1]
        doh = x["do"][b:b + 1, :, h:h + 1]
        ref.forward(qh, kh, vh, wf.causal, wf.scale)
        ref.backward(qh, kh, vh, doh, wb.causal, wb.scale)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    del np
    return per_head_flops * done / dt / 1e12, f"{done} of {len(heads)} (b,h) heads, fwd+bwd, full S", cores, dt


# --------------------------------------------------------------------------- our implementation

def run_ours(args):
    import torch

    import attention_attn_fwd_10_b200 as attn

    world, rank, local = dist_setup(args.gpus)
    wf, wb = WORKLOADS[args.workload]
    dev = torch.device("cuda", local if world > 1 else 0)
    x = workloads.make_inputs(wb)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((wf.B, wf.H_q, wf.S_q), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn.bwd_workspace_size(wb.B, wb.H_q, wb.S_q, wb.D), dtype=torch.uint8, device=dev)
    flush = L2Flush(attn, dev)
    stream = torch.cuda.current_stream()

    have_bwd = True
    try:
        attn.bwd(q, k, v, o, lse, do, causal=True, dq=dq, dk=dk, dv=dv, workspace=ws)
    except RuntimeError:
        have_bwd = False

    def fwd():
        attn.fwd(q, k, v, causal=wf.causal, scale=wf.scale, out=o, lse=lse)

    def bwd(events=None):
        attn.bwd(q, k, v, o, lse, do, causal=wb.causal, scale=wb.scale, dq=dq, dk=dk, dv=dv, workspace=ws,
                 main_pass_events=events)

    for _ in range(args.warmup):
        fwd()
        if have_bwd:
            bwd()
    torch.cuda.synchronize()
    if attn.device_status() != 0:
        raise RuntimeError("device status not OK after warm-up")

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    f_ms, b_ms, s_ms, m_ms = [], [], [], []
    with ClockSampler(dev.index) as clk:
        for _ in range(args.steps):
            flush()
            barrier(world)
            torch.cuda.synchronize()
            e0, e1, e2, m0, m1 = ev(), ev(), ev(), ev(), ev()
            e0.record(stream)
            fwd()
            e1.record(stream)
            if have_bwd:
                bwd((m0, m1))
            e2.record(stream)
            torch.cuda.synchronize()
            f_ms.append(e0.elapsed_time(e1))
            b_ms.append(e1.elapsed_time(e2))
            s_ms.append(e0.elapsed_time(e2))
            if have_bwd:
                m_ms.append(m0.elapsed_time(m1))
        barrier(world)
    clocks = clk.summary()
    if attn.device_status() != 0:
        raise RuntimeError("device status not OK after the timed region")

    step_ms = max_over_ranks(world, sum(s_ms) / len(s_ms))
    fwd_ms = sum(f_ms) / len(f_ms)
    bwd_ms = sum(b_ms) / len(b_ms) if have_bwd else 0.0
    main_ms = sum(m_ms) / len(m_ms) if have_bwd else 0.0
    flops_step = wf.fwd_flops() + (wb.bwd_flops() if have_bwd else 0.0)
    value = replica_throughput(world, flops_step, step_ms)

    # end to end through the public API with pinned host buffers
    e2e = run_e2e(args, attn, x, wf, wb, have_bwd, dev, world)

    peaks, peaks_src = measured_peaks()
    configs = None
    if world == 1 and not args.no_configs:
        del q, k, v, do, o, lse, dq, dk, dv, ws
        configs = run_configs(attn, dev, flush, peaks, peaks_src)
    fwd_tf = wf.fwd_flops() / (fwd_ms * 1e-3) / 1e12
    bwd_tf = wb.bwd_flops() / (bwd_ms * 1e-3) / 1e12 if have_bwd else None
    # dominant kernel: the one with the larger share of the step
    if have_bwd and main_ms > fwd_ms:
        dom, dom_flops, dom_ms = "attn_bwd_kernel (main pass)", wb.bwd_flops(), main_ms
    else:
        dom, dom_flops, dom_ms = "attn_fwd_kernel", wf.fwd_flops(), fwd_ms
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) rounded to bf16)",
        "config": {
            "workload": wf.name.replace("fwd_", "fwd+bwd_") if have_bwd else wf.name,
            "step": "forward + backward" if have_bwd else "forward only (backward not built)",
            "B": wf.B, "H_q": wf.H_q, "H_kv": wf.H_kv, "S": wf.S_q, "D": wf.D, "causal": wf.causal,
            "global_batch": wf.B * world, "seq_len": wf.S_q, "parallelism": f"replicas x{world}",
            "l2": "flushed before every timed step: 256 MiB written, then 256 MiB of another buffer read "
                  "(the write's dirty lines are evicted before the timed region)",
        },
        "fwd": {"ms": round(fwd_ms, 4), "tflops": round(fwd_tf, 1),
                "frac_of_spec_2250": round(fwd_tf / SPEC_PEAK_TFLOPS, 4),
                frac_key(peaks_src): round(fwd_tf / peak, 4)},
        "bwd": ({"ms": round(bwd_ms, 4), "main_pass_ms": round(main_ms, 4), "tflops": round(bwd_tf, 1),
                 "frac_of_spec_2250": round(bwd_tf / SPEC_PEAK_TFLOPS, 4),
                 frac_key(peaks_src): round(bwd_tf / peak, 4)} if have_bwd else None),
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{peaks_src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
                     if peaks_src == "measured" else "fallback 1.59 PFLOP/s burst",
                     "traffic": captured_traffic("attn_bwd_kernel" if dom.startswith("attn_bwd") else "attn_fwd_kernel"),
                     "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "e2e": e2e,
        "configs": configs,
        "gpu_launches": args.steps * (1 + (3 if have_bwd else 0)),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, sample, cores, dt = oracle_sample_time(wf, wb if have_bwd else wb, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                                "sample": sample + f" ({dt:.1f} s, fp64 numpy)"}
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, attn, x, wf, wb, have_bwd, dev, world):
    """Same metric through the public API with pinned host buffers.  Every
    timed step copies its inputs q, k, v (and dO) host -> device, runs the
    kernels, and copies o, lse (and dq, dk, dv) device -> host.  With the
    backward the steps go through attn.FwdBwdPipeline, which overlaps one step's
    copies with its neighbours' kernels (separate copy and compute streams);
    the time is from the first upload to the last download, divided by the
    number of steps."""
    import torch

    hq, hk, hv, hdo = (x[n].pin_memory() for n in ("q", "k", "v", "do"))
    host_out = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in
                (("o", hq), ("dq", hq), ("dk", hk), ("dv", hv))}
    host_out["lse"] = torch.empty((wf.B, wf.H_q, wf.S_q), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in ((hq, hk, hv, hdo) if have_bwd else (hq, hk, hv)))
    d2h_names = ("o", "lse", "dq", "dk", "dv") if have_bwd else ("o", "lse")
    d2h = sum(host_out[n].numel() * host_out[n].element_size() for n in d2h_names)
    n_steps = max(3, min(args.steps, 10))

    if have_bwd:
        pipe = attn.FwdBwdPipeline(wf.B, wf.S_q, wf.S_k, wf.H_q, wf.H_kv, wf.D, causal=wf.causal, scale=wf.scale)
        for _ in range(2):
            pipe.submit(hq, hk, hv, hdo, host_out)
        pipe.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(pipe.up)
        for _ in range(n_steps):
            pipe.submit(hq, hk, hv, hdo, host_out)
        e1.record(pipe.down)
        pipe.synchronize()
        step_ms = e0.elapsed_time(e1) / n_steps
        mode = "pipelined: copy streams overlap the compute stream across steps"
    else:
        def step():
            o, lse = attn.fwd(hq, hk, hv, causal=wf.causal, scale=wf.scale)
            host_out["o"].copy_(o)
            host_out["lse"].copy_(lse)

        for _ in range(2):
            step()
        torch.cuda.synchronize()
        ms = []
        for _ in range(n_steps):
            barrier(world)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            step()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        step_ms = sum(ms) / len(ms)
        mode = "sequential"
    step_ms = max_over_ranks(world, step_ms)
    flops = wf.fwd_flops() + (wb.bwd_flops() if have_bwd else 0.0)
    res = {"value": round(world * flops / (step_ms * 1e-3) / 1e12, 2), "unit": "TFLOPS",
           "ms_per_step": round(step_ms, 3), "steps": n_steps, "mode": mode,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if have_bwd:
        # the latency one call sees: attn.fwd_bwd uploads the step's inputs, runs the
        # forward and the backward, downloads every result and synchronises, nothing overlapped
        for _ in range(2):
            attn.fwd_bwd(hq, hk, hv, hdo, causal=wf.causal, scale=wf.scale, host_out=host_out)
        ms = []
        for _ in range(n_steps):
            barrier(world)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            attn.fwd_bwd(hq, hk, hv, hdo, causal=wf.causal, scale=wf.scale, host_out=host_out)
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        seq_ms = max_over_ranks(world, sum(ms) / len(ms))
        res["sequential"] = {"value": round(world * flops / (seq_ms * 1e-3) / 1e12, 2), "unit": "TFLOPS",
                             "ms_per_step": round(seq_ms, 3), "steps": n_steps,
                             "mode": "one attn.fwd_bwd call per step: upload, kernels, download, in sequence"}
    return res


def timed_calls(fn, flush, stream, min_ms: float = 250.0, min_reps: int = 10, warmup: int = 3):
    """Median device time (ms) of fn() over enough calls to span about min_ms of
    kernel time, each call bracketed by CUDA events on `stream` with L2 flushed
    before it (outside the events).  Returns (median_ms, reps)."""
    import torch

    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    fn()
    e1.record(stream)
    torch.cuda.synchronize()
    est = max(e0.elapsed_time(e1), 1e-3)
    reps = max(min_reps, int(math.ceil(min_ms / est)))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs), reps


def run_configs(attn, dev, flush, peaks, peaks_src="fallback"):
    """Every forward configuration of the workload set, the split-KV decode shape
    and the deterministic backward, each timed on its own (L2 flushed before each
    call) with the SM clock sampled during its timed calls.  Returns a dict for
    the JSON line's "configs" key."""
    import torch

    stream = torch.cuda.current_stream()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    out = {}

    def fwd_entry(w, extra=None):
        x = workloads.make_inputs(w)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H_q, w.S_q), dtype=torch.float32, device=dev)
        with ClockSampler(dev.index) as clk:
            ms, reps = timed_calls(lambda: attn.fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse),
                                   flush, stream)
        c = clk.summary()
        # the same forward with one CTA per work unit instead of persistent CTAs
        ms1, _ = timed_calls(lambda: attn.fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse,
                                              persistent=False), flush, stream)
        tf = w.fwd_flops() / (ms * 1e-3) / 1e12
        e = {"ms": round(ms, 4), "tflops": round(tf, 1), frac_key(peaks_src): round(tf / peak, 4),
             "frac_of_spec_2250": round(tf / SPEC_PEAK_TFLOPS, 4), "reps": reps,
             "sm_mhz": c["sm_mhz"], "clock_samples": c.get("samples"), "clock_reasons": c["reasons"],
             "one_cta_per_unit": {"ms": round(ms1, 4), "tflops": round(w.fwd_flops() / (ms1 * 1e-3) / 1e12, 1)}}
        # O rescales counted at the default threshold (tau = 8) and with a rescale on
        # every increase of the running max (tau = 0)
        counts = {}
        for tau in (8.0, 0.0):
            cnt = torch.zeros(1, dtype=torch.int64, device=dev)
            attn.fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse, rescale_threshold=tau,
                     rescale_count=cnt)
            counts[tau] = int(cnt.item())
        e["rescale_count"] = {"tau8": counts[8.0], "tau0": counts[0.0],
                              "tau0_over_tau8": round(counts[0.0] / counts[8.0], 1) if counts[8.0] else None}
        if extra:
            e.update(extra)
        out[w.name] = e
        del q, k, v, o, lse, x

    for w in (workloads.FWD_NONCAUSAL, workloads.FWD_CAUSAL, workloads.FWD_CAUSAL_SPIKY, workloads.FWD_CAUSAL_GQA):
        fwd_entry(w)

    # the causal forward workload with 8-bit inputs: e4m3 Q, K (bf16 V, P), and e4m3 Q, K, V (e4m3 P)
    w = workloads.FWD_CAUSAL
    x = workloads.make_inputs(w)
    q8, k8, v8 = (x[n].to(dev).to(torch.float8_e4m3fn) for n in ("q", "k", "v"))
    v16 = x["v"].to(dev)
    o = torch.empty((w.B, w.S_q, w.H_q, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H_q, w.S_q), dtype=torch.float32, device=dev)
    for tag, vv in (("e4m3_qk", v16), ("e4m3_qkv", v8)):
        with ClockSampler(dev.index) as clk:
            ms, reps = timed_calls(lambda: attn.fwd_qk8(q8, k8, vv, causal=True, scale=w.scale, out=o, lse=lse),
                                   flush, stream)
        c = clk.summary()
        tf = w.fwd_flops() / (ms * 1e-3) / 1e12
        # fraction of the measured bf16 peak (the 8-bit products themselves run at up to twice that rate)
        out[f"{w.name}_{tag}"] = {"ms": round(ms, 4), "tflops": round(tf, 1), frac_key(peaks_src, "_bf16"): round(tf / peak, 4),
                                  "reps": reps, "sm_mhz": c["sm_mhz"], "clock_samples": c.get("samples")}
    del q8, k8, v8, v16, o, lse, x

    # decode: one query row per head against 32768 keys, split-KV forward (bytes-bound: K and V stream once)
    w = workloads.small(B=1, H_q=32, H_kv=8, S_q=1, S_k=32768, D=128, causal=True, seed=1)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    n = attn.fwd_split_count(w.B, w.H_q, w.H_kv, w.S_q, w.S_k, True)
    ws = torch.empty(attn.load().attn_fwd_split_workspace_size(w.B, w.H_q, w.S_q, w.D, n), dtype=torch.uint8,
                     device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H_q, w.S_q), dtype=torch.float32, device=dev)
    with ClockSampler(dev.index) as clk:
        ms, reps = timed_calls(lambda: attn.fwd_split(q, k, v, causal=True, scale=w.scale, num_splits=n, out=o,
                                                      lse=lse, workspace=ws), flush, stream)
    c = clk.summary()
    bytes_alg = sum(t.numel() * t.element_size() for t in (q, k, v, o, lse))
    gbs = bytes_alg / (ms * 1e-3) / 1e9
    # What one plain pass over as many bytes as K and V takes here (the library's
    # read probe): a 134 MB read does not reach the copy bandwidth of a GB-sized
    # stream, start-up and drain being a large share of it.
    kv_bytes = (k.numel() * k.element_size() + v.numel() * v.element_size() + 15) // 16 * 16
    rbuf = torch.ones(kv_bytes // 4, dtype=torch.int32, device=dev)
    sink = torch.zeros(1, dtype=torch.int64, device=dev)
    lib = attn.load()

    def read_once():
        code = lib.attn_read_probe(rbuf.data_ptr(), kv_bytes, sink.data_ptr(), stream.cuda_stream)
        if code != 0:
            raise RuntimeError(f"attn_read_probe failed: {code}")

    ms_read, _ = timed_calls(read_once, flush, stream)
    del rbuf, sink
    out["decode_split_B1_Hq32_Hkv8_Sq1_Sk32768_D128"] = {
        "us": round(ms * 1e3, 2), "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / hbm, 4),
        "hbm_gbs": hbm, "hbm_source": peaks_src, "n_splits": n,
        "algorithmic_bytes": bytes_alg, "reps": reps, "sm_mhz": c["sm_mhz"], "clock_samples": c.get("samples"),
        "plain_read_of_kv_us": round(ms_read * 1e3, 2), "plain_read_over_decode": round(ms_read / ms, 4)}
    del q, k, v, o, lse, ws, x

    # the backward workload in its deterministic mode (fixed dQ order), and both modes
    # with the main pass on CTA pairs (cta_group::2)
    wb = workloads.BWD_CAUSAL
    x = workloads.make_inputs(wb)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = attn.fwd(q, k, v, causal=True, scale=wb.scale)
    ws = torch.empty(attn.bwd_workspace_size(wb.B, wb.H_q, wb.S_q, wb.D), dtype=torch.uint8, device=dev)
    g = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    for det, mode in ((False, 1), (True, 1), (False, 2), (True, 2)):  # explicit kernels (0 picks per mode)
        with ClockSampler(dev.index) as clk:
            ms, reps = timed_calls(lambda: attn.bwd(q, k, v, o, lse, do, causal=True, scale=wb.scale, dq=g[0],
                                                    dk=g[1], dv=g[2], workspace=ws, deterministic=det,
                                                    cta_mode=mode),
                                   flush, stream)
        c = clk.summary()
        tf = wb.bwd_flops() / (ms * 1e-3) / 1e12
        default_kernel = mode == (2 if det else 1)  # what cta_mode 0 picks for this mode
        out[wb.name + ("_deterministic" if det else "") + ("_cta_pairs" if mode == 2 else "_one_cta_per_tile")] = {
            "ms": round(ms, 4), "tflops": round(tf, 1), frac_key(peaks_src): round(tf / peak, 4), "reps": reps,
            "default": default_kernel,
            "sm_mhz": c["sm_mhz"], "clock_samples": c.get("samples")}
    del q, k, v, do, o, lse, ws, g, x
    torch.cuda.synchronize()
    if attn.device_status() != 0:
        raise RuntimeError("device status not OK after the per-configuration measurements")
    return out


# --------------------------------------------------------------------------- reference arm (the oracle)

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return  # rank 0 alone runs the CPU oracle
    wf, wb = WORKLOADS[args.workload]
    budget = max(5.0, min(60.0, args.cpu_budget))
    vals, samples = [], []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        tf, sample, cores, dt = oracle_sample_time(wf, wb, budget_s=budget / max(1, args.steps))
        vals.append(tf)
        samples.append(dt)
    value = statistics.mean(vals)
    step_ms = statistics.mean(samples) * 1e3
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) rounded to bf16)",
        "impl": "reference",
        "config": {"workload": wf.name.replace("fwd_", "fwd+bwd_"), "B": wf.B, "H_q": wf.H_q, "S": wf.S_q,
                   "D": wf.D, "causal": wf.causal, "parallelism": "CPU oracle on rank 0"},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": sample + " per step (fp64 numpy)"},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(time.perf_counter() - t_all, 1),
    }
    print(json.dumps(line), flush=True)


def run_profile(args):
    """Launch only one pass (--profile fwd|bwd|bwd_pairs|decode) W + K times on the workload, no
    timing: the driver for ncu captures of a single kernel."""
    import torch

    import attention_attn_fwd_10_b200 as attn

    wf, wb = WORKLOADS[args.workload]
    torch.cuda.set_device(0)
    if args.profile == "decode":
        # one query row per head against 32768 keys: the split-KV forward and its merge
        w = workloads.small(B=1, H_q=32, H_kv=8, S_q=1, S_k=32768, D=128, causal=True, seed=1)
        xd = workloads.make_inputs(w)
        q, k, v = (xd[n].cuda() for n in ("q", "k", "v"))
        for _ in range(args.warmup + args.steps):
            attn.fwd_split(q, k, v, causal=True, scale=w.scale)
        torch.cuda.synchronize()
        st = attn.device_status()
        print(f"profile decode: {args.warmup + args.steps} calls, device status {st}")
        if st != 0:
            sys.exit(1)
        return
    x = workloads.make_inputs(wb)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.fwd(q, k, v, causal=wf.causal, scale=wf.scale)
    ws = torch.empty(attn.bwd_workspace_size(wb.B, wb.H_q, wb.S_q, wb.D), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup + args.steps):
        if args.profile == "fwd":
            attn.fwd(q, k, v, causal=wf.causal, scale=wf.scale, out=o, lse=lse, poly_exp_every=args.poly_exp_every)
        else:
            attn.bwd(q, k, v, o, lse, do, causal=wb.causal, scale=wb.scale, workspace=ws,
                     cta_mode=2 if args.profile == "bwd_pairs" else 0)
    torch.cuda.synchronize()
    st = attn.device_status()
    print(f"profile {args.profile}: {args.warmup + args.steps} launches, device status {st}")
    if st != 0:
        sys.exit(1)


def run_variants(args):
    """Side measurements (not the contract line): the forward on each forward
    configuration in bf16 and with 8-bit Q/K, the decode shapes through the plain
    and the split-KV forward, and the backward in its normal and deterministic
    modes.  CUDA events around each call, L2 flushed before each, median of
    K timed calls after W warm-up calls.  One human-readable line each."""
    import torch

    import attention_attn_fwd_10_b200 as attn

    torch.cuda.set_device(0)
    flush = L2Flush(attn, "cuda")

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ts = []
        for _ in range(args.steps):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        if attn.device_status() != 0:
            raise RuntimeError("device status not OK")
        return statistics.median(ts)

    for w in (workloads.FWD_CAUSAL, workloads.FWD_NONCAUSAL, workloads.FWD_CAUSAL_GQA):
        x = workloads.make_inputs(w)
        q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
        q8, k8 = q.to(torch.float8_e4m3fn), k.to(torch.float8_e4m3fn)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H_q, w.S_q), dtype=torch.float32, device="cuda")
        ms16 = timed(lambda: attn.fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse))
        ms8 = timed(lambda: attn.fwd_qk8(q8, k8, v, causal=w.causal, scale=w.scale, out=o, lse=lse))
        print(f"forward {w.name}: bf16 {ms16:.3f} ms {w.fwd_flops() / ms16 / 1e9:.0f} TFLOPS | "
              f"e4m3 Q/K {ms8:.3f} ms {w.fwd_flops() / ms8 / 1e9:.0f} TFLOPS", flush=True)
        del q, k, v, q8, k8, o, lse, x
    for (B, H_q, H_kv, S_q, S_k) in ((1, 32, 8, 1, 32768), (8, 32, 8, 1, 8192), (4, 32, 8, 16, 65536),
                                     (1, 16, 16, 128, 16384)):
        w = workloads.small(B=B, H_q=H_q, H_kv=H_kv, S_q=S_q, S_k=S_k, D=128, causal=True, seed=1)
        x = workloads.make_inputs(w)
        q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
        q8, k8 = q.to(torch.float8_e4m3fn), k.to(torch.float8_e4m3fn)
        ms_plain = timed(lambda: attn.fwd(q, k, v, causal=True, scale=w.scale))
        ms_split = timed(lambda: attn.fwd_split(q, k, v, causal=True, scale=w.scale))
        ms_split8 = timed(lambda: attn.fwd_split(q8, k8, v, causal=True, scale=w.scale))
        kv_bytes = 2 * B * S_k * H_kv * 128 * 2
        n = attn.fwd_split_count(B, H_q, H_kv, S_q, S_k, True)
        print(f"decode B{B} H_q{H_q} H_kv{H_kv} S_q{S_q} S_k{S_k}: forward {ms_plain * 1e3:.1f} us | "
              f"split-KV ({n} ranges) {ms_split * 1e3:.1f} us, K+V {kv_bytes / ms_split / 1e9:.2f} TB/s | "
              f"split-KV with e4m3 Q/K {ms_split8 * 1e3:.1f} us", flush=True)
        del q, k, v, q8, k8, x
    for wb in (workloads.BWD_CAUSAL,
               workloads.small(B=2, H_q=16, S_q=8192, S_k=8192, D=64, causal=True, seed=2, backward=True)):
        x = workloads.make_inputs(wb)
        q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
        o, lse = attn.fwd(q, k, v, causal=True, scale=wb.scale)
        if wb.D == 64:
            ms = timed(lambda: attn.fwd(q, k, v, causal=True, scale=wb.scale, out=o, lse=lse))
            print(f"forward {wb.name}: bf16 {ms:.3f} ms {wb.fwd_flops() / ms / 1e9:.0f} TFLOPS", flush=True)
        ws = torch.empty(attn.bwd_workspace_size(wb.B, wb.H_q, wb.S_q, wb.D), dtype=torch.uint8, device="cuda")
        grads = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
        for det in (False, True):
            ms = timed(lambda: attn.bwd(q, k, v, o, lse, do, causal=True, scale=wb.scale, dq=grads[0],
                                        dk=grads[1], dv=grads[2], workspace=ws, deterministic=det))
            print(f"backward {wb.name} deterministic={det}: {ms:.3f} ms {wb.bwd_flops() / ms / 1e9:.0f} TFLOPS",
                  flush=True)
        del q, k, v, do, o, lse, ws, grads, x


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="causal8k")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle CPU time to sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration measurements")
    ap.add_argument("--profile", choices=("fwd", "bwd", "bwd_pairs", "decode"), default=None,
                    help="only launch one pass W+K times (driver for ncu captures); prints no JSON")
    ap.add_argument("--poly-exp-every", type=int, default=8, choices=(0, 4, 8),
                    help="--profile fwd: one column pair in N on the FMA-pipe cubic (0: MUFU only)")
    ap.add_argument("--variants", action="store_true",
                    help="side measurements (bf16 / e4m3 Q-K forward, decode shapes, deterministic backward); "
                         "prints lines, not the JSON contract")
    args = ap.parse_args()
    if args.profile:
        run_profile(args)
        return
    if args.variants:
        run_variants(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
