#!/usr/bin/env python3
"""Benchmark of the B200 attention forward pass; prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload causal_8k] [--impl fa2|reference]

A step is one forward pass (one launch of the CUDA kernel) over the workload's
synthetic inputs, already resident in HBM.  L2 is flushed (a 256 MiB write)
before every step, outside the per-step CUDA events that time the launch on
its own stream.  ``value`` = algorithmic TFLOP/s of all ranks (4*B*Hq*Nq*Nk*d,
halved when causal) / max-over-ranks mean step time.  With N > 1 (torchrun),
the job is one problem whose KV-head groups are split over the ranks, each
rank holding one workload's worth of heads (weak scaling; the ranks exchange
nothing but the timing reduction).

``e2e`` measures the same metric through the public API with host buffers:
pinned-host Q/K/V -> device, the C-ABI call, O and LSE -> pinned host.
``--impl reference`` times the CPU fp64 oracle on a bounded sample instead.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_tiled_attention_29_b200.inputs import (EXTRA_WORKLOADS, WORKLOADS, bf16_bits,  # noqa: E402
                                                  make_qkv, shard_seed)

ALL_WORKLOADS = {**WORKLOADS, **EXTRA_WORKLOADS}

METRIC = "attention fwd TFLOP/s (bf16, 1 B200) and % of dense BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SRC = os.path.join(ROOT, "exact_tiled_attention_29_b200", "csrc", "fa2_forward.cu")
L2_FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="causal_8k", choices=sorted(ALL_WORKLOADS))
    ap.add_argument("--impl", default="fa2", choices=["fa2", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--direction", default="fwd", choices=["fwd", "bwd"],
                    help="fwd: the forward pass (the headline); bwd: fa2_backward on the forward's "
                         "outputs, FLOPs counted as 2.5x the forward's (five matrix products "
                         "instead of two)")
    ap.add_argument("--schedule", default="units", choices=["units", "streamk", "auto"],
                    help="auto: fa2_forward_auto with a workspace (the library picks); "
                         "streamk: fa2_forward_ws, one persistent block per SM over a workspace; "
                         "units: fa2_forward, one block per (query block, head, batch)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# files whose code each kernel family is compiled from (the backward file is
# included into the forward translation unit but adds no forward code)
KERNEL_FILES = {"fa2_fwd_kernel": ("fa2_forward.cu", "sm100_ptx.cuh"),
                "fa2_bwd_kernel": ("fa2_forward.cu", "fa2_backward.cuh", "sm100_ptx.cuh")}


def _code_only(text: str) -> str:
    """C/C++ source with comments and blank lines removed (so that editing a
    comment does not retire a profile taken on the same code)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash(kernel: str = "fa2_fwd_kernel") -> str:
    """Hash of the code (comments stripped) of the files a kernel family is compiled from."""
    h = hashlib.sha256()
    for name in KERNEL_FILES[kernel]:
        with open(os.path.join(ROOT, "exact_tiled_attention_29_b200", "csrc", name)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str = "fa2_fwd_kernel"):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m_b or not m_h or m_h.group(1) != kernel_source_hash(kernel):
        return None
    return float(m_b.group(1))


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """Samples nvidia-smi clocks/throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self._thr = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self._thr = threading.Thread(target=self._read, daemon=True)
        self._thr.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._thr:
            self._thr.join(timeout=2)
        return self.summary()

    def summary(self):
        mhz, maxmhz, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                maxmhz = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() in ("active", "1", "yes"):
                    reasons.add(n)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": maxmhz, "reasons": sorted(reasons),
                "samples": len(mhz), "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- CPU arm --

def oracle_sample_rows(w, seconds: float, orc, q, k, v):
    """Pick evenly spaced rows of head (b=0, all heads) so the oracle runs for ~`seconds`."""
    import numpy as np
    # calibrate on a handful of rows spread over the sequence
    cal = np.linspace(0, w.Nq - 1, 16).astype(np.int32)
    t0 = time.perf_counter()
    orc.attention(q, k, v, w.causal, w.softmax_scale, rows=cal, window=window_of(w))
    dt = max(time.perf_counter() - t0, 1e-4)
    per_row = dt / (len(cal) * w.B * w.Hq)
    n = int(max(8, min(w.Nq, seconds / per_row / (w.B * w.Hq))))
    return np.unique(np.linspace(0, w.Nq - 1, n).astype(np.int32))


def window_of(w):
    return (w.window_left, w.window_right)


def sample_flops(w, rows) -> float:
    """Algorithmic FLOPs of the sampled rows: 4 d per visible (row, key) pair."""
    vis = []
    for r in rows:
        g = int(r) + w.Nk - w.Nq
        hi = w.Nk - 1
        if w.causal:
            hi = min(hi, g)
        if w.window_right >= 0:
            hi = min(hi, g + w.window_right)
        lo = max(0, g - w.window_left) if w.window_left >= 0 else 0
        vis.append(max(0, hi - lo + 1))
    return 4.0 * w.d * w.B * w.Hq * float(sum(vis))


def sampled_errors(o_gpu, lse_gpu, o_ref, lse_ref, rows):
    """Max / mean |O error| and max |LSE error| of the GPU result on the oracle's rows."""
    import numpy as np
    o = np.asarray(o_gpu)[:, rows].astype(np.float64)
    lse = np.asarray(lse_gpu)[:, :, rows].astype(np.float64)
    err = np.abs(o - o_ref)
    fin = np.isfinite(lse_ref)
    lerr = float(np.abs(lse[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    return {"rows_per_head": int(len(rows)), "o_max_abs": float(err.max()),
            "o_mean_abs": float(err.mean()), "lse_max_abs": lerr,
            "lse_neg_inf_pattern_equal": bool(np.array_equal(np.isneginf(lse), np.isneginf(lse_ref)))}


def cpu_oracle_baseline(w, seconds: float, o_gpu=None, lse_gpu=None):
    """Times the fp64 oracle on a bounded row sample; when the GPU's O and LSE
    for the same inputs are given, also reports their errors on those rows."""
    import oracle
    orc = oracle._get()
    q, k, v = (bf16_bits(t) for t in make_qkv(w))
    rows = oracle_sample_rows(w, seconds, orc, q, k, v)
    t0 = time.perf_counter()
    o_ref, lse_ref = orc.attention(q, k, v, w.causal, w.softmax_scale, rows=rows, window=window_of(w))
    dt = time.perf_counter() - t0
    fl = sample_flops(w, rows)
    line = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": orc.default_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} evenly spaced query rows x all {w.B * w.Hq} (batch, head) pairs "
                      f"of {w.name}, every visible key, fp64 C oracle; {fl:.3g} algorithmic FLOP in "
                      f"{dt:.2f} s"}
    if o_gpu is not None:
        try:
            line["parity_of_timed_output"] = sampled_errors(o_gpu, lse_gpu, o_ref, lse_ref, rows)
        except Exception as e:  # the report must never break the benchmark line
            line["parity_of_timed_output"] = {"error": repr(e)}
    return line


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    orc = oracle._get()
    q, k, v = (bf16_bits(t) for t in make_qkv(w))
    per_step = max(0.02, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    rows = oracle_sample_rows(w, per_step, orc, q, k, v)
    fl = sample_flops(w, rows)
    for _ in range(args.warmup):
        orc.attention(q, k, v, w.causal, w.softmax_scale, rows=rows, window=window_of(w))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.attention(q, k, v, w.causal, w.softmax_scale, rows=rows, window=window_of(w))
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    val = fl / dt / 1e12
    sample = (f"{len(rows)} evenly spaced query rows x all {w.B * w.Hq} (batch, head) pairs of "
              f"{w.name} per step, every visible key, fp64 C oracle")
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.gpus, args.schedule),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": orc.default_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def rank_seed(w, rank: int) -> int:
    """Seed of rank `rank`'s share of the job: its KV-head groups of the whole
    problem (``inputs.global_workload``), drawn independently of the other
    ranks' (weak scaling: every rank holds one workload's worth of heads)."""
    return shard_seed(w, rank)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks of the default
    process group (identity when torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def throughput_tflops(w, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank processes one workload per step."""
    return world * w.flops() / (ms_per_step * 1e-3) / 1e12


def workload_config(w, n_gpus, schedule="units"):
    cfg = {"workload": w.name, "schedule": schedule, "description": w.description, "B": w.B,
           "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d, "causal": w.causal}
    if w.windowed:
        cfg["window"] = [w.window_left, w.window_right]
    return {**cfg,
            "softmax_scale": w.softmax_scale, "seed": w.seed,
            "flops_per_step_per_rank": w.flops(),
            "parallelism": (f"KV-head groups split over {n_gpus} ranks (rank r: query heads "
                            f"[r*{w.Hq}, (r+1)*{w.Hq}), KV heads [r*{w.Hkv}, (r+1)*{w.Hkv})), "
                            "no collective on the data path") if n_gpus > 1 else "single GPU",
            "l2": "flushed before every step (256 MiB write), outside the per-step events"}


# ---------------------------------------------------------------- GPU arm --

def run_fa2(args, w):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    import exact_tiled_attention_29_b200 as fa2

    q_h, k_h, v_h = make_qkv(w, seed=rank_seed(w, rank))
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # stream-K takes a scratch workspace, allocated once; calls ordered on one
    # stream reuse it.  It launches the persistent kernel and, when some unit
    # is split, the combine kernel.
    ws = None
    launches_per_step = 1
    # the library runs whole units on persistent CTAs when there are at least
    # two units per SM (the persistent instantiation of the kernel)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    if args.schedule != "units" and w.windowed:
        raise SystemExit("the local-window workloads run the one-block-per-unit schedule only")
    # under "auto" the library's own choice decides which kernels a step runs
    split = args.schedule == "streamk" or (
        args.schedule == "auto" and
        fa2.fa2_schedule_choice(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, sms)[1] == 1)
    persistent = split or fa2.fa2_launch_plan(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d)[1] >= 2 * sms
    if args.schedule != "units":
        ws = fa2.alloc_workspace(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, dev)
    if split:
        _, _, ctas, _ = fa2.fa2_streamk_plan(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, sms)
        launches_per_step = 2 if ctas > 1 else 1

    def call(qq, kk, vv, oo, ll):
        if w.windowed:
            st = fa2.fa2_forward_local(qq, kk, vv, oo, ll, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                                       w.window_left, 0 if w.causal else w.window_right,
                                       w.softmax_scale, stream)
        elif ws is None:
            st = fa2.fa2_forward(qq, kk, vv, oo, ll, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal,
                                 w.softmax_scale, stream)
        elif args.schedule == "auto":
            st = fa2.fa2_forward_auto(qq, kk, vv, oo, ll, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                                      w.causal, w.softmax_scale, ws, ws.numel(), stream)
        else:
            st = fa2.fa2_forward_ws(qq, kk, vv, oo, ll, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                                    w.causal, w.softmax_scale, ws, ws.numel(), stream)
        if st != 0:
            raise fa2.FA2Error(st)

    def forward():
        call(q, k, v, o, lse)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        forward()
    torch.cuda.synchronize()
    dstat = fa2.fa2_debug_status(stream)
    if dstat != 0:
        raise RuntimeError(f"device status {dstat:#x} after warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        forward()
        ends[i].record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    mean_ms = sum(step_ms) / len(step_ms)
    bracket_ms = t_all0.elapsed_time(t_all1)
    dstat = fa2.fa2_debug_status(stream)
    if dstat != 0:
        raise RuntimeError(f"device status {dstat:#x} after the timed region")

    mean_ms, bracket_ms = max_over_ranks([mean_ms, bracket_ms], device=dev)

    # ---- end-to-end through the public API with host buffers ----
    # The job is cut into its batch elements (contiguous slices of every
    # tensor): H2D of element b + 1 on one stream, the C-ABI call on element b
    # on the launch stream, D2H of element b - 1 on a third, so the transfers
    # over the host link overlap each other and the kernels.
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
        op = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lp = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        od, ld = torch.empty_like(o), torch.empty_like(lse)
        n_e2e = max(3, min(args.steps, 50))
        h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        chunks = w.B

        def call_b(b, qq, kk, vv, oo, ll):
            if w.windowed:
                st = fa2.fa2_forward_local(qq, kk, vv, oo, ll, 1, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                                           w.window_left, 0 if w.causal else w.window_right,
                                           w.softmax_scale, stream)
            elif ws is None:
                st = fa2.fa2_forward(qq, kk, vv, oo, ll, 1, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal,
                                     w.softmax_scale, stream)
            elif args.schedule == "auto":
                st = fa2.fa2_forward_auto(qq, kk, vv, oo, ll, 1, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                                          w.causal, w.softmax_scale, ws, ws.numel(), stream)
            else:
                st = fa2.fa2_forward_ws(qq, kk, vv, oo, ll, 1, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                                        w.causal, w.softmax_scale, ws, ws.numel(), stream)
            if st != 0:
                raise fa2.FA2Error(st)

        done_in = [torch.cuda.Event() for _ in range(chunks)]
        done_out = [torch.cuda.Event() for _ in range(chunks)]

        def e2e_step():
            if chunks == 1:  # one stream, in order, as a caller would
                qd.copy_(qp, non_blocking=True)
                kd.copy_(kp, non_blocking=True)
                vd.copy_(vp, non_blocking=True)
                call_b(0, qd, kd, vd, od, ld)
                op.copy_(od, non_blocking=True)
                lp.copy_(ld, non_blocking=True)
                return
            with torch.cuda.stream(h2d_stream):
                h2d_stream.wait_stream(stream)  # the previous step's kernels read these buffers
                for b in range(chunks):
                    qd[b].copy_(qp[b], non_blocking=True)
                    kd[b].copy_(kp[b], non_blocking=True)
                    vd[b].copy_(vp[b], non_blocking=True)
                    done_in[b].record(h2d_stream)
            for b in range(chunks):
                stream.wait_event(done_in[b])
                call_b(b, qd[b], kd[b], vd[b], od[b], ld[b])
                done_out[b].record(stream)
                d2h_stream.wait_event(done_out[b])
                with torch.cuda.stream(d2h_stream):
                    op[b].copy_(od[b], non_blocking=True)
                    lp[b].copy_(ld[b], non_blocking=True)
            stream.wait_stream(d2h_stream)  # the step ends when its results are on the host

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks([e0.elapsed_time(e1) / n_e2e], device=dev)[0]
        if not torch.isfinite(lp).any():
            raise RuntimeError("e2e produced no finite LSE")
        # the pipelined run returns the device-timed run's bits
        same = bool(torch.equal(op, o.cpu()) and torch.equal(lp, lse.cpu()))
        h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
        d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()
        e2e = {"value": throughput_tflops(w, world, e_ms), "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": n_e2e, "equals_device_run": same,
               "chunks": f"{chunks} (batch elements), H2D / compute / D2H on three streams"}

    value = throughput_tflops(w, world, mean_ms)
    line = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        peak = float(peaks["bf16_tflops"])
        achieved = w.flops() / (mean_ms * 1e-3) / 1e12
        traffic = profiled_traffic(w.name)
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            # rank 0's inputs are make_qkv(w) (seed w.seed): the timed output can be checked
            cpu = cpu_oracle_baseline(w, args.cpu_seconds, o_gpu=o.float().cpu().numpy(),
                                      lse_gpu=lse.cpu().numpy())
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, world, args.schedule),
            "pct_of_peak": 100.0 * achieved / peak,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"bf16_tflops (burst, kernel timed alone), {peak_src}",
                         "frac_of_sustained": achieved / float(peaks["bf16_tflops_sustained"]),
                         "kernel": f"fa2_fwd_kernel<{w.d}, {'true' if persistent else 'false'}>"
                                   + (" + fa2_combine_kernel (timed together)" if launches_per_step > 1 else "")},
            "hbm_gbs_compulsory": w.compulsory_bytes() / (mean_ms * 1e-3) / 1e9,
            "bracket_ms_per_step_incl_flush": bracket_ms / args.steps,
            "gpu_launches": args.steps * launches_per_step,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "kernel_source_sha256_16": kernel_source_hash(),
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def run_fa2_backward(args, w):
    """Times fa2_backward (its three kernels) on one GPU; same timing rules as the forward."""
    import torch
    import exact_tiled_attention_29_b200 as fa2

    if int(os.environ.get("WORLD_SIZE", "1")) > 1 or w.windowed:
        raise SystemExit("--direction bwd runs on one GPU, without a window")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    q_h, k_h, v_h = make_qkv(w)
    g_h = torch.randn(q_h.shape, generator=torch.Generator().manual_seed(w.seed + 7)).to(torch.bfloat16)
    q, k, v, g = (t.to(dev) for t in (q_h, k_h, v_h, g_h))
    stream = torch.cuda.current_stream(dev)
    o, lse = fa2.attention(q, k, v, causal=w.causal, softmax_scale=w.softmax_scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa2.fa2_backward_workspace_size(w.B, w.Hq, w.Nq, w.d), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(qq, kk, vv, oo, ll, gg, a, b_, c):
        st = fa2.fa2_backward(qq, kk, vv, oo, ll, gg, a, b_, c, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                              w.causal, w.softmax_scale, ws, ws.numel(), stream)
        if st != 0:
            raise fa2.FA2Error(st, "fa2_backward")

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step(q, k, v, o, lse, g, dq, dk, dv)
    torch.cuda.synchronize()
    if fa2.fa2_debug_status(stream) != 0:
        raise RuntimeError("device status after warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    sampler.start()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step(q, k, v, o, lse, g, dq, dk, dv)
        ends[i].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    mean_ms = sum(s_.elapsed_time(e) for s_, e in zip(starts, ends)) / args.steps
    if fa2.fa2_debug_status(stream) != 0:
        raise RuntimeError("device status after the timed region")
    flops = 2.5 * w.flops()
    e2e = None
    if not args.no_e2e:
        hosts = [t.cpu().pin_memory() for t in (q, k, v, o, lse, g)]
        devs = [torch.empty_like(t) for t in (q, k, v, o, lse, g)]
        outs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]
        n_e2e = max(3, min(args.steps, 30))

        def e2e_step():
            for d_, h_ in zip(devs, hosts):
                d_.copy_(h_, non_blocking=True)
            step(*devs, dq, dk, dv)
            for h_, d_ in zip(outs_h, (dq, dk, dv)):
                h_.copy_(d_, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = e0.elapsed_time(e1) / n_e2e
        e2e = {"value": flops / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hosts),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs_h),
               "steps": n_e2e}
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        sub = w.with_(B=1, Hq=w.Hq // w.Hkv, Hkv=1, Nq=min(w.Nq, 1024), Nk=min(w.Nk, 1024))
        sq, sk, sv = (bf16_bits(t) for t in make_qkv(sub))
        sg = bf16_bits(torch.randn((sub.B, sub.Nq, sub.Hq, sub.d),
                                   generator=torch.Generator().manual_seed(1)).to(torch.bfloat16))
        t0 = time.perf_counter()
        oracle.backward(sq, sk, sv, sg, sub.causal, sub.softmax_scale)
        dt = time.perf_counter() - t0
        cpu = {"value": 2.5 * sub.flops() / dt / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": f"backward of one KV-head group (B=1, Hq={sub.Hq}, Hkv=1) at "
                         f"N={sub.Nq}, d={sub.d}, causal={sub.causal}: fp64 C oracle, one group "
                         f"per thread; {2.5 * sub.flops():.3g} algorithmic FLOP in {dt:.2f} s"}
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (mean_ms * 1e-3) / 1e12
    line = {"metric": "attention backward TFLOP/s (2.5x forward FLOPs)", "value": achieved,
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": {**workload_config(w, 1), "direction": "bwd"},
            "pct_of_peak": 100.0 * achieved / peak,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(w.name, "fa2_bwd_kernel"),
                         "peak_source": f"bf16_tflops (burst), {peak_src}",
                         "kernel": f"fa2_bwd_kernel<{w.d}> + prep + dq rounding (timed together)"},
            "gpu_launches": 3 * args.steps, "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu,
            "kernel_source_sha256_16": kernel_source_hash("fa2_bwd_kernel")}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    w = ALL_WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.direction == "bwd":
        return run_fa2_backward(args, w)
    return run_fa2(args, w)


if __name__ == "__main__":
    sys.exit(main())
