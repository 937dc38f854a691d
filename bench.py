#!/usr/bin/env python
"""Benchmark of the MSA hot path on B200: one step = the index branch
(msa_index_topk) and the sparse branch (msa_sparse_attn: inversion,
attention, log-sum-exp combine) over one batch of synthetic input.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl msa|reference]

Prints ONE JSON line (rank 0).  Multi-GPU (torchrun, one process per GPU):
every rank processes its own sequences of the workload (independent
problems, no data-path collective): weak scaling; the step time is the max
over ranks.  ``--impl reference`` times the CPU oracle on this host's cores
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import threading
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MSA prefill & decode tokens/s at 1 B200; % of HBM / bf16 tensor roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "prefill_T65536"
SECONDARY_DECODE = "decode_4x1048576"
L2_BYTES = 126 << 20  # B200 L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the secondary decode line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


# ---------------------------------------------------------------- peaks
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons (200 ms)."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self, ready_timeout: float = 20.0):
        """Start sampling; returns once the first sample has been printed, so
        nvidia-smi's own start-up (which can stall driver calls of other
        processes) lies before the timed region."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        first = threading.Event()

        def reader():
            for ln in self.proc.stdout:
                self.lines.append(ln)
                first.set()
            first.set()

        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        first.wait(ready_timeout)

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.thread.join(timeout=5)
        out = "".join(self.lines)
        rows = []
        for ln in out.strip().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]),
                             "power": float(parts[3]) if parts[3] not in ("[N/A]", "N/A") else 0.0,
                             "hw": parts[5], "hw_thermal": parts[6], "sw_thermal": parts[7],
                             "power_cap": parts[8]})
            except ValueError:
                continue
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("power_cap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------- work model
def attended_pairs(ids, w):
    """Number of (query, key) pairs the sparse branch attends (exact)."""
    import torch
    rows = w.Bt * w.n_q
    t = (w.T - w.n_q) + torch.arange(rows, device=ids.device) % w.n_q
    j = ids.reshape(rows, w.K).long()
    lo = j * w.block
    hi = torch.minimum(torch.minimum(lo + w.block, torch.full_like(lo, w.T)), t[:, None] + 1)
    n = torch.clamp(hi - lo, min=0)
    n = torch.where(j >= 0, n, torch.zeros_like(n))
    return int(n.sum().item())


def index_macs(w):
    """Multiply-adds of the index branch: every key of every candidate block."""
    total = 0
    for i in range(w.n_q):
        t = w.T - w.n_q + i
        total += (t // w.block) * w.block
    return total * w.d_idx * w.Bt


def decode_bytes(w, ids):
    """Algorithmic HBM bytes of one decode step (per stage)."""
    own = (w.T - 1) // w.block
    scan = w.Bt * own * w.block * w.d_idx * 2 + w.Bt * w.d_idx * 2
    pairs = attended_pairs(ids, w)  # keys read per sequence summed (1 query per sequence)
    kv = pairs * w.Hkv * w.d * 2 * 2 + w.Bt * w.Hq * w.d * 2
    return scan, kv


# ---------------------------------------------------------------- ranks
def rank_seed(w, rank: int) -> int:
    """Weak scaling: rank r runs its own Bt sequences of the workload, drawn
    with seed w.seed + r (independent problems; no data-path collective)."""
    return w.seed + rank


def max_over_ranks(values, world: int, device):
    """Element-wise maximum of per-rank floats (step times) over all ranks;
    every rank takes part and gets the result."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(w, ms: float, world: int) -> float:
    """Whole-job tokens/s: the query tokens all ranks processed in one step
    divided by the slowest rank's step time."""
    return w.Bt * w.n_q * world / (ms / 1e3)


# ---------------------------------------------------------------- MSA arm
def run_msa(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from block_sparse_long_05_b200 import msa
    from block_sparse_long_05_b200.inputs import WORKLOADS, make_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    peaks, peak_src = load_peaks()

    def measure(w, steps, warmup, with_e2e):
        x = make_inputs(w, device=dev, seed=rank_seed(w, rank))
        ws = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K,
                                     device=dev)
        ids = torch.empty((w.Bt, w.n_q, w.K), dtype=torch.int32, device=dev)
        out = torch.empty((w.Bt, w.n_q, w.Hq, w.d), dtype=torch.float32, device=dev)
        lse = torch.empty((w.Bt, w.n_q, w.Hq), dtype=torch.float32, device=dev)
        n_idx_stages = 2 if w.is_decode else 1

        def step(ev=None):
            msa.index_topk(x["q_idx"], x["k_idx"], w.block, w.K, ws, ids=ids,
                           events=ev[0] if ev else None)
            msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws, out=out, lse=lse,
                            events=ev[1] if ev else None)

        for _ in range(warmup):
            step()
        st = msa.device_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {msa.status_string(st)}")
        # bytes one step touches; below twice the L2 size, L2 is flushed
        # between timed steps (a 256 MB write outside each step's events)
        if w.is_decode:
            touched = sum(decode_bytes(w, ids))
        else:
            touched = (x["q"].numel() + x["k"].numel() + x["v"].numel() + x["q_idx"].numel() +
                       x["k_idx"].numel()) * 2 + w.Bt * w.n_q * w.K * w.Hq * (w.d * 2 + 4) + \
                out.numel() * 4
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) \
            if touched < 2 * L2_BYTES else None
        E = torch.cuda.Event
        evs = []
        for _ in range(steps):
            a = {i: (E(enable_timing=True), E(enable_timing=True)) for i in range(n_idx_stages)}
            b = {i: (E(enable_timing=True), E(enable_timing=True))
                 for i in ((1, 2) if w.is_decode else (0, 1, 2))}
            evs.append((a, b))
        for a, b in evs:  # materialise the events outside the timed region
            for d_ in (a, b):
                for s_, e_ in d_.values():
                    s_.record()
                    e_.record()
        t0, t1 = E(enable_timing=True), E(enable_timing=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clocks = ClockSampler(local_rank)
        clocks.start()
        time.sleep(0.3)
        if flush is None:
            t0.record()
            for _ in range(steps):
                step()
            t1.record()
        else:
            per_step = [(E(enable_timing=True), E(enable_timing=True)) for _ in range(steps)]
            for s_, e_ in per_step:
                flush.fill_(1)
                s_.record()
                step()
                e_.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        clk = clocks.stop()
        if flush is None:
            ms = t0.elapsed_time(t1) / steps
        else:
            ms = sum(s_.elapsed_time(e_) for s_, e_ in per_step) / steps
        st = msa.device_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {msa.status_string(st)}")
        # stage times from a second, separate pass (events between the stages
        # would stop consecutive kernels from overlapping their launch)
        for ev in evs:
            if flush is not None:
                flush.fill_(1)
            step(ev)
        torch.cuda.synchronize()
        stage_ms = {}
        for a, b in evs:
            for i, (s_, e_) in a.items():
                stage_ms[f"index{i}"] = stage_ms.get(f"index{i}", 0.0) + s_.elapsed_time(e_) / steps
            for i, (s_, e_) in b.items():
                stage_ms[f"attn{i}"] = stage_ms.get(f"attn{i}", 0.0) + s_.elapsed_time(e_) / steps
        ms = max_over_ranks([ms], world, dev)[0]
        launches = (1 + 5 + 1 + 1) if not w.is_decode else \
            ((1 if (w.T - 1) // w.block > 0 else 0) + 1 + 1 + 1)
        res = {"ms": ms, "stage_ms": stage_ms, "clocks": clk, "launches": launches * steps,
               "l2": ("inputs and partials larger than L2 (126 MB): no flush needed"
                      if flush is None else
                      "L2 flushed between timed steps (256 MB write outside each step's events; "
                      "the step time is the mean of per-step events)")}
        del flush

        # e2e through the public API with host buffers (pinned), copies timed.
        # Serial: each step uploads its inputs, runs, and reads its result back.
        # Pipelined (the reported value): two device buffer sets and three
        # streams, so step i+1's upload and step i-1's download (PCIe is full
        # duplex) overlap step i's kernels, as a stream of requests would run.
        if with_e2e:
            hx = {k: v.cpu().pin_memory() for k, v in x.items()}
            hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
            hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
            h2d = sum(v.numel() * v.element_size() for v in hx.values())
            d2h = hout.numel() * 4 + hlse.numel() * 4
            e_steps = max(1, min(steps, 5))

            def e2e_step():
                for k_, v_ in hx.items():
                    x[k_].copy_(v_, non_blocking=True)
                step()
                hout.copy_(out, non_blocking=True)
                hlse.copy_(lse, non_blocking=True)

            e2e_step()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a0, a1 = E(enable_timing=True), E(enable_timing=True)
            a0.record()
            for _ in range(e_steps):
                e2e_step()
            a1.record()
            torch.cuda.synchronize()
            serial_ms = a0.elapsed_time(a1) / e_steps

            # pipelined: buffer set i % 2 holds step i's inputs and outputs
            sets = [(x, out, lse),
                    ({k: torch.empty_like(v) for k, v in x.items()}, torch.empty_like(out),
                     torch.empty_like(lse))]
            s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
            p_steps = max(4, min(steps, 8)) + 2
            ev_in = [E() for _ in range(p_steps)]
            ev_run = [E() for _ in range(p_steps)]
            ev_out = [E() for _ in range(p_steps)]

            def pipelined(i):
                xs, os_, ls = sets[i % 2]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_run[i - 2])      # step i-2 has read this input set
                    for k_, v_ in hx.items():
                        xs[k_].copy_(v_, non_blocking=True)
                    ev_in[i].record(s_in)
                s_run.wait_event(ev_in[i])
                if i >= 2:
                    s_run.wait_event(ev_out[i - 2])         # step i-2's result has been read back
                msa.index_topk(xs["q_idx"], xs["k_idx"], w.block, w.K, ws, ids=ids, stream=s_run)
                msa.sparse_attn(xs["q"], xs["k"], xs["v"], ids, w.block, ws, out=os_, lse=ls,
                                stream=s_run)
                ev_run[i].record(s_run)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_run[i])
                    hout.copy_(os_, non_blocking=True)
                    hlse.copy_(ls, non_blocking=True)
                    ev_out[i].record(s_out)

            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            b0, b1 = E(enable_timing=True), E(enable_timing=True)
            b0.record(s_in)
            for i in range(p_steps):
                pipelined(i)
            b1.record(s_out)
            torch.cuda.synchronize()
            ems = b0.elapsed_time(b1) / p_steps
            if msa.device_status(ws) != 0:
                raise RuntimeError("device status after the pipelined e2e steps")
            ems, serial_ms = max_over_ranks([ems, serial_ms], world, dev)
            res["e2e"] = {"ms": ems, "serial_ms": serial_ms, "h2d": h2d, "d2h": d2h,
                          "steps": p_steps}
            del sets
        res["pairs"] = attended_pairs(ids, w)
        res["ids"] = ids
        del x, ws, out, lse
        return res

    r = measure(w, args.steps, args.warmup, not args.no_e2e)
    tokens_per_step = w.Bt * w.n_q * world
    value = job_throughput(w, r["ms"], world)

    # roofline of the dominant kernel
    sm = r["stage_ms"]
    if w.is_decode:
        scan_b, kv_b = decode_bytes(w, r["ids"])
        cands = {"index0": ("hbm", scan_b), "attn1": ("hbm", kv_b)}
    else:
        idx_flops = 2.0 * index_macs(w)
        attn_flops = 4.0 * w.d * w.Hq * r["pairs"]
        cands = {"index0": ("tensor", idx_flops), "attn1": ("tensor", attn_flops)}
    dom = max(cands, key=lambda k: sm.get(k, 0.0))
    bound, work = cands[dom]
    kern_ms = sm[dom]
    kernel_names = {"index0": "prefill_index_kernel" if not w.is_decode else "decode_index_scan_kernel",
                    "attn1": ("prefill_attn_resident_kernel" if w.block <= 128 else "prefill_attn_streamed_kernel")
                    if not w.is_decode else "decode_attn_kernel"}
    if bound == "tensor":
        achieved = work / (kern_ms / 1e3) / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
        unit = "TFLOP/s"
        peak_note = f"bf16 dense, sustained (kernel timed inside the step loop), of {peak_src}"
    else:
        achieved = work / (kern_ms / 1e3) / 1e9
        peak = float(peaks["hbm_gbs"])
        unit = "GB/s"
        peak_note = f"HBM copy bandwidth, of {peak_src}"
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tr = json.load(f)
        ent = tr.get(f"{kernel_names[dom]}@{w.name}")
        if ent and ent.get("valid", True):
            traffic = ent["bytes_per_launch"]

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "Bt_per_gpu": w.Bt, "n_q": w.n_q, "T": w.T, "Hq": w.Hq,
                   "Hkv": w.Hkv, "d": w.d, "block": w.block, "K": w.K, "d_idx": w.d_idx,
                   "global_batch": w.Bt * world, "seq_len": w.T, "parallelism": f"dp{world}",
                   "l2": r["l2"]},
        "gpu_launches": r["launches"],
        "stage_ms": {k: round(v, 4) for k, v in sm.items()},
        "roofline": {"bound": bound, "kernel": kernel_names[dom], "achieved": achieved,
                     "peak": peak, "unit": unit, "frac": achieved / peak, "traffic": traffic,
                     "work_per_launch": work, "peak_note": peak_note},
    }
    if r["clocks"]:
        line["clocks"] = r["clocks"]
    if "e2e" in r:
        e = r["e2e"]
        line["e2e"] = {"value": tokens_per_step / (e["ms"] / 1e3), "unit": UNIT,
                       "ms_per_step": e["ms"], "h2d_bytes_per_step": e["h2d"],
                       "d2h_bytes_per_step": e["d2h"],
                       "pipelined": f"{e['steps']} steps; upload of step i+1 and download of "
                                    "step i-1 overlap step i (two device buffer sets, three "
                                    "streams, pinned host buffers)",
                       "serial_ms_per_step": e["serial_ms"],
                       "serial_value": tokens_per_step / (e["serial_ms"] / 1e3)}

    # secondary: the 1M-context decode step (HBM-bound), same protocol
    if not args.no_decode and not w.is_decode and world == 1:
        wd = WORKLOADS[SECONDARY_DECODE]
        rd = measure(wd, max(args.steps, 20), max(args.warmup, 3), False)
        scan_b, kv_b = decode_bytes(wd, rd["ids"])
        smd = rd["stage_ms"]
        step_b = scan_b + kv_b
        line["decode"] = {
            "workload": wd.name, "value": wd.Bt / (rd["ms"] / 1e3), "unit": UNIT,
            "ms_per_step": rd["ms"], "stage_ms": {k: round(v, 4) for k, v in smd.items()},
            "step_bytes": step_b,
            "step_hbm_frac": step_b / (rd["ms"] / 1e3) / 1e9 / float(peaks["hbm_gbs"]),
            "scan_gbs": scan_b / (smd["index0"] / 1e3) / 1e9,
            "scan_frac": scan_b / (smd["index0"] / 1e3) / 1e9 / float(peaks["hbm_gbs"]),
        }

    # decode step at this prefill workload's context: one sequence of T keys,
    # same heads, block, K and index dim (a failure here is reported in the
    # object and leaves the line above intact)
    if not args.no_decode and not w.is_decode and world == 1:
        from block_sparse_long_05_b200.inputs import Workload
        wt = Workload(f"decode_1x{w.T}", 1, 1, w.T, w.Hq, w.Hkv, w.d, w.block, w.K, w.d_idx)
        try:
            rt = measure(wt, max(args.steps, 20), max(args.warmup, 3), False)
            scan_b, kv_b = decode_bytes(wt, rt["ids"])
            line["decode_at_T"] = {
                "workload": wt.name, "value": 1 / (rt["ms"] / 1e3), "unit": UNIT,
                "ms_per_step": rt["ms"],
                "stage_ms": {k: round(v, 4) for k, v in rt["stage_ms"].items()},
                "step_bytes": scan_b + kv_b,
                "step_hbm_frac": (scan_b + kv_b) / (rt["ms"] / 1e3) / 1e9 / float(peaks["hbm_gbs"]),
            }
        except Exception as e:  # noqa: BLE001 -- recorded, not hidden
            line["decode_at_T"] = {"workload": wt.name, "error": f"{type(e).__name__}: {e}"[:300]}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    return line


# ---------------------------------------------------------------- oracle arm
def oracle_sample(w, rows, x):
    from oracle import oracle
    ids = oracle.index_topk(x["q_idx"], x["k_idx"], w.Bt, w.n_q, w.T, w.d_idx, w.block, w.K,
                            rows=rows)
    oracle.sparse_attn(x["q"], x["k"], x["v"], ids, w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.block,
                       w.K, rows=rows)


def cpu_inputs(w):
    from block_sparse_long_05_b200.inputs import make_inputs
    return make_inputs(w, device="cpu")


def cpu_baseline(w, seconds):
    """The oracle as it stands, on this host's cores, on a bounded sample of
    query rows of the same workload (index + attention per row)."""
    import numpy as np
    from block_sparse_long_05_b200.inputs import sample_rows
    from oracle import oracle
    x = cpu_inputs(w)
    probe = sample_rows(w, 8).numpy()
    t = time.perf_counter()
    oracle_sample(w, probe, x)
    per_row = (time.perf_counter() - t) / len(probe)
    n = int(max(8, min(w.Bt * w.n_q, seconds / max(per_row, 1e-6))))
    rows = np.sort(sample_rows(w, n).numpy())
    t = time.perf_counter()
    oracle_sample(w, rows, x)
    dt = time.perf_counter() - t
    return {"value": len(rows) / dt, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} query rows of {w.name} (uniform, seed 1), index branch + "
                      f"sparse branch per row, {dt:.1f} s; tokens/s = rows / time"}


def run_reference(args):
    import numpy as np
    from block_sparse_long_05_b200.inputs import WORKLOADS, sample_rows
    from oracle import oracle
    w = WORKLOADS[args.workload]
    x = cpu_inputs(w)
    probe = sample_rows(w, 4).numpy()
    t = time.perf_counter()
    oracle_sample(w, probe, x)
    per_row = (time.perf_counter() - t) / len(probe)
    budget = 150.0 / max(1, args.steps + args.warmup)  # whole run within a few minutes
    n = int(max(4, min(w.Bt * w.n_q, budget / max(per_row, 1e-6))))
    rows = np.sort(sample_rows(w, n, seed=3).numpy())
    for _ in range(args.warmup):
        oracle_sample(w, rows, x)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(w, rows, x)
    dt = (time.perf_counter() - t) / args.steps
    value = len(rows) / dt
    sample = (f"{len(rows)} query rows of {w.name} per step (uniform, seed 3), index branch + "
              f"sparse branch per row")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name},
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle",
                             "cores": oracle.num_threads(), "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_msa(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
