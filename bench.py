#!/usr/bin/env python
"""Benchmark of the MSA hot path on B200: one step = the index branch
(msa_index_topk) and the sparse branch (msa_sparse_attn: inversion,
attention, log-sum-exp combine) over one batch of synthetic input.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl msa|reference] [--only]

Prints ONE JSON line (rank 0).  The headline is the 256K-token long prefill
(1 x 262144, 64 query heads, block 512, top-8); at one GPU the line also
carries every workload of the hot path ("configs": the tiny, 64K and 256K
prefills, the 32 x 128K and 4 x 1M decode steps), each with its step time,
stage times and roofline (--only: the headline alone).

Multi-GPU (torchrun, one process per GPU):
  * one long prefill (Bt = 1): kv-head sharding.  Each rank computes the
    index branch for its range of query rows, the ids are all-gathered
    (NCCL), and each rank runs the sparse branch for its kv heads over every
    row: strong scaling, the step time is the max over ranks.
  * decode / batched workloads: every rank its own sequences, no data-path
    collective: weak scaling.
``--impl reference`` times the CPU oracle on this host's cores on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import contextlib
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
DEFAULT_WORKLOAD = "long_prefill_T262144"
CONFIGS = ("tiny_prefill_T4096", "prefill_T65536", "decode_32x131072", "long_prefill_T262144",
           "decode_4x1048576")
L2_BYTES = 126 << 20  # B200 L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--only", action="store_true", help="the headline workload alone")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode step at each prefill workload's context")
    ap.add_argument("--no-int8", action="store_true",
                    help="skip the variant of each step with the int8 index path")
    ap.add_argument("--no-paged", action="store_true",
                    help="skip the paged-KV variant of each decode step")
    ap.add_argument("--no-min-ws", action="store_true",
                    help="skip the prefill step with the minimum workspace")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample (headline)")
    return ap.parse_args(argv)


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


def index_macs(w, r0=0, r1=None):
    """Multiply-adds of the index branch for query rows [r0, r1) of every
    sequence: every key of every candidate block (blocks j < own(t))."""
    import torch
    r1 = w.n_q if r1 is None else r1
    t = torch.arange(r0, r1, dtype=torch.int64) + (w.T - w.n_q)
    total = int(torch.div(t, w.block, rounding_mode="floor").sum().item()) * w.block
    return total * w.d_idx * w.Bt


def decode_bytes(w, ids, Hq=None, Hkv=None):
    """Algorithmic HBM bytes of one decode step: (k_idx scan, selected K/V
    rows + q); Hq, Hkv: the heads this rank holds (default all)."""
    Hq = w.Hq if Hq is None else Hq
    Hkv = w.Hkv if Hkv is None else Hkv
    own = (w.T - 1) // w.block
    scan = w.Bt * own * w.block * w.d_idx * 2 + w.Bt * w.d_idx * 2
    pairs = attended_pairs(ids, w)  # keys read per sequence summed (1 query per sequence)
    kv = pairs * Hkv * w.d * 2 * 2 + w.Bt * Hq * w.d * 2
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
class Problem:
    """One rank's share of one workload: its device inputs and outputs, the
    workspace, and the library calls of one step.

    mode "whole": the full workload (one GPU); "seq": this rank's own
    sequences (seed w.seed + rank, weak scaling); "heads": one long prefill
    sharded by kv head (the index branch split by query rows, ids
    all-gathered; see block_sparse_long_05_b200.shard)."""

    def __init__(self, w, dev, rank, world, mode):
        import torch
        from block_sparse_long_05_b200 import msa, shard
        from block_sparse_long_05_b200.inputs import make_inputs
        self.w, self.dev, self.rank, self.world, self.mode = w, dev, rank, world, mode
        self.r0, self.r1 = 0, w.n_q
        self.hk0, self.hk1 = 0, w.Hkv
        if mode == "heads":
            full = make_inputs(w, device=dev, seed=w.seed)  # the same problem on every rank
            self.hk0, self.hk1 = shard.head_range(w.Hkv, world, rank)
            self.ranges = shard.index_row_ranges(w.n_q, w.T, w.block, world)
            self.r0, self.r1 = self.ranges[rank]
            qi, ki, self.T_cut = shard.row_slice_args(full["q_idx"], full["k_idx"], w.T,
                                                      self.r0, self.r1)
            G = w.G
            self.x = {"q_idx": qi.contiguous(), "k_idx": ki.contiguous(),
                      "q": full["q"][:, :, self.hk0 * G:self.hk1 * G].contiguous(),
                      "k": full["k"][:, :, self.hk0:self.hk1].contiguous(),
                      "v": full["v"][:, :, self.hk0:self.hk1].contiguous()}
            del full
            self.ids_local = torch.empty((1, self.r1 - self.r0, w.K), dtype=torch.int32,
                                         device=dev)
        else:
            seed = rank_seed(w, rank) if mode == "seq" else w.seed
            self.x = make_inputs(w, device=dev, seed=seed)
        self.int8_index = False  # index branch on int8 copies of the (integer) index keys
        self.paged = False       # decode through the paged entry points (use_paged)
        self.Hq = (self.hk1 - self.hk0) * w.G
        self.Hkv = self.hk1 - self.hk0
        # prefill: the one-pass workspace (all of this rank's kv heads per
        # attention launch), the fastest choice when the memory is there
        self.kv_group = None if w.is_decode else self.Hkv
        self.ws = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, self.Hq, self.Hkv, w.d, w.d_idx,
                                          w.block, w.K, device=dev, kv_group=self.kv_group)
        self.ids = torch.empty((w.Bt, w.n_q, w.K), dtype=torch.int32, device=dev)
        self.y = {"out": torch.empty((w.Bt, w.n_q, self.Hq, w.d), dtype=torch.float32, device=dev),
                  "lse": torch.empty((w.Bt, w.n_q, self.Hq), dtype=torch.float32, device=dev)}

    @property
    def launches_per_step(self):
        """Kernels of this library one step launches."""
        w = self.w
        if w.is_decode:  # scan (when there are blocks before own), select, attention, combine
            return (1 if (w.T - 1) // w.block > 0 else 0) + 3
        # index, 5 inversion kernels (+3 for the own-block work list when
        # blocks are longer than 128 keys), per kv-head group the attention
        # launch(es) and the combine
        own = w.block > 128
        groups = self.Hkv // (self.kv_group or self.Hkv)
        return ((1 if self.r1 > self.r0 else 0) + 5 + (3 if own else 0) +
                groups * ((2 if own else 1) + 1))

    def stage_keys(self):
        w = self.w
        idx = (0, 1) if w.is_decode else (0,)
        attn = (1, 2) if w.is_decode else (0, 1, 2)
        return idx, attn

    def step(self, x=None, y=None, stream=None, ev=None):
        """One step on buffers x (inputs) and y (out, lse); ev = (index
        stage events, attention stage events, gather events) or None."""
        import torch
        from block_sparse_long_05_b200 import msa, shard
        w = self.w
        x = x or self.x
        y = y or self.y
        ev_idx, ev_attn, ev_gather = ev if ev else (None, None, None)
        if self.paged:  # decode over a permuted page store (no stage events)
            msa.index_topk_paged(x["q_idx"], x["k_idx_pages"], x["page_table"], w.T, w.K,
                                 self.ws, ids=self.ids, stream=stream)
            msa.sparse_attn_paged(x["q"], x["k_pages"], x["v_pages"], x["page_table"], w.T,
                                  self.ids, self.ws, out=y["out"], lse=y["lse"], stream=stream)
            return
        index = msa.index_topk
        qi, ki = x["q_idx"], x["k_idx"]
        if self.int8_index:
            index, qi, ki = msa.index_topk_i8, x["q_idx8"], x["k_idx8"]
        if self.mode == "heads":
            if self.r1 > self.r0:
                index(qi, ki, w.block, w.K, self.ws, ids=self.ids_local, stream=stream,
                      events=ev_idx)
            ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
            with ctx:
                if ev_gather:
                    ev_gather[0].record()
                full = shard.gather_rows(self.ids_local.view(self.r1 - self.r0, w.K), self.ranges)
                self.ids.view(w.n_q, w.K).copy_(full)
                if ev_gather:
                    ev_gather[1].record()
        else:
            index(qi, ki, w.block, w.K, self.ws, ids=self.ids, stream=stream, events=ev_idx)
        msa.sparse_attn(x["q"], x["k"], x["v"], self.ids, w.block, self.ws, out=y["out"],
                        lse=y["lse"], stream=stream, events=ev_attn)

    def use_int8_index(self):
        """Switch the step to the int8 index path (msa_index_topk_i8) on int8
        copies of the index keys (exact: the keys are small integers)."""
        import torch
        self.x["q_idx8"] = self.x["q_idx"].to(torch.int8)
        self.x["k_idx8"] = self.x["k_idx"].to(torch.int8)
        self.int8_index = True

    def use_paged(self, seed=5):
        """Switch the decode step to the paged entry points: k_idx, K and V
        scattered block by block into a page store in a seeded random order,
        with the page table [Bt, N] that maps them back."""
        import torch
        w = self.w
        N = w.n_blocks
        if not w.is_decode or w.T % w.block:
            raise ValueError("paged timing covers decode workloads of whole blocks")
        g = torch.Generator(device=self.dev)
        g.manual_seed(seed)
        perm = torch.randperm(w.Bt * N, generator=g, device=self.dev)

        def scatter(t):
            src = t.view(w.Bt * N, w.block, *t.shape[2:])
            out = torch.empty_like(src)
            out[perm] = src
            return out

        for k in ("k_idx", "k", "v"):
            self.x[k + "_pages"] = scatter(self.x[k])
        self.x["page_table"] = perm.view(w.Bt, N).to(torch.int32)
        self.paged = True

    def touched_bytes(self):
        """Bytes one step reads and writes (to decide whether L2 must be
        flushed between timed steps)."""
        w = self.w
        if w.is_decode:
            return sum(decode_bytes(w, self.ids, self.Hq, self.Hkv))
        inputs = sum(t.numel() * t.element_size() for k, t in self.x.items()
                     if k in ("q", "k", "v", "q_idx", "k_idx"))
        partials = w.Bt * w.n_q * w.K * self.Hq * (w.d * 2 + 4)
        return inputs + partials + self.y["out"].numel() * 4

    def free(self):
        del self.x, self.y, self.ws, self.ids


def measure(prob, steps, warmup, with_e2e):
    """Time `steps` steps of `prob` (after `warmup`), then the per-stage
    times in a second pass, then (with_e2e) the end-to-end variant with
    host buffers.  Every rank takes the same collective steps."""
    import torch
    import torch.distributed as dist
    from block_sparse_long_05_b200 import msa
    w, world, dev = prob.w, prob.world, prob.dev
    for _ in range(warmup):
        prob.step()
    st = msa.device_status(prob.ws)
    if st != 0:
        raise RuntimeError(f"{w.name}: device status {msa.status_string(st)}")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) \
        if prob.touched_bytes() < 2 * L2_BYTES else None
    E = torch.cuda.Event
    idx_keys, attn_keys = prob.stage_keys()
    evs = []
    for _ in range(steps):
        a = {i: (E(enable_timing=True), E(enable_timing=True)) for i in idx_keys}
        b = {i: (E(enable_timing=True), E(enable_timing=True)) for i in attn_keys}
        g = (E(enable_timing=True), E(enable_timing=True)) if prob.mode == "heads" else None
        evs.append((a, b, g))
    for a, b, g in evs:  # materialise the events outside the timed region
        for pair in list(a.values()) + list(b.values()) + ([g] if g else []):
            pair[0].record()
            pair[1].record()
    t0, t1 = E(enable_timing=True), E(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.3)
    if flush is None:
        t0.record()
        for _ in range(steps):
            prob.step()
        t1.record()
    else:
        per_step = [(E(enable_timing=True), E(enable_timing=True)) for _ in range(steps)]
        for s_, e_ in per_step:
            flush.fill_(1)
            s_.record()
            prob.step()
            e_.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    if flush is None:
        ms = t0.elapsed_time(t1) / steps
    else:
        ms = sum(s_.elapsed_time(e_) for s_, e_ in per_step) / steps
    st = msa.device_status(prob.ws)
    if st != 0:
        raise RuntimeError(f"{w.name}: device status {msa.status_string(st)}")
    # stage times from a second, separate pass (events between the stages
    # would stop consecutive kernels from overlapping their launch)
    if prob.paged:
        evs = []
    for ev in evs:
        if flush is not None:
            flush.fill_(1)
        prob.step(ev=ev)
    torch.cuda.synchronize()
    stage_ms = {}
    for a, b, g in evs:
        for i, (s_, e_) in a.items():
            stage_ms[f"index{i}"] = stage_ms.get(f"index{i}", 0.0) + s_.elapsed_time(e_) / steps
        for i, (s_, e_) in b.items():
            stage_ms[f"attn{i}"] = stage_ms.get(f"attn{i}", 0.0) + s_.elapsed_time(e_) / steps
        if g:
            stage_ms["gather"] = stage_ms.get("gather", 0.0) + g[0].elapsed_time(g[1]) / steps
    if prob.r1 == prob.r0 and not w.is_decode:
        stage_ms["index0"] = 0.0
    ms = max_over_ranks([ms], world, dev)[0]
    res = {"ms": ms, "stage_ms": stage_ms, "clocks": clk,
           "launches": prob.launches_per_step * steps,
           "l2": ("inputs and partials larger than L2 (126 MB): no flush needed"
                  if flush is None else
                  "L2 flushed between timed steps (256 MB write outside each step's events; "
                  "the step time is the mean of per-step events)")}
    del flush
    if with_e2e:
        res["e2e"] = measure_e2e(prob, steps)
    return res


def measure_e2e(prob, steps):
    """The same step through the public API with host buffers: every step
    uploads its inputs from pinned host memory and reads its result (out,
    lse) back.  Serial: one step at a time.  Pipelined (the reported value):
    two device buffer sets and three streams, so step i+1's upload and step
    i-1's download (PCIe is full duplex) overlap step i's kernels, as a
    stream of requests would run."""
    import torch
    import torch.distributed as dist
    from block_sparse_long_05_b200 import msa
    world, dev = prob.world, prob.dev
    E = torch.cuda.Event
    hx = {k: v.cpu().pin_memory() for k, v in prob.x.items()}
    hy = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in prob.y.items()}
    h2d = sum(v.numel() * v.element_size() for v in hx.values())
    d2h = sum(v.numel() * v.element_size() for v in hy.values())
    e_steps = max(1, min(steps, 5))

    def serial_step():
        for k_, v_ in hx.items():
            prob.x[k_].copy_(v_, non_blocking=True)
        prob.step()
        for k_, v_ in hy.items():
            v_.copy_(prob.y[k_], non_blocking=True)

    serial_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a0, a1 = E(enable_timing=True), E(enable_timing=True)
    a0.record()
    for _ in range(e_steps):
        serial_step()
    a1.record()
    torch.cuda.synchronize()
    serial_ms = a0.elapsed_time(a1) / e_steps

    sets = [(prob.x, prob.y),
            ({k: torch.empty_like(v) for k, v in prob.x.items()},
             {k: torch.empty_like(v) for k, v in prob.y.items()})]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    p_steps = max(4, min(steps, 8)) + 2
    ev_in = [E() for _ in range(p_steps)]
    ev_run = [E() for _ in range(p_steps)]
    ev_out = [E() for _ in range(p_steps)]

    def pipelined(i):
        xs, ys = sets[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_run[i - 2])      # step i-2 has read this input set
            for k_, v_ in hx.items():
                xs[k_].copy_(v_, non_blocking=True)
            ev_in[i].record(s_in)
        s_run.wait_event(ev_in[i])
        if i >= 2:
            s_run.wait_event(ev_out[i - 2])         # step i-2's result has been read back
        prob.step(xs, ys, stream=s_run)
        ev_run[i].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[i])
            for k_, v_ in hy.items():
                v_.copy_(ys[k_], non_blocking=True)
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
    if msa.device_status(prob.ws) != 0:
        raise RuntimeError("device status after the pipelined e2e steps")
    ems, serial_ms = max_over_ranks([ems, serial_ms], world, dev)
    h2d, d2h = sum_over_ranks([h2d, d2h], world, dev)
    del sets, hx, hy
    return {"ms": ems, "serial_ms": serial_ms, "h2d": int(h2d), "d2h": int(d2h),
            "steps": p_steps}


def sum_over_ranks(values, world: int, device):
    """Element-wise sum of per-rank numbers over all ranks."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(v) for v in t.tolist()]


def load_traffic():
    """DRAM bytes per launch from ncu captures (profiles/dram_traffic.json):
    {"kernel@workload": bytes}, the entries marked valid only."""
    tpath = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(tpath):
        return {}
    with open(tpath) as f:
        tr = json.load(f)
    return {k: v["bytes_per_launch"] for k, v in tr.items() if v.get("valid", True)}


def kernel_name(w, stage):
    if w.is_decode:
        return {"index0": "decode_index_scan_kernel", "index1": "decode_select_kernel",
                "attn1": "decode_attn_kernel", "attn2": "lse_combine_split_kernel"}[stage]
    return {"index0": "prefill_index_kernel", "attn0": "inversion (5 kernels)",
            "attn1": "prefill_attn_resident_kernel" if w.block <= 128
            else "prefill_attn_streamed_kernel",
            "attn2": "lse_combine_kernel"}[stage]


def stage_work(w, prob, pairs):
    """Algorithmic work of each timed stage of one step of this rank:
    {stage: (bound, amount, unit)} -- flops for tensor-core stages, bytes
    for HBM stages."""
    Hq, Hkv = prob.Hq, prob.Hkv
    if w.is_decode:
        scan_b, kv_b = decode_bytes(w, prob.ids, Hq, Hkv)
        S = -(-w.block // 64)
        comb = w.Bt * w.K * S * Hq * (w.d * 4 + 4) + w.Bt * Hq * (w.d * 4 + 4)
        return {"index0": ("hbm", scan_b), "attn1": ("hbm", kv_b), "attn2": ("hbm", comb)}
    rows = w.Bt * w.n_q
    comb = rows * w.K * Hq * (w.d * 2 + 4) + rows * Hq * (w.d * 4 + 4) + rows * w.K * 4
    return {"index0": ("tensor", 2.0 * index_macs(w, prob.r0, prob.r1)),
            "attn1": ("tensor", 4.0 * w.d * Hq * pairs),
            "attn2": ("hbm", comb)}


def stage_launches(w, prob, stage):
    """Kernel launches that one stage's event time (and its work and DRAM
    traffic figures) span: a prefill attention stage runs once per kv-head
    group, twice per group (hit lists, then each block's own rows) for
    blocks longer than 128 keys."""
    if w.is_decode or stage != "attn1":
        return 1
    groups = prob.Hkv // (prob.kv_group or prob.Hkv)
    return groups * (2 if w.block > 128 else 1)


def roofline(w, prob, r, peaks, peak_src, traffic):
    """Roofline of the dominant kernel of the step (and of every timed
    stage): achieved = algorithmic work / the stage's event time."""
    sm = r["stage_ms"]
    work = stage_work(w, prob, r["pairs"])
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    hbm = float(peaks["hbm_gbs"])
    kernels = {}
    for st, (bound, amount) in work.items():
        t = sm.get(st, 0.0)
        if t <= 0:
            continue
        if bound == "tensor":
            ach = amount / (t / 1e3) / 1e12
            kernels[st] = {"kernel": kernel_name(w, st), "ms": round(t, 4), "bound": "tensor",
                           "achieved": ach, "unit": "TFLOP/s", "frac": ach / burst,
                           "frac_sustained": ach / sustained, "work_per_launch": amount}
        else:
            ach = amount / (t / 1e3) / 1e9
            kernels[st] = {"kernel": kernel_name(w, st), "ms": round(t, 4), "bound": "hbm",
                           "achieved": ach, "unit": "GB/s", "frac": ach / hbm,
                           "work_per_launch": amount}
    dom = max((s for s in ("index0", "attn1") if s in kernels), key=lambda s: sm.get(s, 0.0))
    k = kernels[dom]
    tr = traffic.get(f"{k['kernel']}@{w.name}")
    roof = {"bound": k["bound"], "kernel": k["kernel"], "achieved": k["achieved"],
            "peak": burst if k["bound"] == "tensor" else hbm, "unit": k["unit"],
            "frac": k["frac"], "traffic": tr, "work_per_launch": k["work_per_launch"],
            "launches": stage_launches(w, prob, dom),
            "peak_note": (f"bf16 dense burst (cuBLAS, a ms-scale kernel timed alone), of "
                          f"{peak_src}; frac_sustained uses the sustained {sustained} TFLOP/s"
                          if k["bound"] == "tensor" else f"HBM copy bandwidth, of {peak_src}")}
    if k["bound"] == "tensor":
        roof["frac_sustained"] = k["frac_sustained"]
    else:
        roof["frac_of_8tbs_nominal"] = k["achieved"] / 8000.0
    return roof, kernels


def measure_int8_index(w, prob, r, steps, warmup, peaks, peak_src):
    """The same step with the index branch on int8 index keys
    (msa_index_topk_i8); its ids must equal the bf16 path's."""
    import torch
    ids_bf16 = prob.ids.clone()
    prob.use_int8_index()
    try:
        ri = measure(prob, steps, warmup, False)
    finally:
        prob.int8_index = False
    sm = ri["stage_ms"]
    obj = {"ms_per_step": ri["ms"], "value": w.Bt * w.n_q / (ri["ms"] / 1e3), "unit": UNIT,
           "stage_ms": {k: round(v, 4) for k, v in sm.items()},
           "ids_equal_bf16_path": bool(torch.equal(prob.ids, ids_bf16))}
    t = sm.get("index0", 0.0)
    if t > 0:
        if w.is_decode:
            scan_b = decode_bytes(w, prob.ids)[0] // 2  # int8 keys: half the bytes
            obj["index_kernel"] = {"kernel": "decode_index_scan_kernel (int8)", "ms": round(t, 4),
                                   "bound": "hbm", "achieved": scan_b / (t / 1e3) / 1e9,
                                   "unit": "GB/s",
                                   "frac": scan_b / (t / 1e3) / 1e9 / float(peaks["hbm_gbs"])}
        else:
            peak8 = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
            ach = 2.0 * index_macs(w) / (t / 1e3) / 1e12
            obj["index_kernel"] = {"kernel": "prefill_index_kernel (kind::i8)", "ms": round(t, 4),
                                   "bound": "tensor", "achieved": ach, "unit": "TOP/s",
                                   "peak": peak8, "frac": ach / peak8,
                                   "peak_note": f"int8 dense = 2 x the bf16 burst of {peak_src} "
                                                "(nominal 4.5 / 2.25 PFLOP/s ratio)"}
    del prob.x["q_idx8"], prob.x["k_idx8"]
    return obj


def measure_min_workspace(w, prob, r, steps, warmup):
    """The prefill step with the minimum workspace (msa_workspace_size): the
    kv heads are attended and merged in groups whose partials fit in it."""
    from block_sparse_long_05_b200 import msa
    one = prob.ws
    prob.ws = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, prob.Hq, prob.Hkv, w.d, w.d_idx,
                                      w.block, w.K, device=prob.dev)
    try:
        rm = measure(prob, steps, warmup, False)
        nbytes = prob.ws.nbytes
    finally:
        prob.ws = one
    return {"ms_per_step": rm["ms"], "value": w.Bt * w.n_q / (rm["ms"] / 1e3), "unit": UNIT,
            "workspace_bytes": nbytes, "one_pass_workspace_bytes": one.nbytes,
            "vs_one_pass": r["ms"] / rm["ms"]}


def measure_paged(w, prob, r, steps, warmup):
    """The decode step through the paged entry points on a permuted page
    store (same values, same ids)."""
    import torch
    ids_contig = prob.ids.clone()
    prob.use_paged()
    try:
        rp = measure(prob, steps, warmup, False)
    finally:
        prob.paged = False
    obj = {"ms_per_step": rp["ms"], "value": w.Bt / (rp["ms"] / 1e3), "unit": UNIT,
           "vs_contiguous": r["ms"] / rp["ms"],
           "ids_equal_contiguous": bool(torch.equal(prob.ids, ids_contig)),
           "layout": "k_idx, K and V in pages of one block each, scattered in a seeded random "
                     "order; page table [Bt, N] int32"}
    for k in ("k_idx_pages", "k_pages", "v_pages", "page_table"):
        del prob.x[k]
    return obj


def bench_workload(w, args, rank, world, dev, peaks, peak_src, traffic, mode, steps, warmup,
                   with_e2e, decode_at_T, cpu_seconds):
    """Measure one workload; returns its JSON object (the headline's fields
    for the main line, or one entry of "configs")."""
    import torch
    prob = Problem(w, dev, rank, world, mode)
    r = measure(prob, steps, warmup, with_e2e)
    r["pairs"] = attended_pairs(prob.ids, w)
    roof, kernels = roofline(w, prob, r, peaks, peak_src, traffic)
    tokens = w.Bt * w.n_q * (world if mode == "seq" else 1)
    with_i8 = mode == "whole" and not getattr(args, "no_int8", False)
    if with_i8:
        obj_i8 = measure_int8_index(w, prob, r, steps, warmup, peaks, peak_src)
    with_paged = mode == "whole" and w.is_decode and w.T % w.block == 0 and \
        not getattr(args, "no_paged", False)
    if with_paged:
        obj_paged = measure_paged(w, prob, r, steps, warmup)
    with_minws = mode == "whole" and not w.is_decode and not getattr(args, "no_min_ws", False)
    if with_minws:
        obj_minws = measure_min_workspace(w, prob, r, steps, warmup)
    obj = {"workload": w.name, "value": tokens / (r["ms"] / 1e3), "unit": UNIT,
           "ms_per_step": r["ms"], "stage_ms": {k: round(v, 4) for k, v in r["stage_ms"].items()},
           "roofline": roof, "kernels": kernels, "gpu_launches": r["launches"],
           "l2": r["l2"], "clocks": r["clocks"]}
    if w.is_decode:
        scan_b, kv_b = decode_bytes(w, prob.ids, prob.Hq, prob.Hkv)
        obj["step_bytes"] = scan_b + kv_b
        obj["step_hbm_frac"] = (scan_b + kv_b) / (r["ms"] / 1e3) / 1e9 / float(peaks["hbm_gbs"])
        obj["step_frac_of_8tbs_nominal"] = (scan_b + kv_b) / (r["ms"] / 1e3) / 1e9 / 8000.0
    else:
        obj["attended_pairs"] = r["pairs"]
    if with_i8:
        obj["int8_index"] = obj_i8
    if with_paged:
        obj["paged"] = obj_paged
    if with_minws:
        obj["min_workspace"] = obj_minws
    if "e2e" in r:
        e = r["e2e"]
        obj["e2e"] = {"value": tokens / (e["ms"] / 1e3), "unit": UNIT, "ms_per_step": e["ms"],
                      "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                      "pipelined": f"{e['steps']} steps; upload of step i+1 and download of "
                                   "step i-1 overlap step i (two device buffer sets, three "
                                   "streams, pinned host buffers)",
                      "serial_ms_per_step": e["serial_ms"],
                      "serial_value": tokens / (e["serial_ms"] / 1e3)}
    prob.free()
    del prob
    torch.cuda.empty_cache()
    # decode step at this prefill workload's context: one sequence of T keys,
    # same heads, block, K and index dim (a failure is recorded in the object)
    if decode_at_T and not w.is_decode and world == 1:
        from block_sparse_long_05_b200.inputs import Workload
        wt = Workload(f"decode_1x{w.T}", 1, 1, w.T, w.Hq, w.Hkv, w.d, w.block, w.K, w.d_idx)
        try:
            pt = Problem(wt, dev, rank, world, "whole")
            rt = measure(pt, max(steps, 20), max(warmup, 3), False)
            scan_b, kv_b = decode_bytes(wt, pt.ids, pt.Hq, pt.Hkv)
            obj["decode_at_T"] = {
                "workload": wt.name, "value": 1 / (rt["ms"] / 1e3), "unit": UNIT,
                "ms_per_step": rt["ms"],
                "stage_ms": {k: round(v, 4) for k, v in rt["stage_ms"].items()},
                "step_bytes": scan_b + kv_b,
                "step_hbm_frac": (scan_b + kv_b) / (rt["ms"] / 1e3) / 1e9 / float(peaks["hbm_gbs"]),
            }
            pt.free()
            del pt
        except Exception as e:  # noqa: BLE001 -- recorded, not hidden
            obj["decode_at_T"] = {"workload": wt.name, "error": f"{type(e).__name__}: {e}"[:300]}
        torch.cuda.empty_cache()
    if cpu_seconds > 0 and rank == 0 and world == 1:
        obj["cpu_baseline"] = cpu_baseline(w, cpu_seconds)
    return obj


def parallel_mode(w, world):
    """How `world` GPUs share workload w (see Problem)."""
    if world == 1:
        return "whole"
    if not w.is_decode and w.Bt == 1 and w.Hkv % world == 0:
        return "heads"
    return "seq"


def config_for(w, world, mode):
    """The "config" object of the JSON line (both arms)."""
    parallelism = {"whole": "dp1", "seq": f"dp{world} (sequences)",
                   "heads": f"kv-head sharding over {world} GPUs (index rows split, ids "
                            f"all-gathered)"}[mode]
    return {"workload": w.name, "Bt_per_gpu": w.Bt if mode != "heads" else 1,
            "n_q": w.n_q, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "block": w.block, "K": w.K, "d_idx": w.d_idx,
            "global_batch": w.Bt * (world if mode == "seq" else 1), "seq_len": w.T,
            "parallelism": parallelism}


def run_msa(args, rank, world, local_rank):
    import torch
    from block_sparse_long_05_b200.inputs import WORKLOADS

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    peaks, peak_src = load_peaks()
    traffic = load_traffic()
    mode = parallel_mode(w, world)
    cpu_s = 0.0 if args.no_cpu_baseline else args.cpu_seconds
    head = bench_workload(w, args, rank, world, dev, peaks, peak_src, traffic, mode, args.steps,
                          args.warmup, not args.no_e2e, not args.no_decode, cpu_s)
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "strong" if mode == "heads" else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_for(w, world, mode), l2=head["l2"]),
        "gpu_launches": head["gpu_launches"],
        "stage_ms": head["stage_ms"],
        "roofline": head["roofline"],
        "kernels": head["kernels"],
    }
    if head.get("clocks"):
        line["clocks"] = head["clocks"]
    if "e2e" in head:
        line["e2e"] = head["e2e"]
    for key in ("decode_at_T", "int8_index", "paged", "min_workspace", "attended_pairs",
                "step_bytes", "step_hbm_frac", "step_frac_of_8tbs_nominal"):
        if key in head:
            line[key] = head[key]
    if "cpu_baseline" in head:
        line["cpu_baseline"] = head["cpu_baseline"]
    # every workload of the hot path (one GPU): each with its own numbers
    if world == 1 and not args.only:
        configs = {}
        for name in CONFIGS:
            if name == w.name:
                configs[name] = {k: v for k, v in head.items() if k not in ("e2e", "kernels")}
                continue
            try:
                wc = WORKLOADS[name]
                configs[name] = bench_workload(wc, args, rank, world, dev, peaks, peak_src,
                                               traffic, "whole", args.steps, args.warmup, False,
                                               not args.no_decode, cpu_s / 3)
            except Exception as e:  # noqa: BLE001 -- recorded, not hidden
                configs[name] = {"workload": name, "error": f"{type(e).__name__}: {e}"[:300]}
        line["configs"] = configs
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
    world = int(os.environ.get("WORLD_SIZE", "1"))
    mode = parallel_mode(w, world)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "strong" if mode == "heads" else "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(config_for(w, world, mode),
                           sample=f"sampled-row rate: {sample}; the oracle runs on the host "
                                  "cores of rank 0 alone"),
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
