"""Runs bench.py's measurement logic on the CPU with the CUDA library, CUDA
events and the clock sampler replaced by fakes, on small stand-ins for the
default prefill and decode workloads; prints the JSON line.  Launched in its
own process by tests/test_bench_model.py (it patches torch for that process).

argv[1]: "flush" (small steps: L2 flushed between timed steps) or "noflush"
(the L2 threshold set to one byte: back-to-back timing)."""
import json
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

_device = torch.device
torch.device = lambda *a, **k: _device("cpu")
torch.cuda.set_device = lambda *a, **k: None
torch.cuda.synchronize = lambda *a, **k: None


class FakeEvent:
    clock = 0.0

    def __init__(self, enable_timing=False):
        self.t = None

    def record(self, stream=None):
        FakeEvent.clock += 0.25
        self.t = FakeEvent.clock

    def elapsed_time(self, other):
        return other.t - self.t


torch.cuda.Event = FakeEvent

import bench  # noqa: E402
from block_sparse_long_05_b200 import inputs, msa  # noqa: E402


class FakeClocks:
    def __init__(self, gpu_index):
        pass

    def start(self):
        pass

    def stop(self):
        return {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}


class FakeWorkspace:
    @classmethod
    def for_shape(cls, *args, **kwargs):
        return cls()


def fake_index_topk(q_idx, k_idx, block, K, ws, ids=None, stream=None, events=None):
    """Own block plus the K-1 blocks before it (a valid selection)."""
    Bt, n_q, _ = q_idx.shape
    T = k_idx.shape[1]
    for b in range(Bt):
        for i in range(n_q):
            own = (T - n_q + i) // block
            sel = list(range(max(0, own - K + 1), own + 1))
            ids[b, i] = torch.tensor(sel + [-1] * (K - len(sel)), dtype=torch.int32)
    for s_, e_ in (events or {}).values():
        s_.record()
        e_.record()
    return ids


def fake_sparse_attn(q, k, v, ids, block, ws, out=None, lse=None, stream=None, events=None):
    for s_, e_ in (events or {}).values():
        s_.record()
        e_.record()
    return out, lse


def main():
    bench.ClockSampler = FakeClocks
    msa.Workspace = FakeWorkspace
    msa.index_topk = fake_index_topk
    msa.sparse_attn = fake_sparse_attn
    msa.device_status = lambda ws, stream=None: 0
    W = inputs.Workload
    inputs.WORKLOADS[bench.DEFAULT_WORKLOAD] = W(bench.DEFAULT_WORKLOAD, 1, 256, 256, 8, 2, 64, 32, 4, 64)
    inputs.WORKLOADS[bench.SECONDARY_DECODE] = W(bench.SECONDARY_DECODE, 4, 1, 4096, 8, 2, 64, 128, 4, 64)
    if sys.argv[1] == "noflush":
        bench.L2_BYTES = 1
    args = types.SimpleNamespace(workload=bench.DEFAULT_WORKLOAD, steps=3, warmup=1, no_e2e=True,
                                 no_cpu_baseline=True, no_decode=False, cpu_seconds=1.0)
    print(json.dumps(bench.run_msa(args, 0, 1, 0)))


if __name__ == "__main__":
    main()
