"""Runs bench.py's measurement logic on the CPU with the CUDA library, CUDA
events and the clock sampler replaced by fakes, on small stand-ins for the
default prefill and decode workloads; prints the JSON line.  Launched in its
own process by tests/test_bench_model.py (it patches torch for that process).

argv[1]: "flush" (small steps: L2 flushed between timed steps), "noflush"
(the L2 threshold set to one byte: back-to-back timing) or "heads" (run
under torch.distributed.run with gloo ranks: the kv-head-sharded long
prefill, its ids all-gathered between the ranks)."""
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
    nbytes = 1 << 20

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
    msa.index_topk_i8 = fake_index_topk
    msa.index_topk_paged = lambda q_idx, k_idx_pages, table, T, K, ws, ids=None, stream=None: \
        fake_index_topk(q_idx, torch.empty((q_idx.shape[0], T, 1)), k_idx_pages.shape[1], K, ws,
                        ids=ids)
    msa.sparse_attn_paged = lambda q, kp, vp, table, T, ids, ws, out=None, lse=None, stream=None: \
        (out, lse)
    msa.sparse_attn = fake_sparse_attn
    msa.device_status = lambda ws, stream=None: 0
    W = inputs.Workload
    # small stand-ins with each workload's kind (prefill / decode)
    small = {"tiny_prefill_T4096": W("tiny_prefill_T4096", 1, 128, 128, 8, 2, 64, 32, 4, 64),
             "prefill_T65536": W("prefill_T65536", 1, 256, 256, 8, 2, 64, 32, 4, 64),
             "decode_32x131072": W("decode_32x131072", 3, 1, 2048, 8, 2, 64, 128, 4, 64),
             # blocks of two 128-key sub-tiles, like the 256K prefill's 512
             "long_prefill_T262144": W("long_prefill_T262144", 1, 1024, 1024, 8, 2, 64, 256, 4,
                                       64),
             "decode_4x1048576": W("decode_4x1048576", 4, 1, 4096, 8, 2, 64, 128, 4, 64)}
    inputs.WORKLOADS.update(small)
    if sys.argv[1] == "noflush":
        bench.L2_BYTES = 1
    args = types.SimpleNamespace(workload=bench.DEFAULT_WORKLOAD, steps=3, warmup=1, no_e2e=True,
                                 no_cpu_baseline=True, no_decode=False, cpu_seconds=1.0,
                                 only=False)
    if sys.argv[1] == "heads":
        import datetime
        import torch.distributed as dist
        rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        seen = []
        real_attn = msa.sparse_attn

        def recording_attn(q, k, v, ids, block, ws, **kw):
            seen.append((tuple(q.shape), tuple(k.shape), ids.clone()))
            return real_attn(q, k, v, ids, block, ws, **kw)
        msa.sparse_attn = recording_attn
        try:
            line = bench.run_msa(args, rank, world, rank)
            q_shape, k_shape, ids = seen[-1]
            mine = torch.tensor([float(ids.long().sum()), float(q_shape[2]), float(k_shape[2])],
                                dtype=torch.float64)
            parts = [torch.zeros_like(mine) for _ in range(world)]
            dist.all_gather(parts, mine)
            w = inputs.WORKLOADS[bench.DEFAULT_WORKLOAD]
            ref = torch.empty((1, w.n_q, w.K), dtype=torch.int32)
            fake_index_topk(torch.empty((1, w.n_q, w.d_idx)), torch.empty((1, w.T, w.d_idx)),
                            w.block, w.K, None, ids=ref)
            if rank == 0:
                line["_ranks"] = [p.tolist() for p in parts]
                line["_ids_sum"] = float(ref.long().sum())
                print(json.dumps(line))
        finally:
            dist.destroy_process_group()
        return
    print(json.dumps(bench.run_msa(args, 0, 1, 0)))


if __name__ == "__main__":
    main()
