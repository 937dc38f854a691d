"""One rank of the two-rank CPU (gloo) exercise of bench.py's multi-GPU
plumbing; launched by tests/test_multirank.py through torch.distributed.run.

Each rank draws its own shard of a small decode-shaped workload (weak
scaling: seed w.seed + rank), runs the CPU oracle on it (standing in for the
kernels, which need a GPU), and takes the same collective steps as bench.py:
a barrier, the max over ranks of per-rank step times, the whole-job
throughput.  Rank 0 prints one JSON line with what every rank saw."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402
from block_sparse_long_05_b200.inputs import Workload, make_inputs  # noqa: E402
from oracle import oracle  # noqa: E402

SHARD = Workload("multirank_decode", 2, 1, 300, 4, 2, 64, 64, 4, 64)


def shard_result(rank: int):
    w = SHARD
    x = make_inputs(w, device="cpu", seed=bench.rank_seed(w, rank))
    ids = oracle.index_topk(x["q_idx"], x["k_idx"], w.Bt, w.n_q, w.T, w.d_idx, w.block, w.K)
    out, lse = oracle.sparse_attn(x["q"], x["k"], x["v"], ids, w.Bt, w.n_q, w.T, w.Hq, w.Hkv,
                                  w.d, w.block, w.K)
    return ids, out, lse


def main():
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ids, out, lse = shard_result(rank)
        dist.barrier()
        # step times that differ per rank: the job's time is the slowest rank's
        ms = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world, torch.device("cpu"))
        value = bench.job_throughput(SHARD, ms[0], world)
        mine = torch.tensor([float(np.abs(out).sum()), float(lse.sum()), float(ids.sum())],
                            dtype=torch.float64)
        allv = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(allv, mine)
        if rank == 0:
            print(json.dumps({"world": world, "ms": ms, "value": value,
                              "digests": [v.tolist() for v in allv]}), flush=True)
        dist.barrier()
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
