"""One rank of the CPU (gloo) exercise of the kv-head-sharded prefill
partition (block_sparse_long_05_b200.shard); launched by
tests/test_multirank.py through torch.distributed.run.

Each rank runs the CPU oracle, standing in for the kernels, on its query-row
range of the index branch.  The ids are all-gathered over gloo.  Then each
rank runs the oracle's sparse branch on its own kv heads (and their query
heads) over every row.  Rank 0 gathers the head-sharded outputs and prints
them, with the ids, as one JSON line; the test compares them with a
single-process oracle run over all heads."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from block_sparse_long_05_b200 import shard  # noqa: E402
from block_sparse_long_05_b200.inputs import Workload, make_inputs  # noqa: E402
from oracle import oracle  # noqa: E402

# one sequence, ragged last block, 4 kv heads (G = 2)
PREFILL = Workload("shard_prefill", 1, 600, 600, 8, 4, 64, 64, 4, 64)


def main():
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w = PREFILL
        x = make_inputs(w, device="cpu")
        hk0, hk1 = shard.head_range(w.Hkv, world, rank)
        G = w.G
        q_h = x["q"][:, :, hk0 * G:hk1 * G].contiguous()
        k_h = x["k"][:, :, hk0:hk1].contiguous()
        v_h = x["v"][:, :, hk0:hk1].contiguous()

        def index_fn(qi, ki, T_cut):
            ids = oracle.index_topk(qi, ki, 1, qi.shape[1], T_cut, w.d_idx, w.block, w.K)
            return torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32))
        index_fn.K = w.K

        def attn_fn(ids):
            return oracle.sparse_attn(q_h, k_h, v_h, ids.numpy(), 1, w.n_q, w.T, q_h.shape[2],
                                      hk1 - hk0, w.d, w.block, w.K)

        ids, (out, lse) = shard.prefill_head_sharded(x["q_idx"], x["k_idx"], w.T, w.block, world,
                                                     rank, index_fn, attn_fn)
        mine = torch.from_numpy(np.concatenate([out.reshape(w.n_q, -1), lse.reshape(w.n_q, -1)],
                                               axis=1).astype(np.float64))
        parts = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(parts, mine)
        if rank == 0:
            print(json.dumps({"world": world, "ids": ids.tolist(),
                              "ranges": shard.index_row_ranges(w.n_q, w.T, w.block, world),
                              "parts": [p.tolist() for p in parts]}), flush=True)
        dist.barrier()
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
