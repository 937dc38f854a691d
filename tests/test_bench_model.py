"""The work model behind bench.py's roofline numbers, on the CPU: the
attended (query, key) pair count, the index multiply-adds and the decode
bytes, each against a direct count on small inputs."""
import numpy as np
import torch

import bench
from block_sparse_long_05_b200.inputs import Workload, random_selection


def _direct_pairs(ids, w):
    """Keys i <= t inside the selected blocks (ragged tail included), summed
    over every query row."""
    n = 0
    ids = ids.reshape(w.Bt * w.n_q, w.K).numpy()
    for r in range(w.Bt * w.n_q):
        t = w.T - w.n_q + r % w.n_q
        for j in ids[r]:
            if j < 0:
                continue
            for i in range(j * w.block, min((j + 1) * w.block, w.T)):
                n += i <= t
    return n


def test_attended_pairs_counts_causal_keys_of_selected_blocks():
    for w in (Workload("m_prefill", 2, 50, 50, 4, 2, 64, 8, 3, 64),      # ragged last block
              Workload("m_chunk", 1, 20, 77, 4, 2, 64, 16, 4, 64),       # last n_q queries
              Workload("m_decode", 3, 1, 100, 4, 2, 64, 32, 2, 64)):
        ids = random_selection(w, device="cpu")
        assert bench.attended_pairs(ids, w) == _direct_pairs(ids, w), w.name
    # -1 slots contribute nothing
    w = Workload("m_pad", 1, 4, 16, 1, 1, 64, 4, 3, 64)
    ids = torch.tensor([[[0, -1, -1], [0, -1, -1], [0, -1, -1], [0, -1, -1]]], dtype=torch.int32)
    assert bench.attended_pairs(ids, w) == 4 * 4  # t = 12..15, all four keys of block 0


def test_index_macs_counts_every_key_of_every_candidate_block():
    w = Workload("m_idx", 2, 30, 45, 4, 2, 64, 8, 3, 16)
    exp = 0
    for b in range(w.Bt):
        for i in range(w.n_q):
            t = w.T - w.n_q + i
            exp += (t // w.block) * w.block * w.d_idx  # blocks j < own(t), whole blocks
    assert bench.index_macs(w) == exp


def test_decode_bytes():
    w = Workload("m_dec", 2, 1, 100, 8, 2, 64, 32, 3, 16)
    ids = torch.tensor([[[0, 2, 3]], [[1, -1, 3]]], dtype=torch.int32)
    scan, kv = bench.decode_bytes(w, ids)
    own = (w.T - 1) // w.block  # 3
    assert scan == w.Bt * own * w.block * w.d_idx * 2 + w.Bt * w.d_idx * 2
    keys = (32 + 32 + 4) + (32 + 4)  # block 3 holds keys 96..99
    assert kv == keys * w.Hkv * w.d * 2 * 2 + w.Bt * w.Hq * w.d * 2
    assert np.isclose(bench.job_throughput(w, 0.5, 4), 2 * 1 * 4 / 0.5e-3)
