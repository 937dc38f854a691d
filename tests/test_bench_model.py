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


def _host_run(mode):
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "tests", "bench_host_worker.py"), mode],
                       cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_bench_line_structure_with_and_without_l2_flush():
    """bench.py's measurement logic end to end on the CPU (library, events and
    clocks faked): the JSON line carries every key the benchmark contract
    names, for both timing paths, with both decode secondaries."""
    for mode, l2_word in (("flush", "flushed"), ("noflush", "no flush")):
        line = _host_run(mode)
        for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                    "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                    "gpu_launches", "roofline", "clocks", "decode", "decode_at_T"):
            assert key in line, (mode, key)
        assert l2_word in line["config"]["l2"], (mode, line["config"]["l2"])
        assert line["gpu_launches"] == 8 * line["steps"]
        for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
            assert key in line["roofline"], key
        assert "error" not in line["decode_at_T"], line["decode_at_T"]
        assert line["decode_at_T"]["workload"] == f"decode_1x{line['config']['T']}"
        if mode == "flush":  # fake events tick 0.25 ms per record: one step = 0.25 ms
            assert abs(line["ms_per_step"] - 0.25) < 1e-9
