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
    names, for both timing paths, with every workload under "configs"."""
    for mode, l2_word in (("flush", "flushed"), ("noflush", "no flush")):
        line = _host_run(mode)
        for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                    "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                    "gpu_launches", "roofline", "clocks", "decode_at_T", "configs", "kernels"):
            assert key in line, (mode, key)
        assert line["config"]["workload"] == bench.DEFAULT_WORKLOAD
        assert l2_word in line["config"]["l2"], (mode, line["config"]["l2"])
        # 256K prefill (block 512): index, 5 inversion kernels, 3 for the
        # own-block work list, hit-list and own-block attention, combine
        assert line["gpu_launches"] == 12 * line["steps"]
        for key in ("bound", "achieved", "peak", "unit", "frac", "traffic", "frac_sustained"):
            assert key in line["roofline"], key
        # the tensor-core fraction is taken against the burst peak
        assert abs(line["roofline"]["frac"] * line["roofline"]["peak"] -
                   line["roofline"]["achieved"]) < 1e-6 * line["roofline"]["achieved"]
        assert "error" not in line["decode_at_T"], line["decode_at_T"]
        assert line["decode_at_T"]["workload"] == f"decode_1x{line['config']['T']}"
        # every workload of the hot path, each with its own numbers
        assert sorted(line["configs"]) == sorted(bench.CONFIGS)
        for name, c in line["configs"].items():
            assert "error" not in c, (name, c)
            for key in ("value", "ms_per_step", "stage_ms", "roofline"):
                assert key in c, (name, key)
            exp_bound = "hbm" if name.startswith("decode") else "tensor"
            assert c["roofline"]["bound"] == exp_bound, (name, c["roofline"])
            # the same step with the int8 index path, whose ids match the bf16 path's
            assert c["int8_index"]["ids_equal_bf16_path"], name
            assert c["int8_index"]["index_kernel"]["bound"] == exp_bound, name
            if name.startswith("decode"):  # and through the paged entry points
                assert c["paged"]["ids_equal_contiguous"], name
                assert c["paged"]["ms_per_step"] > 0, name
            else:  # and with the minimum (kv-head grouped) workspace
                assert c["min_workspace"]["ms_per_step"] > 0, name
        if mode == "flush":  # fake events tick 0.25 ms per record: one step = 0.25 ms
            assert abs(line["ms_per_step"] - 0.25) < 1e-9


def test_bench_head_sharded_prefill_on_two_gloo_ranks():
    """bench.py's kv-head-sharded long prefill on two gloo ranks (library
    faked): each rank holds half of the heads, and the ids every rank's
    sparse branch sees, all-gathered from the two row ranges, are the full
    selection; the line reports strong scaling over 2 GPUs."""
    import json
    import os
    import socket
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.join(root, "tests", "bench_host_worker.py"), "heads"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, OMP_NUM_THREADS="1"))
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["scaling"] == "strong"
    assert "kv-head" in line["config"]["parallelism"]
    assert "gather" in line["stage_ms"]
    assert "configs" not in line  # the other workloads are timed at one GPU only
    for ids_sum, hq, hkv in line["_ranks"]:
        assert ids_sum == line["_ids_sum"]       # the full selection on every rank
        assert hq == line["config"]["Hq"] // 2 and hkv == line["config"]["Hkv"] // 2


def test_launch_count_model():
    """Kernels of the library one step launches, as the C ABI sequences them:
    prefill = index, 5 inversion kernels (+3 for the own-block work list with
    blocks longer than 128 keys), then per kv-head group the attention
    launch(es) (hit lists, own blocks) and the combine; decode = k_idx scan
    (when a block precedes the query's own), select, attention, combine."""
    import types
    count = bench.Problem.launches_per_step.fget
    W = Workload

    def prob(w, kv_group=None, r0=0, r1=None):
        return types.SimpleNamespace(w=w, Hkv=w.Hkv, kv_group=kv_group, r0=r0,
                                     r1=w.n_q if r1 is None else r1)

    small = W("m_b64", 1, 256, 256, 8, 4, 64, 64, 4, 64)
    wide = W("m_b512", 1, 2048, 2048, 8, 4, 64, 512, 3, 64)
    assert count(prob(small, kv_group=4)) == 1 + 5 + 1 + 1
    assert count(prob(wide, kv_group=4)) == 1 + 5 + 3 + 2 + 1
    assert count(prob(wide, kv_group=2)) == 1 + 5 + 3 + 2 * (2 + 1)
    assert count(prob(small, kv_group=4, r0=5, r1=5)) == 5 + 1 + 1  # no index rows on this rank
    assert count(prob(W("m_dec", 2, 1, 300, 8, 4, 64, 64, 4, 64))) == 4
    assert count(prob(W("m_dec1", 2, 1, 60, 8, 4, 64, 64, 4, 64))) == 3  # own block only: no scan
    # the attention stage's launches behind its roofline figures
    assert bench.stage_launches(small, prob(small, kv_group=4), "attn1") == 1
    assert bench.stage_launches(wide, prob(wide, kv_group=4), "attn1") == 2
    assert bench.stage_launches(wide, prob(wide, kv_group=2), "attn1") == 4
    assert bench.stage_launches(wide, prob(wide, kv_group=4), "attn2") == 1


def test_dram_traffic_entries_match_the_bench_headlines():
    """profiles/dram_traffic.json holds a valid entry, keyed as bench.py looks
    it up (dominant kernel @ workload), for both prefill workloads the bench
    reports a roofline on, each near or above the stage's algorithmic bytes (q
    once, K and V once, the bf16 partials with their lse).  The lower bound is
    0.9 x: partial rows still in the 126 MB L2 when a launch ends reach DRAM
    after it, and the entries are captures of a smaller case scaled up."""
    from block_sparse_long_05_b200.inputs import WORKLOADS
    traffic = bench.load_traffic()
    for name in ("prefill_T65536", "long_prefill_T262144"):
        w = WORKLOADS[name]
        key = f"{bench.kernel_name(w, 'attn1')}@{name}"
        assert key in traffic, key
        rows = w.Bt * w.n_q
        algo = (rows * w.Hq * w.d * 2 + 2 * w.Bt * w.T * w.Hkv * w.d * 2 +
                rows * w.K * w.Hq * (w.d * 2 + 4))
        assert 0.9 * algo <= traffic[key] <= 2 * algo, (key, traffic[key], algo)
