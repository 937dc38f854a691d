"""The multi-rank paths on CPU: gloo ranks launched the way the benchmark is
launched on several GPUs (torch.distributed.run, 127.0.0.1).
Checks weak-scaling sharding (each rank its own seeded sequences, equal to a
single-process run of that shard), the max over ranks of the step time, the
whole-job throughput, that the reference arm prints on rank 0 only, and the
kv-head-sharded prefill partition (row-split index branch, all-gathered ids,
head-sliced sparse branch) against a single-process oracle run."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(script, nproc=2):
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={nproc}", "--master-addr=127.0.0.1",
           f"--master-port={_free_port()}", os.path.join(ROOT, "tests", script)]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_two_gloo_ranks_shard_and_reduce(orc):
    r = _launch("multirank_worker.py")
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout  # rank 0 alone prints
    res = json.loads(lines[0])
    assert res["world"] == 2
    assert res["ms"] == [11.0, 5.0]  # element-wise max over the two ranks
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import multirank_worker as mw
    w = mw.SHARD
    assert abs(res["value"] - w.Bt * w.n_q * 2 / 11.0e-3) < 1e-6
    # every rank ran its own shard: digests differ, and each equals a
    # single-process run of that rank's seed
    d0, d1 = res["digests"]
    assert d0 != d1
    for rank, got in enumerate((d0, d1)):
        ids, out, lse = mw.shard_result(rank)
        exp = [float(np.abs(out).sum()), float(lse.sum()), float(ids.sum())]
        assert np.allclose(got, exp, rtol=0, atol=1e-9), (rank, got, exp)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("nproc", [2, 4])
def test_head_sharded_prefill_equals_single_rank(orc, nproc):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import shard_worker as sw
    from block_sparse_long_05_b200.inputs import make_inputs
    r = _launch("shard_worker.py", nproc)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    res = json.loads(lines[0])
    w = sw.PREFILL
    # the row ranges tile the query rows, one per rank, in order
    rg = res["ranges"]
    assert len(rg) == nproc and rg[0][0] == 0 and rg[-1][1] == w.n_q
    assert all(a[1] == b[0] for a, b in zip(rg, rg[1:]))
    x = make_inputs(w, device="cpu")
    ids = orc.index_topk(x["q_idx"], x["k_idx"], w.Bt, w.n_q, w.T, w.d_idx, w.block, w.K)
    assert np.array_equal(np.asarray(res["ids"]), ids)  # the gathered ids, bit for bit
    out, lse = orc.sparse_attn(x["q"], x["k"], x["v"], ids, w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d,
                               w.block, w.K)
    Hr = w.Hq // nproc
    for rank, part in enumerate(res["parts"]):
        part = np.asarray(part)
        h0 = rank * Hr
        got_out = part[:, :Hr * w.d].reshape(w.n_q, Hr, w.d)
        got_lse = part[:, Hr * w.d:]
        assert np.array_equal(got_out, out[:, h0:h0 + Hr]), rank
        assert np.array_equal(got_lse, lse[:, h0:h0 + Hr]), rank


def test_index_row_ranges_balance_and_tile():
    from block_sparse_long_05_b200 import shard
    for n_q, T, block, world in ((65536, 65536, 128, 4), (262144, 262144, 512, 8),
                                 (1000, 3000, 64, 3), (300, 300, 64, 4), (100, 100, 64, 8)):
        rg = shard.index_row_ranges(n_q, T, block, world)
        assert len(rg) == world and rg[0][0] == 0 and rg[-1][1] == n_q
        for (a0, a1), (b0, b1) in zip(rg, rg[1:]):
            assert a1 == b0 and a0 <= a1
            assert a1 % 128 == 0 or a1 == n_q
        if n_q >= 128 * world * 8:
            # work per rank (candidate blocks + 1 per row) within 2% of the mean
            t = np.arange(n_q) + (T - n_q)
            cost = t // block + 1
            per = [cost[r0:r1].sum() for r0, r1 in rg]
            assert max(per) <= 1.02 * np.mean(per), per
    assert shard.head_range(8, 4, 3) == (6, 8)
    with pytest.raises(ValueError):
        shard.head_range(8, 3, 0)
