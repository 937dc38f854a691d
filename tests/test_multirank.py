"""bench.py's multi-rank path on CPU: two gloo ranks launched the way the
benchmark is launched on several GPUs (torch.distributed.run, 127.0.0.1).
Checks weak-scaling sharding (each rank its own seeded sequences, equal to a
single-process run of that shard), the max over ranks of the step time, the
whole-job throughput, and that the reference arm prints on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_shard_and_reduce(orc):
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}",
           os.path.join(ROOT, "tests", "multirank_worker.py")]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
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
