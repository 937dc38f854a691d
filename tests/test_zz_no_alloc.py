"""The decode attention entry point that allocates nothing
(msa_sparse_attn_decode_noalloc), for callers that cannot allocate device
memory or pass a workspace.  Called through the C ABI, its output must match
the workspace-based msa_sparse_attn on the same decode inputs, on two calls in
a row (the static scratch keeps the previous call's contents).  This file is
collected last so that a run stopping at the first failure has already run
every other test."""
import pytest
import torch

from gpu_helpers import MAX_ABS, MEAN_ABS, lib_ready

pytestmark = pytest.mark.gpu


def _compare(a, b, what):
    err = (a.double() - b.double()).abs()
    assert torch.isfinite(a).all(), what
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, \
        f"{what}: max-abs {err.max().item():.3e} mean-abs {err.mean().item():.3e}"


def test_noalloc_decode_matches_workspace_path_twice():
    from block_sparse_long_05_b200 import msa
    from block_sparse_long_05_b200.inputs import DECODE_1M, Workload, make_inputs
    lib_ready()
    cases = [Workload("noalloc_small", 3, 1, 5000, 16, 2, 128, 128, 8, 64),
             DECODE_1M]
    for w in cases:
        x = make_inputs(w, device="cuda")
        ws = msa.Workspace.for_shape(w.Bt, 1, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
        ids = msa.index_topk(x["q_idx"], x["k_idx"], w.block, w.K, ws)
        ref_out, ref_lse = msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws)
        assert msa.device_status(ws) == 0
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for call in range(2):
            out = torch.full_like(ref_out, float("nan"))
            lse = torch.full_like(ref_lse, float("nan"))
            msa.sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], ids, w.block, out=out,
                                           lse=lse, status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            _compare(out, ref_out, f"{w.name} out, call {call}")
            _compare(lse, ref_lse, f"{w.name} lse, call {call}")
        del x, ws
        torch.cuda.empty_cache()


def test_noalloc_rejects_oversized_shape():
    from block_sparse_long_05_b200 import msa
    from block_sparse_long_05_b200.inputs import DECODE_128K
    lib = lib_ready()
    w = DECODE_128K  # 32 sequences x 16 blocks x 2 splits x 64 heads: 33.5 MB of partials
    fake = 1 << 20
    rc = lib.msa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, fake, w.Bt, w.T, w.Hq,
                                            w.Hkv, w.d, w.block, w.K, None, None)
    assert rc == 3  # MSA_ERR_WORKSPACE, nothing enqueued


def test_noalloc_without_status_and_with_many_rows():
    # status = NULL (the library clears and uses a word of its own scratch),
    # and a shape with Bt * Hq >= 4096, where the combine takes its
    # row-parallel kernel; two calls in a row, against the workspace path
    from block_sparse_long_05_b200 import msa
    from block_sparse_long_05_b200.inputs import Workload, make_inputs
    lib_ready()
    for w in (Workload("noalloc_nostatus", 3, 1, 5000, 16, 2, 128, 128, 8, 64),
              Workload("noalloc_wide", 64, 1, 2048, 64, 8, 128, 128, 3, 64)):
        x = make_inputs(w, device="cuda")
        ws = msa.Workspace.for_shape(w.Bt, 1, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
        ids = msa.index_topk(x["q_idx"], x["k_idx"], w.block, w.K, ws)
        ref_out, ref_lse = msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws)
        assert msa.device_status(ws) == 0
        for call in range(2):
            out = torch.full_like(ref_out, float("nan"))
            lse = torch.full_like(ref_lse, float("nan"))
            msa.sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], ids, w.block, out=out,
                                           lse=lse, status=None)
            torch.cuda.synchronize()
            _compare(out, ref_out, f"{w.name} out, call {call}")
            _compare(lse, ref_lse, f"{w.name} lse, call {call}")
