"""Paged-KV decode (msa_index_topk_paged, msa_sparse_attn_paged) against the
CPU oracle run on the same keys laid out contiguously: the pages are a
random permutation of a store with spare pages, the page-table rows have
unused tail entries, and every row the kernels must not read (spare pages,
the rows past T in the last page) holds large values that would change the
result if read.  A page id outside the store is reported as MSA_ERR_BAD_IDS."""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_close, host, lib_ready

pytestmark = pytest.mark.gpu

from block_sparse_long_05_b200.inputs import Workload, make_inputs

POISON = 64.0  # a value no kept row holds (keys are N(0,1) or integers in [-3, 3])


def _paged(w, x, spare=5, pad=3, seed=11):
    """Scatter x's k_idx, k, v into a permuted page store; returns the store
    and the page table [Bt, N + pad]."""
    N = (w.T + w.block - 1) // w.block
    n_pages = w.Bt * N + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)
    table = torch.full((w.Bt, N + pad), -7, dtype=torch.int32)
    ki = torch.full((n_pages, w.block, w.d_idx), POISON, dtype=torch.bfloat16, device="cuda")
    kp = torch.full((n_pages, w.block, w.Hkv, w.d), POISON, dtype=torch.bfloat16, device="cuda")
    vp = torch.full((n_pages, w.block, w.Hkv, w.d), POISON, dtype=torch.bfloat16, device="cuda")
    for b in range(w.Bt):
        for j in range(N):
            p = int(perm[b * N + j])
            table[b, j] = p
            lo, hi = j * w.block, min((j + 1) * w.block, w.T)
            ki[p, :hi - lo] = x["k_idx"][b, lo:hi]
            kp[p, :hi - lo] = x["k"][b, lo:hi]
            vp[p, :hi - lo] = x["v"][b, lo:hi]
    return ki, kp, vp, table.cuda()


@pytest.mark.parametrize("w", [
    Workload("paged_small", 3, 1, 1000, 8, 2, 64, 64, 4, 64),       # ragged last page
    Workload("paged_d128", 2, 1, 4096, 16, 2, 128, 128, 8, 128),
    Workload("paged_b512", 2, 1, 5000, 16, 4, 128, 512, 4, 128),    # 8 splits per page
    Workload("paged_one_block", 2, 1, 50, 8, 8, 64, 64, 4, 64),     # T < block
    Workload("paged_k32", 1, 1, 20000, 4, 1, 64, 32, 32, 64),
], ids=lambda w: w.name)
def test_paged_decode_matches_oracle(w):
    from block_sparse_long_05_b200 import msa
    from oracle import oracle
    lib_ready()
    x = make_inputs(w, device="cuda")
    ki, kp, vp, table = _paged(w, x)
    ws = msa.Workspace.for_shape(w.Bt, 1, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
    ids = msa.index_topk_paged(x["q_idx"], ki, table, w.T, w.K, ws)
    out, lse = msa.sparse_attn_paged(x["q"], kp, vp, table, w.T, ids, ws)
    st = msa.device_status(ws)
    assert st == 0, msa.status_string(st)
    hx = {k: host(v) for k, v in x.items()}
    ids_ref = oracle.index_topk(hx["q_idx"], hx["k_idx"], w.Bt, 1, w.T, w.d_idx, w.block, w.K)
    assert np.array_equal(host(ids).numpy().reshape(-1, w.K), ids_ref), "ids differ from oracle"
    o_ref, l_ref = oracle.sparse_attn(hx["q"], hx["k"], hx["v"], ids_ref, w.Bt, 1, w.T, w.Hq,
                                      w.Hkv, w.d, w.block, w.K)
    assert_close(host(out).numpy().reshape(o_ref.shape), o_ref, "out")
    assert_close(host(lse).numpy().reshape(l_ref.shape), l_ref, "lse")


def test_paged_bad_page_reported():
    from block_sparse_long_05_b200 import msa
    lib_ready()
    w = Workload("paged_bad", 2, 1, 1024, 8, 2, 64, 64, 4, 64)
    x = make_inputs(w, device="cuda")
    ki, kp, vp, table = _paged(w, x)
    ws = msa.Workspace.for_shape(w.Bt, 1, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
    bad = table.clone()
    bad[0, 3] = ki.shape[0] + 9  # past the store
    msa.index_topk_paged(x["q_idx"], ki, bad, w.T, w.K, ws)
    assert msa.device_status(ws) == 6  # MSA_ERR_BAD_IDS
    ids = msa.index_topk_paged(x["q_idx"], ki, table, w.T, w.K, ws)
    assert msa.device_status(ws) == 0
    bad = table.clone()
    bad[1, int(ids[1, 0, 0])] = -2  # a selected block of sequence 1
    msa.sparse_attn_paged(x["q"], kp, vp, bad, w.T, ids, ws)
    assert msa.device_status(ws) == 6
    torch.cuda.synchronize()
