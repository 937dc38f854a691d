"""Prefill path (n_q > 1) of the CUDA library against the CPU oracle:
tcgen05 index kernel (bit-exact ids), selection inversion (bit-exact CSR),
KV-block-outer tcgen05 attention + log-sum-exp combine (within tolerance).
Small shapes are checked on every row; the full-size workloads on sampled
rows (uniform, seed 1, plus each sequence's first, last and a dense-early
row)."""
import os

import numpy as np
import pytest
import torch

from gpu_helpers import assert_close, host, lib_ready, rows_of, run_attn, run_index

pytestmark = pytest.mark.gpu

from block_sparse_long_05_b200.inputs import (PREFILL_256K, PREFILL_64K, TINY_PREFILL, Workload,
                                              make_inputs, random_selection, sample_rows)

N_SAMPLE = int(os.environ.get("MSA_TEST_SAMPLE_ROWS", "4096"))


def _ws(w):
    from block_sparse_long_05_b200 import msa
    return msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)


def _check_ids(w, x, ids, rows):
    from oracle import oracle
    exp = oracle.index_topk(host(x["q_idx"]), host(x["k_idx"]), w.Bt, w.n_q, w.T, w.d_idx,
                            w.block, w.K, rows=rows.numpy())
    got = host(rows_of(ids, rows, w.K)).numpy()
    bad = np.nonzero(~np.all(got == exp, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first row {int(rows[bad[0]])}: " \
                          f"{got[bad[0]]} vs {exp[bad[0]]}"
    return exp


def _check_attn(w, x, ids_rows, out, lse, rows):
    from oracle import oracle
    hq, hk, hv = host(x["q"]), host(x["k"]), host(x["v"])
    o_ref, l_ref = oracle.sparse_attn(hq, hk, hv, ids_rows, w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d,
                                      w.block, w.K, rows=rows.numpy())
    assert_close(host(rows_of(out, rows, 0)).numpy(), o_ref, "out")
    assert_close(host(rows_of(lse, rows, 0)).numpy(), l_ref, "lse")


def _end_to_end(w, rows=None, index_values="int3"):
    lib_ready()
    x = make_inputs(w, device="cuda", index_values=index_values)
    ws = _ws(w)
    ids = run_index(w, x, ws)
    if rows is None:
        rows = torch.arange(w.Bt * w.n_q, dtype=torch.int64)
    ids_ref = _check_ids(w, x, ids, rows)
    out, lse = run_attn(w, x, ids, ws)
    _check_attn(w, x, ids_ref, out, lse, rows)


SMALL = [
    Workload("pf_tiny_b64", 1, 512, 512, 8, 2, 64, 64, 4, 64),
    Workload("pf_ragged", 2, 1000, 1000, 8, 2, 64, 64, 4, 64),        # T % block != 0, Bt = 2
    Workload("pf_b128_d128", 1, 2048, 2048, 16, 2, 128, 128, 8, 128),
    Workload("pf_b256", 1, 2048, 2048, 8, 1, 128, 256, 4, 128),       # streamed KV sub-tiles, G=8
    Workload("pf_b512", 1, 3000, 3000, 8, 4, 128, 512, 3, 64),        # ragged, 4 sub-tiles
    Workload("pf_b32_k32", 1, 1500, 1500, 4, 4, 64, 32, 32, 64),      # G = 1, K = 32
    Workload("pf_dense", 1, 700, 700, 8, 2, 64, 64, 16, 128),         # K >= N: dense causal
    Workload("pf_k1", 2, 600, 600, 8, 2, 128, 64, 1, 64),             # own block only
    Workload("pf_chunk", 2, 300, 2000, 8, 2, 64, 128, 6, 64),         # last n_q queries only
    Workload("pf_short", 1, 40, 40, 8, 2, 64, 64, 4, 64),             # single block, T < block
    # own-block pass with the first own rows mid-block (T - n_q = 2300), Bt = 2
    Workload("pf_chunk_b512", 2, 700, 3000, 8, 2, 64, 512, 4, 64),
    # 8 sub-tiles; G = 16 splits each block's 1024 own rows into two work items
    Workload("pf_b1024_g16", 1, 2500, 2500, 16, 1, 64, 1024, 2, 64),
    # own block only: every hit list is empty, the own-block launch does all the work
    Workload("pf_k1_b256", 2, 900, 900, 8, 2, 64, 256, 1, 64),
    # K >= N: dense causal over 256-key blocks
    Workload("pf_dense_b256", 1, 1100, 1100, 8, 2, 128, 256, 8, 128),
    # d = 128, G = 8, chunked queries over 512-key blocks, own rows from mid-block
    Workload("pf_chunk_b512_g8", 1, 1500, 4000, 16, 2, 128, 512, 3, 128),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_prefill_small_all_rows(w):
    _end_to_end(w)


def test_prefill_index_ties():
    _end_to_end(Workload("pf_ties", 1, 1024, 1024, 8, 2, 64, 64, 5, 64), index_values="zeros")


def test_prefill_tiny_workload_all_rows():
    _end_to_end(TINY_PREFILL)


@pytest.mark.parametrize("w", [SMALL[1], SMALL[3], SMALL[4], SMALL[8]], ids=lambda w: w.name)
def test_inversion_exact(w):
    from block_sparse_long_05_b200 import msa
    from oracle import oracle
    lib_ready()
    ids = random_selection(w, device="cuda")
    ws = _ws(w)
    row_ptr, entries = msa.select_invert(ids, w.T, w.block, ws)
    assert msa.device_status(ws) == 0
    rp_ref, ent_ref = oracle.select_invert(host(ids), w.Bt, w.n_q, w.T, w.block, w.K)
    rp = host(row_ptr).numpy()
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(host(entries).numpy()[: rp[-1]], ent_ref)


def test_inversion_full_size():
    from block_sparse_long_05_b200 import msa
    from oracle import oracle
    lib_ready()
    w = PREFILL_256K
    ids = random_selection(w, device="cuda")
    ws = msa.Workspace(1 << 28)
    row_ptr, entries = msa.select_invert(ids, w.T, w.block, ws)
    assert msa.device_status(ws) == 0
    rp_ref, ent_ref = oracle.select_invert(host(ids), w.Bt, w.n_q, w.T, w.block, w.K)
    rp = host(row_ptr).numpy()
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(host(entries).numpy()[: rp[-1]], ent_ref)


@pytest.mark.parametrize("w", [SMALL[2], SMALL[4], SMALL[5]], ids=lambda w: w.name)
def test_attention_random_selection(w):
    # the sparse branch alone, on a seeded random selection of the same structure
    lib_ready()
    x = make_inputs(w, device="cuda")
    ids = random_selection(w, device="cuda")
    out, lse = run_attn(w, x, ids, _ws(w))
    rows = torch.arange(w.Bt * w.n_q, dtype=torch.int64)
    _check_attn(w, x, host(ids).reshape(-1, w.K).numpy(), out, lse, rows)


@pytest.mark.parametrize("w", [SMALL[0], SMALL[2], SMALL[3]], ids=lambda w: w.name)
@pytest.mark.parametrize("rising", [True, False], ids=["rising", "falling"])
def test_attention_score_spread(w, rising):
    # Keys far apart in score within one block (x6 on one side of the block),
    # so a row's largest scores sit in a later (rising) or the first (falling)
    # 32-key group: exercises the softmax reference-max updates.
    lib_ready()
    x = make_inputs(w, device="cuda")
    pos = torch.arange(w.T, device="cuda") % w.block
    big = (pos >= w.block // 2) if rising else (pos < 32)
    scale = torch.where(big, 6.0, 1.0).to(torch.float32)
    x["k"] = (x["k"].float() * scale.view(1, -1, 1, 1)).to(torch.bfloat16)
    ids = random_selection(w, device="cuda")
    out, lse = run_attn(w, x, ids, _ws(w))
    rows = torch.arange(w.Bt * w.n_q, dtype=torch.int64)
    _check_attn(w, x, host(ids).reshape(-1, w.K).numpy(), out, lse, rows)


def test_prefill_max_blocks():
    # N = 8192 blocks (the largest supported: inversion histograms of 4 x N
    # counters in shared memory) and K = 32 (the largest): the last 256
    # queries of a 262144-key context with 32-key blocks, every row checked
    _end_to_end(Workload("pf_max_blocks", 1, 256, 8192 * 32, 4, 1, 64, 32, 32, 64))


@pytest.mark.parametrize("w", [PREFILL_64K, PREFILL_256K], ids=lambda w: w.name)
def test_prefill_full_size_sampled(w):
    _end_to_end(w, rows=sample_rows(w, N_SAMPLE))
    torch.cuda.empty_cache()


def test_prefill_bad_ids_reported():
    from block_sparse_long_05_b200 import msa
    lib_ready()
    w = Workload("pf_bad", 1, 256, 256, 8, 2, 64, 64, 2, 64)
    x = make_inputs(w, device="cuda")
    ids = random_selection(w, device="cuda")
    ids[0, 5, 1] = 77      # beyond N = 4
    ids[0, 9, 1] = -3
    ws = _ws(w)
    out, lse = msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws)
    assert msa.device_status(ws) == 6  # MSA_ERR_BAD_IDS
    assert torch.isfinite(out[0, 100]).all()


def _with_odd_ids(w, ids, beyond_own=True, out_of_range=True):
    """A copy of a selection with, in some rows, one slot replaced by a block
    after the row's own block (such a block holds no key at or before t) and,
    in other rows, one slot replaced by an id >= N (skipped and reported)."""
    h = ids.cpu().clone().view(-1, w.K)
    N = w.n_blocks
    for r in range(h.shape[0]):
        t = w.T - w.n_q + r % w.n_q
        own = t // w.block
        row = h[r].tolist()
        # the slot to replace: a -1 pad if there is one, else a non-own block
        cand = [s for s in range(w.K) if row[s] == -1] or [s for s in range(w.K) if row[s] != own]
        if not cand:
            continue
        s = cand[r % len(cand)]
        if beyond_own and r % 3 == 0 and own + 1 < N:
            later = [j for j in range(own + 1, N) if j not in row]
            h[r, s] = later[r % len(later)]
        elif out_of_range and r % 3 == 1:
            h[r, s] = N + r % 5
    return h.view_as(ids).to(ids.device)


@pytest.mark.parametrize("out_of_range", [False, True], ids=["beyond_own", "beyond_own_and_N"])
def test_prefill_ids_beyond_own_and_out_of_range(out_of_range):
    # a block after own(t) contributes no key; an id >= N is skipped (and
    # reported): either way the row equals the attention over its other ids
    from block_sparse_long_05_b200 import msa
    lib_ready()
    for w in (Workload("pf_odd_ids", 1, 1024, 1024, 8, 2, 64, 64, 4, 64),
              Workload("pf_odd_ids_b512", 1, 3000, 3000, 8, 4, 128, 512, 3, 64)):
        x = make_inputs(w, device="cuda")
        ids = _with_odd_ids(w, random_selection(w, device="cuda"), out_of_range=out_of_range)
        ws = _ws(w)
        out, lse = msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws)
        assert msa.device_status(ws) == (6 if out_of_range else 0)
        rows = torch.arange(w.Bt * w.n_q, dtype=torch.int64)
        _check_attn(w, x, host(ids).reshape(-1, w.K).numpy(), out, lse, rows)


def _without_own(w, ids):
    """A copy of a selection in which every other row that also selected an
    earlier block drops its own block (the slot becomes -1; the own block is
    the row's largest id, so the row stays ascending)."""
    h = ids.cpu().clone().view(-1, w.K)
    for r in range(0, h.shape[0], 2):
        own = (w.T - w.n_q + r % w.n_q) // w.block
        row = h[r].tolist()
        if own in row and any(0 <= j < own for j in row):
            h[r, row.index(own)] = -1
    return h.view_as(ids).to(ids.device)


def test_prefill_rows_without_own_block():
    # the selection is the caller's: a row that left out its own block attends
    # its other blocks only (the own-block launch skips it)
    from block_sparse_long_05_b200 import msa
    lib_ready()
    for w in (Workload("pf_no_own", 1, 1024, 1024, 8, 2, 64, 64, 4, 64),
              Workload("pf_no_own_b512", 1, 3000, 3000, 8, 4, 128, 512, 3, 64)):
        x = make_inputs(w, device="cuda")
        ids = _without_own(w, random_selection(w, device="cuda"))
        ws = _ws(w)
        out, lse = msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws)
        assert msa.device_status(ws) == 0
        rows = torch.arange(w.Bt * w.n_q, dtype=torch.int64)
        _check_attn(w, x, host(ids).reshape(-1, w.K).numpy(), out, lse, rows)


@pytest.mark.parametrize("w", [SMALL[2], SMALL[3], SMALL[4], SMALL[5], SMALL[10]],
                         ids=lambda w: w.name)
def test_attention_kv_head_groups(w):
    # workspaces that hold the partials of 1 and of 2 kv heads: the kv heads
    # are attended and merged group by group; every row must equal the oracle
    # (and the one-pass result)
    from block_sparse_long_05_b200 import msa
    lib_ready()
    x = make_inputs(w, device="cuda")
    ids = random_selection(w, device="cuda")
    one = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K,
                                  kv_group=w.Hkv)
    ref_out, ref_lse = run_attn(w, x, ids, one)
    rows = torch.arange(w.Bt * w.n_q, dtype=torch.int64)
    for g in sorted({1, 2} & {d for d in range(1, w.Hkv + 1) if w.Hkv % d == 0}):
        ws = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K,
                                     kv_group=g)
        out, lse = run_attn(w, x, ids, ws)
        _check_attn(w, x, host(ids).reshape(-1, w.K).numpy(), out, lse, rows)
        assert torch.allclose(out, ref_out, atol=1e-6, rtol=0) and \
            torch.allclose(lse, ref_lse, atol=1e-6, rtol=0), f"kv_group {g} differs from one pass"
