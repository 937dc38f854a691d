"""Decode path (n_q = 1) of the CUDA library against the CPU oracle: index
scan + top-K select (bit-exact ids) and split-K attention + combine (within
tolerance), at the full decode workload sizes and on edge shapes."""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_close, host, lib_ready, run_attn, run_index

pytestmark = pytest.mark.gpu

from block_sparse_long_05_b200.inputs import (DECODE_128K, DECODE_1M, Workload, make_inputs,
                                              random_selection)


def _decode_case(w, index_values="int3"):
    from block_sparse_long_05_b200 import msa
    from oracle import oracle
    lib_ready()
    x = make_inputs(w, device="cuda", index_values=index_values)
    ws = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
    ids = run_index(w, x, ws)
    hx = {k: host(v) for k, v in x.items()}
    ids_ref = oracle.index_topk(hx["q_idx"], hx["k_idx"], w.Bt, w.n_q, w.T, w.d_idx, w.block, w.K)
    assert np.array_equal(host(ids).numpy().reshape(-1, w.K), ids_ref), "ids differ from oracle"
    out, lse = run_attn(w, x, ids, ws)
    o_ref, l_ref = oracle.sparse_attn(hx["q"], hx["k"], hx["v"], ids_ref, w.Bt, w.n_q, w.T, w.Hq,
                                      w.Hkv, w.d, w.block, w.K)
    assert_close(host(out).numpy().reshape(o_ref.shape), o_ref, "out")
    assert_close(host(lse).numpy().reshape(l_ref.shape), l_ref, "lse")


@pytest.mark.parametrize("w", [
    Workload("dec_small", 3, 1, 1000, 8, 2, 64, 64, 4, 64),          # ragged last block
    Workload("dec_d128", 2, 1, 4096, 16, 2, 128, 128, 8, 128),
    Workload("dec_one_block", 2, 1, 50, 8, 8, 64, 64, 4, 64),        # T < block, G = 1
    Workload("dec_dense", 2, 1, 700, 8, 1, 64, 128, 16, 64),         # K >= N, G = 8
    Workload("dec_k1", 2, 1, 3000, 8, 2, 128, 512, 1, 128),          # own block only
    Workload("dec_k32", 1, 1, 20000, 4, 1, 64, 32, 32, 64),          # K = 32, block 32
    Workload("dec_max_blocks", 2, 1, 8192 * 32, 4, 1, 64, 32, 32, 64),  # N = 8192: 8 per select thread
    Workload("dec_many_heads", 48, 1, 3000, 32, 4, 64, 64, 4, 64),   # 4-warp split combine at d = 64
], ids=lambda w: w.name)
def test_decode_small(w):
    _decode_case(w)


def test_decode_index_ties():
    # all-zero index keys: every score ties, the lowest blocks win
    _decode_case(Workload("dec_ties", 2, 1, 5000, 8, 2, 64, 128, 6, 64), index_values="zeros")


def test_decode_attention_random_selection():
    from block_sparse_long_05_b200 import msa
    from oracle import oracle
    lib_ready()
    w = Workload("dec_rand", 4, 1, 9000, 16, 4, 128, 512, 8, 64)
    x = make_inputs(w, device="cuda")
    ids = random_selection(w, device="cuda")
    ws = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
    out, lse = run_attn(w, x, ids, ws)
    hx = {k: host(v) for k, v in x.items()}
    o_ref, l_ref = oracle.sparse_attn(hx["q"], hx["k"], hx["v"], host(ids).reshape(-1, w.K), w.Bt,
                                      1, w.T, w.Hq, w.Hkv, w.d, w.block, w.K)
    assert_close(host(out).numpy().reshape(o_ref.shape), o_ref, "out")
    assert_close(host(lse).numpy().reshape(l_ref.shape), l_ref, "lse")


@pytest.mark.parametrize("w", [DECODE_128K, DECODE_1M], ids=lambda w: w.name)
def test_decode_full_size(w):
    _decode_case(w)
    torch.cuda.empty_cache()


def test_decode_bad_ids_reported():
    # ids outside [-1, N) are skipped and reported through the status word
    from block_sparse_long_05_b200 import msa
    lib_ready()
    w = Workload("dec_bad", 2, 1, 1024, 8, 2, 64, 64, 4, 64)
    x = make_inputs(w, device="cuda")
    ids = torch.tensor([[[0, 3, 15, 99]], [[-7, 1, 2, 15]]], dtype=torch.int32, device="cuda")
    ws = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
    out, lse = msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws)
    assert msa.device_status(ws) == 6  # MSA_ERR_BAD_IDS
    assert msa.device_status(ws) == 0  # read-and-clear
    # the skipped ids contribute no key: each row equals the oracle over the rest
    from oracle import oracle
    hx = {k: host(v) for k, v in x.items()}
    o_ref, l_ref = oracle.sparse_attn(hx["q"], hx["k"], hx["v"], host(ids).reshape(-1, w.K), w.Bt,
                                      1, w.T, w.Hq, w.Hkv, w.d, w.block, w.K)
    assert_close(host(out).numpy().reshape(o_ref.shape), o_ref, "out")
    assert_close(host(lse).numpy().reshape(l_ref.shape), l_ref, "lse")


def test_decode_many_rows_and_heads():
    # Bt * Hq >= 4096: the combine takes the row-parallel kernel (fp32
    # partials, two splits per 128-key block) instead of the split combine
    _decode_case(Workload("dec_wide", 64, 1, 2048, 64, 8, 128, 128, 4, 64))


def test_decode_repeated_calls_one_workspace():
    # three calls in a row on one workspace, with different selections: each
    # equals the oracle (the partials of the previous call are never used)
    from block_sparse_long_05_b200 import msa
    from oracle import oracle
    lib_ready()
    w = Workload("dec_repeat", 6, 1, 5000, 16, 4, 128, 128, 6, 64)
    x = make_inputs(w, device="cuda")
    hx = {k: host(v) for k, v in x.items()}
    ws = msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
    for seed in (3, 4, 5):
        ids = random_selection(w, device="cuda", seed=seed)
        out, lse = msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws)
        assert msa.device_status(ws) == 0
        o_ref, l_ref = oracle.sparse_attn(hx["q"], hx["k"], hx["v"], host(ids).reshape(-1, w.K),
                                          w.Bt, 1, w.T, w.Hq, w.Hkv, w.d, w.block, w.K)
        assert_close(host(out).numpy().reshape(o_ref.shape), o_ref, f"out (selection {seed})")
        assert_close(host(lse).numpy().reshape(l_ref.shape), l_ref, f"lse (selection {seed})")
