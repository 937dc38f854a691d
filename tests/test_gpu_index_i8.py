"""The index branch on signed 8-bit index keys (msa_index_topk_i8: tcgen05
kind::i8 for prefill, dp4a scan for decode) against the CPU oracle, which
reads the same integer values as bf16: ids bit-exact on every row of small
shapes (both index dims, ragged tails, ties, K = 1 and 32, the largest N),
on 4096 sampled rows of the full 64K and 256K prefills, and on every
sequence of the full decode workloads.  The full-size cases also check that
the i8 ids equal the bf16 path's ids on every row."""
import os

import numpy as np
import pytest
import torch

from gpu_helpers import host, lib_ready, rows_of

pytestmark = pytest.mark.gpu

from block_sparse_long_05_b200.inputs import (DECODE_128K, DECODE_1M, PREFILL_256K, PREFILL_64K,
                                              TINY_PREFILL, Workload, make_inputs, sample_rows)

N_SAMPLE = int(os.environ.get("MSA_TEST_SAMPLE_ROWS", "4096"))


def _ws(w):
    from block_sparse_long_05_b200 import msa
    return msa.Workspace.for_shape(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)


def _i8(t):
    return t.to(torch.int8)  # the integer values, exactly


def _run(w, rows=None, index_values="int3", compare_bf16=False):
    from block_sparse_long_05_b200 import msa
    from oracle import oracle
    lib_ready()
    x = make_inputs(w, device="cuda", index_values=index_values)
    ws = _ws(w)
    ids = msa.index_topk_i8(_i8(x["q_idx"]), _i8(x["k_idx"]), w.block, w.K, ws)
    assert msa.device_status(ws) == 0
    if rows is None:
        rows = torch.arange(w.Bt * w.n_q, dtype=torch.int64)
    exp = oracle.index_topk(host(x["q_idx"]), host(x["k_idx"]), w.Bt, w.n_q, w.T, w.d_idx,
                            w.block, w.K, rows=rows.numpy())
    got = host(rows_of(ids, rows, w.K)).numpy()
    bad = np.nonzero(~np.all(got == exp, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first row {int(rows[bad[0]])}: " \
                          f"{got[bad[0]]} vs {exp[bad[0]]}"
    if compare_bf16:
        ref = msa.index_topk(x["q_idx"], x["k_idx"], w.block, w.K, ws)
        assert msa.device_status(ws) == 0
        assert torch.equal(ids, ref), "i8 ids differ from the bf16 path"


@pytest.mark.parametrize("w", [
    Workload("i8_tiny_b64", 1, 512, 512, 8, 2, 64, 64, 4, 64),
    Workload("i8_ragged", 2, 1000, 1000, 8, 2, 64, 64, 4, 64),
    Workload("i8_d128", 1, 2048, 2048, 16, 2, 128, 128, 8, 128),
    Workload("i8_b512", 1, 3000, 3000, 8, 4, 128, 512, 3, 64),
    Workload("i8_b32_k32", 1, 1500, 1500, 4, 4, 64, 32, 32, 64),
    Workload("i8_k1", 2, 600, 600, 8, 2, 128, 64, 1, 128),
    Workload("i8_chunk", 2, 300, 2000, 8, 2, 64, 128, 6, 128),
    Workload("i8_short", 1, 40, 40, 8, 2, 64, 64, 4, 64),
    Workload("i8_max_blocks", 1, 256, 8192 * 32, 4, 1, 64, 32, 32, 64),
    TINY_PREFILL,
], ids=lambda w: w.name)
def test_index_i8_prefill_all_rows(w):
    _run(w)


@pytest.mark.parametrize("w", [
    Workload("i8_dec_small", 3, 1, 1000, 8, 2, 64, 64, 4, 64),
    Workload("i8_dec_d128", 2, 1, 4096, 16, 2, 128, 128, 8, 128),
    Workload("i8_dec_one_block", 2, 1, 50, 8, 8, 64, 64, 4, 64),
    Workload("i8_dec_k32", 1, 1, 20000, 4, 1, 64, 32, 32, 64),
    Workload("i8_dec_b512", 2, 1, 3000, 8, 2, 128, 512, 4, 128),
], ids=lambda w: w.name)
def test_index_i8_decode(w):
    _run(w)


@pytest.mark.parametrize("w", [Workload("i8_ties", 1, 1024, 1024, 8, 2, 64, 64, 5, 64),
                               Workload("i8_dec_ties", 2, 1, 5000, 8, 2, 64, 128, 6, 128)],
                         ids=lambda w: w.name)
def test_index_i8_ties(w):
    _run(w, index_values="zeros")


@pytest.mark.parametrize("w", [PREFILL_64K, PREFILL_256K], ids=lambda w: w.name)
def test_index_i8_full_prefill_sampled(w):
    _run(w, rows=sample_rows(w, N_SAMPLE), compare_bf16=True)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("w", [DECODE_128K, DECODE_1M], ids=lambda w: w.name)
def test_index_i8_full_decode(w):
    _run(w, compare_bf16=True)
    torch.cuda.empty_cache()


def test_index_i8_rejects_bf16_tensors():
    from block_sparse_long_05_b200 import msa
    lib_ready()
    w = Workload("i8_types", 1, 256, 256, 8, 2, 64, 64, 4, 64)
    x = make_inputs(w, device="cuda")
    with pytest.raises(ValueError):
        msa.index_topk_i8(x["q_idx"], x["k_idx"], w.block, w.K, _ws(w))
