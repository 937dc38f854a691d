"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, sizes workspaces, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_long_05_b200 import build, msa
    build.build()
    return msa.load_library()


def header_functions():
    with open(os.path.join(ROOT, "include", "msa.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^MSA_API\s+(?:const\s+)?\w+\s*\*?\s*(msa_\w+)\s*\(", text, re.M)))


def test_header_symbols_exported(lib):
    names = header_functions()
    assert len(names) >= 7, names
    for n in names:
        assert hasattr(lib, n), n
    from block_sparse_long_05_b200 import msa
    assert sorted(msa.EXPORTED) == names


def test_status_strings(lib):
    from block_sparse_long_05_b200 import msa
    for code, name in msa.STATUS.items():
        assert lib.msa_status_string(code).decode() == name
    assert lib.msa_status_string(99).decode() == "unknown status"


def test_workspace_size(lib):
    from block_sparse_long_05_b200.inputs import WORKLOADS
    for w in WORKLOADS.values():
        n = lib.msa_workspace_size(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
        assert n > 0 and n % 256 == 0, w
    # prefill partials dominate: Bt*n_q*K*(heads of one pass)*(2d + 4) bytes; the
    # minimum holds one kv-head group's partials, the one-pass size all heads'
    for name in ("prefill_T65536", "long_prefill_T262144"):
        w = WORKLOADS[name]
        args = (w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K)
        n_min = lib.msa_workspace_size(*args)
        n_one = lib.msa_workspace_size_kv_group(*args, w.Hkv)
        part = w.T * w.K * w.Hq * (2 * w.d + 4)
        assert n_one >= part
        assert n_min <= max(5 << 30, n_one // w.Hkv + (64 << 20))
        for g in range(1, w.Hkv + 1):
            n_g = lib.msa_workspace_size_kv_group(*args, g)
            if w.Hkv % g:
                assert n_g == 0
            else:
                assert n_g >= part * g // w.Hkv and n_g <= n_one
    w = WORKLOADS["long_prefill_T262144"]
    assert lib.msa_workspace_size(w.Bt, w.n_q, w.T, w.Hq, w.Hkv, w.d, w.d_idx, w.block, w.K) \
        < 5 * 10**9
    # rejected shapes give 0
    assert lib.msa_workspace_size(1, 8, 4, 8, 2, 64, 64, 64, 8) == 0      # n_q > T
    assert lib.msa_workspace_size(1, 8, 64, 8, 3, 64, 64, 64, 8) == 0     # Hq % Hkv
    assert lib.msa_workspace_size(1, 8, 64, 8, 2, 96, 64, 64, 8) == 0     # d unsupported
    assert lib.msa_workspace_size(1, 8, 64, 8, 2, 64, 64, 48, 8) == 0     # block unsupported
    assert lib.msa_workspace_size(1, 8, 64, 8, 2, 64, 64, 64, 33) == 0    # K > 32


FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: every case fails on the host


def test_index_topk_host_validation(lib):
    call = lib.msa_index_topk
    assert call(None, FAKE, FAKE, 1, 8, 8, 64, 64, 4, FAKE, 1 << 20, None) == 1
    assert call(FAKE, FAKE, FAKE, 1, 9, 8, 64, 64, 4, FAKE, 1 << 20, None) == 1   # n_q > T
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 0, 64, 4, FAKE, 1 << 20, None) == 1    # d_idx < 1
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 96, 64, 4, FAKE, 1 << 20, None) == 2   # d_idx
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 64, 100, 4, FAKE, 1 << 20, None) == 2  # block
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 64, 64, 0, FAKE, 1 << 20, None) == 1   # K
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 64, 64, 4, None, 1 << 20, None) == 3   # no ws
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 64, 64, 4, FAKE, 16, None) == 3        # ws small
    mis = ctypes.c_void_p((1 << 20) + 128)
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 64, 64, 4, mis, 1 << 20, None) == 3    # ws align
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert call(odd, FAKE, FAKE, 1, 8, 8, 64, 64, 4, FAKE, 1 << 20, None) == 1    # q align


def test_sparse_attn_host_validation(lib):
    call = lib.msa_sparse_attn
    ok = (FAKE,) * 6
    assert call(None, *ok[1:], 1, 8, 8, 8, 2, 64, 64, 4, FAKE, 1 << 30, None) == 1
    assert call(*ok, 1, 8, 8, 8, 3, 64, 64, 4, FAKE, 1 << 30, None) == 1   # Hq % Hkv
    assert call(*ok, 1, 8, 8, 8, 2, 80, 64, 4, FAKE, 1 << 30, None) == 2   # d
    assert call(*ok, 1, 8, 8, 256, 1, 64, 64, 4, FAKE, 1 << 30, None) == 2  # G = 256 > 128
    assert call(*ok, 1, 8, 8, 8, 2, 64, 64, 4, FAKE, 64, None) == 3        # ws small
    # prefill with more than 8192 blocks is outside the supported shapes
    assert call(*ok, 1, 2, 8193 * 32, 8, 2, 64, 32, 4, FAKE, 1 << 40, None) == 2
    # q larger than 2^34 elements (offsets are 32-bit in 16-byte units)
    assert call(*ok, 1, 1 << 20, 1 << 20, 128, 1, 128, 128, 4, FAKE, 1 << 50, None) == 2


def test_misaligned_outputs_rejected_on_host(lib):
    # out is written with 16-byte stores, ids and lse as 4-byte words: a
    # misaligned pointer is rejected before anything is enqueued
    att = lib.msa_sparse_attn
    odd4 = ctypes.c_void_p((1 << 20) + 4)   # 4-byte but not 16-byte aligned
    odd2 = ctypes.c_void_p((1 << 20) + 2)   # not 4-byte aligned
    # q, k, v, ids, out, lse, Bt, n_q, T, Hq, Hkv, d, block, K, ws, bytes, stream
    args = (1, 8, 8, 8, 2, 64, 64, 4, FAKE, 1 << 30, None)
    assert att(FAKE, FAKE, FAKE, FAKE, odd4, FAKE, *args) == 1      # out
    assert att(FAKE, FAKE, FAKE, FAKE, FAKE, odd2, *args) == 1      # lse
    assert att(FAKE, FAKE, FAKE, odd2, FAKE, FAKE, *args) == 1      # ids
    dec = (1, 1, 8, 8, 2, 64, 64, 4, FAKE, 1 << 30, None)           # decode shape
    assert att(FAKE, FAKE, FAKE, FAKE, odd4, FAKE, *dec) == 1
    idx = lib.msa_index_topk
    assert idx(FAKE, FAKE, odd2, 1, 8, 8, 64, 64, 4, FAKE, 1 << 20, None) == 1  # ids
    inv = lib.msa_select_invert
    assert inv(FAKE, odd2, FAKE, 1, 8, 8, 64, 4, FAKE, 1 << 20, None) == 1      # row_ptr
    na = lib.msa_sparse_attn_decode_noalloc
    # q, k, v, ids, out, lse, Bt, T, Hq, Hkv, d, block, K, status, stream
    assert na(FAKE, FAKE, FAKE, FAKE, odd4, FAKE, 1, 1000, 8, 2, 64, 64, 4, None, None) == 1
    assert na(FAKE, FAKE, FAKE, FAKE, FAKE, odd2, 1, 1000, 8, 2, 64, 64, 4, None, None) == 1
    assert na(FAKE, FAKE, FAKE, odd2, FAKE, FAKE, 1, 1000, 8, 2, 64, 64, 4, None, None) == 1
    pa = lib.msa_sparse_attn_paged
    # q, k_pages, v_pages, table, stride, pages, ids, out, lse, Bt, T, Hq, Hkv, d, block, K, ...
    assert pa(FAKE, FAKE, FAKE, FAKE, 8, 16, FAKE, odd4, FAKE, 1, 512, 8, 2, 64, 64, 4, FAKE,
              1 << 20, None) == 1


def test_paged_decode_host_validation(lib):
    idx = lib.msa_index_topk_paged
    # q_idx, k_idx_pages, page_table, stride, pages, ids, Bt, T, d_idx, block, K, ws, bytes, stream
    assert idx(None, FAKE, FAKE, 8, 16, FAKE, 1, 512, 64, 64, 4, FAKE, 1 << 20, None) == 1
    assert idx(FAKE, FAKE, FAKE, 7, 16, FAKE, 1, 512, 64, 64, 4, FAKE, 1 << 20, None) == 1  # stride < N
    assert idx(FAKE, FAKE, FAKE, 8, 0, FAKE, 1, 512, 64, 64, 4, FAKE, 1 << 20, None) == 1   # no pages
    assert idx(FAKE, FAKE, FAKE, 8, 16, FAKE, 1, 512, 96, 64, 4, FAKE, 1 << 20, None) == 2  # d_idx
    assert idx(FAKE, FAKE, FAKE, 8, 16, FAKE, 1, 512, 64, 64, 4, FAKE, 16, None) == 3       # ws
    att = lib.msa_sparse_attn_paged
    ok = (FAKE,) * 4
    # q, k_pages, v_pages, table, stride, pages, ids, out, lse, Bt, T, Hq, Hkv, d, block, K, ws...
    assert att(*ok, 8, 16, FAKE, FAKE, None, 1, 512, 8, 2, 64, 64, 4, FAKE, 1 << 20, None) == 1
    assert att(*ok, 7, 16, FAKE, FAKE, FAKE, 1, 512, 8, 2, 64, 64, 4, FAKE, 1 << 20, None) == 1
    assert att(*ok, 8, 16, FAKE, FAKE, FAKE, 1, 512, 8, 3, 64, 64, 4, FAKE, 1 << 20, None) == 1
    assert att(*ok, 8, 16, FAKE, FAKE, FAKE, 1, 512, 8, 2, 80, 64, 4, FAKE, 1 << 20, None) == 2
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert att(FAKE, FAKE, FAKE, odd, 8, 16, FAKE, FAKE, FAKE, 1, 512, 8, 2, 64, 64, 4, FAKE,
               1 << 20, None) == 1  # page table not 4-byte aligned


def test_index_topk_i8_host_validation(lib):
    call = lib.msa_index_topk_i8
    assert call(None, FAKE, FAKE, 1, 8, 8, 64, 64, 4, FAKE, 1 << 20, None) == 1
    assert call(FAKE, FAKE, FAKE, 1, 9, 8, 64, 64, 4, FAKE, 1 << 20, None) == 1   # n_q > T
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 96, 64, 4, FAKE, 1 << 20, None) == 2   # d_idx
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 64, 64, 33, FAKE, 1 << 20, None) == 2  # K > 32
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 64, 64, 4, FAKE, 16, None) == 3        # ws small
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert call(odd, FAKE, FAKE, 1, 8, 8, 64, 64, 4, FAKE, 1 << 20, None) == 1    # q_idx align


def test_select_invert_host_validation(lib):
    call = lib.msa_select_invert
    assert call(None, FAKE, FAKE, 1, 8, 8, 64, 4, FAKE, 1 << 20, None) == 1
    assert call(FAKE, FAKE, FAKE, 1, 8, 8, 64, 4, FAKE, 8, None) == 3


def test_binding_fails_loudly_without_library(tmp_path):
    from block_sparse_long_05_b200 import msa
    saved = msa._lib
    msa._lib = None
    try:
        with pytest.raises(RuntimeError, match="missing"):
            msa.load_library(str(tmp_path / "libmsa.so"))
    finally:
        msa._lib = saved
