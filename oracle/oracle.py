"""ctypes front end of the plain-C MSA oracle (``msa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path (the
CUDA library and its binding) never imports this module.

Every function takes CPU tensors or numpy arrays.  bf16 tensors are passed as
their raw 16-bit patterns; the C code widens them exactly to double.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (-O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-Wall", "-Wextra", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _bind(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    L = ctypes.c_int64
    lib.oracle_index_topk.argtypes = [P, P, I, I, I, I, I, I, P, L, P]
    lib.oracle_index_scores.argtypes = [P, P, I, I, I, I, I, P, L, P]
    lib.oracle_select_invert.argtypes = [P, I, I, I, I, I, P, P]
    lib.oracle_sparse_attn.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, P, L, P, P]
    lib.oracle_sparse_attn_partials.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, P, L, P, P]
    lib.oracle_lse_combine.argtypes = [P, P, L, I, I, I, P, P]
    lib.oracle_num_threads.restype = I
    lib.oracle_set_num_threads.argtypes = [I]
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def compile_variant(source_text: str, out_path: str):
    """Compile an edited copy of the oracle source and return an Oracle bound
    to it (used by the tests that check the pins reject planted mistakes)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-fopenmp", "-fPIC",
                           "-shared", "-w", "-o", out_path, src, "-lm"])
    return Oracle(_bind(ctypes.CDLL(out_path)))


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16, x.dtype
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy()
                                        .view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16, a.dtype
    return a


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.int32)


def _rows(rows):
    if rows is None:
        return None, 0, None
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.size, r.ctypes.data


def _check(rc: int, name: str):
    if rc != 0:
        raise RuntimeError(f"{name} failed with status {rc}")


class Oracle:
    """The oracle functions bound to one compiled copy of msa_oracle.c."""

    def __init__(self, lib=None):
        self._lib_override = lib

    @property
    def lib(self):
        return self._lib_override if self._lib_override is not None else _load()

    def num_threads(self) -> int:
        return self.lib.oracle_num_threads()

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    def index_topk(self, q_idx, k_idx, Bt, n_q, T, d_idx, block, K, rows=None) -> np.ndarray:
        """Selected block ids [n_rows, K] int32 (ascending, -1 padded)."""
        lib = self.lib
        qa, ka = _bits(q_idx), _bits(k_idx)
        assert qa.size == Bt * n_q * d_idx and ka.size == Bt * T * d_idx
        r, nr, rp = _rows(rows)
        n = nr if r is not None else Bt * n_q
        ids = np.empty((n, K), dtype=np.int32)
        _check(lib.oracle_index_topk(qa.ctypes.data, ka.ctypes.data, Bt, n_q, T, d_idx, block, K,
                                     rp, nr, ids.ctypes.data), "oracle_index_topk")
        return ids

    def index_scores(self, q_idx, k_idx, Bt, n_q, T, d_idx, block, rows=None) -> np.ndarray:
        """s(t, j) for j < own(t), NaN elsewhere: [n_rows, N] float64."""
        lib = self.lib
        qa, ka = _bits(q_idx), _bits(k_idx)
        r, nr, rp = _rows(rows)
        n = nr if r is not None else Bt * n_q
        nb = (T + block - 1) // block
        out = np.empty((n, nb), dtype=np.float64)
        _check(lib.oracle_index_scores(qa.ctypes.data, ka.ctypes.data, Bt, n_q, T, d_idx, block, rp,
                                       nr, out.ctypes.data), "oracle_index_scores")
        return out

    def select_invert(self, ids, Bt, n_q, T, block, K):
        """(row_ptr [Bt*N+1], entries [nnz]) int32, entries = (b*n_q+i)*K + slot."""
        lib = self.lib
        ia = _i32(ids)
        assert ia.size == Bt * n_q * K
        nb = (T + block - 1) // block
        row_ptr = np.empty(Bt * nb + 1, dtype=np.int32)
        entries = np.empty(max(int((ia >= 0).sum()), 1), dtype=np.int32)
        _check(lib.oracle_select_invert(ia.ctypes.data, Bt, n_q, T, block, K, row_ptr.ctypes.data,
                                        entries.ctypes.data), "oracle_select_invert")
        return row_ptr, entries[: int(row_ptr[-1])]

    def sparse_attn(self, q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block, K, rows=None):
        """(out [n_rows, Hq, d], lse [n_rows, Hq]) float64.  ids: [n_rows, K]."""
        lib = self.lib
        qa, ka, va = _bits(q), _bits(k), _bits(v)
        assert qa.size == Bt * n_q * Hq * d and ka.size == Bt * T * Hkv * d and va.size == ka.size
        r, nr, rp = _rows(rows)
        n = nr if r is not None else Bt * n_q
        ia = _i32(ids).reshape(n, K)
        out = np.empty((n, Hq, d), dtype=np.float64)
        lse = np.empty((n, Hq), dtype=np.float64)
        _check(lib.oracle_sparse_attn(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, ia.ctypes.data,
                                      Bt, n_q, T, Hq, Hkv, d, block, K, rp, nr, out.ctypes.data,
                                      lse.ctypes.data), "oracle_sparse_attn")
        return out, lse

    def sparse_attn_partials(self, q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block, K, rows=None):
        """Per-slot partials: (o [n_rows, K, Hq, d], lse [n_rows, K, Hq]) float64."""
        lib = self.lib
        qa, ka, va = _bits(q), _bits(k), _bits(v)
        r, nr, rp = _rows(rows)
        n = nr if r is not None else Bt * n_q
        ia = _i32(ids).reshape(n, K)
        po = np.empty((n, K, Hq, d), dtype=np.float64)
        pl = np.empty((n, K, Hq), dtype=np.float64)
        _check(lib.oracle_sparse_attn_partials(qa.ctypes.data, ka.ctypes.data, va.ctypes.data,
                                               ia.ctypes.data, Bt, n_q, T, Hq, Hkv, d, block, K, rp,
                                               nr, po.ctypes.data, pl.ctypes.data),
               "oracle_sparse_attn_partials")
        return po, pl

    def lse_combine(self, part_out, part_lse):
        """Merge per-slot partials: (out [n, H, d], lse [n, H]) float64."""
        lib = self.lib
        po = np.ascontiguousarray(part_out, dtype=np.float64)
        pl = np.ascontiguousarray(part_lse, dtype=np.float64)
        n, K, H, d = po.shape
        assert pl.shape == (n, K, H)
        out = np.empty((n, H, d), dtype=np.float64)
        lse = np.empty((n, H), dtype=np.float64)
        _check(lib.oracle_lse_combine(po.ctypes.data, pl.ctypes.data, n, K, H, d, out.ctypes.data,
                                      lse.ctypes.data), "oracle_lse_combine")
        return out, lse


_default = Oracle()
num_threads = _default.num_threads
set_num_threads = _default.set_num_threads
index_topk = _default.index_topk
index_scores = _default.index_scores
select_invert = _default.select_invert
sparse_attn = _default.sparse_attn
sparse_attn_partials = _default.sparse_attn_partials
lse_combine = _default.lse_combine
