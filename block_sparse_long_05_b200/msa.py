"""Python binding of libmsa (the C ABI in include/msa.h), by ctypes.

Argument marshalling only: every step of the MSA hot path runs in the CUDA
kernels behind the C ABI.  torch supplies device memory and the current CUDA
stream.  If libmsa.so is missing, every call raises: there is no CPU path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

STATUS = {
    0: "MSA_OK",
    1: "MSA_ERR_INVALID_ARG",
    2: "MSA_ERR_UNSUPPORTED",
    3: "MSA_ERR_WORKSPACE",
    4: "MSA_ERR_CUDA",
    5: "MSA_ERR_TIMEOUT",
    6: "MSA_ERR_BAD_IDS",
}

EXPORTED = ("msa_workspace_size", "msa_index_topk", "msa_select_invert", "msa_sparse_attn",
            "msa_index_topk_ev", "msa_sparse_attn_ev", "msa_device_status", "msa_status_string",
            "msa_selftest_umma", "msa_sparse_attn_decode_noalloc", "msa_index_topk_paged",
            "msa_sparse_attn_paged", "msa_index_topk_i8", "msa_index_topk_i8_ev",
            "msa_workspace_size_kv_group")

MAX_STAGES = 4


class StageEvents(ctypes.Structure):
    """msa_stage_events: cudaEvent_t handles recorded around each stage."""
    _fields_ = [("start", ctypes.c_void_p * MAX_STAGES), ("stop", ctypes.c_void_p * MAX_STAGES)]


def _event_handle(ev) -> int:
    """Raw cudaEvent_t of a torch.cuda.Event (created on first record)."""
    if ev.cuda_event == 0:
        ev.record()
    return ev.cuda_event


def _stage_events(events):
    """events: {stage: (start torch.cuda.Event, stop torch.cuda.Event)} or None."""
    if not events:
        return None
    se = StageEvents()
    for i, (a, b) in events.items():
        se.start[i] = _event_handle(a) if a is not None else None
        se.stop[i] = _event_handle(b) if b is not None else None
    return ctypes.byref(se)


class MSAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)} ({code})")
        self.code = code


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libmsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m block_sparse_long_05_b200.build` (needs nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.msa_workspace_size.argtypes = [I, I, I, I, I, I, I, I, I]
    lib.msa_workspace_size.restype = Z
    lib.msa_workspace_size_kv_group.argtypes = [I, I, I, I, I, I, I, I, I, I]
    lib.msa_workspace_size_kv_group.restype = Z
    lib.msa_index_topk.argtypes = [P, P, P, I, I, I, I, I, I, P, Z, P]
    lib.msa_index_topk.restype = I
    lib.msa_select_invert.argtypes = [P, P, P, I, I, I, I, I, P, Z, P]
    lib.msa_select_invert.restype = I
    lib.msa_sparse_attn.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]
    lib.msa_sparse_attn.restype = I
    lib.msa_device_status.argtypes = [P, P]
    lib.msa_device_status.restype = I
    lib.msa_status_string.argtypes = [I]
    lib.msa_status_string.restype = ctypes.c_char_p
    lib.msa_index_topk_ev.argtypes = [P, P, P, I, I, I, I, I, I, P, Z, P, P]
    lib.msa_index_topk_ev.restype = I
    lib.msa_index_topk_i8.argtypes = [P, P, P, I, I, I, I, I, I, P, Z, P]
    lib.msa_index_topk_i8.restype = I
    lib.msa_index_topk_i8_ev.argtypes = [P, P, P, I, I, I, I, I, I, P, Z, P, P]
    lib.msa_index_topk_i8_ev.restype = I
    lib.msa_sparse_attn_ev.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P, P]
    lib.msa_sparse_attn_ev.restype = I
    lib.msa_sparse_attn_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P, P]
    lib.msa_sparse_attn_decode_noalloc.restype = I
    lib.msa_index_topk_paged.argtypes = [P, P, P, I, I, P, I, I, I, I, I, P, Z, P]
    lib.msa_index_topk_paged.restype = I
    lib.msa_sparse_attn_paged.argtypes = [P, P, P, P, I, I, P, P, P, I, I, I, I, I, I, I, P, Z, P]
    lib.msa_sparse_attn_paged.restype = I
    lib.msa_selftest_umma.argtypes = [P, P, P, I, I, I, P, P]
    lib.msa_selftest_umma.restype = I
    _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != 0:
        raise MSAError(fn, code)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def workspace_size(Bt, n_q, T, Hq, Hkv, d, d_idx, block, K, kv_group=None) -> int:
    """Workspace bytes: the minimum (msa_workspace_size), or with kv_group
    the size for prefill attention passes of kv_group kv heads each
    (kv_group = Hkv: one pass over all heads)."""
    lib = load_library()
    if kv_group is None:
        return int(lib.msa_workspace_size(Bt, n_q, T, Hq, Hkv, d, d_idx, block, K))
    return int(lib.msa_workspace_size_kv_group(Bt, n_q, T, Hq, Hkv, d, d_idx, block, K, kv_group))


class Workspace:
    """Device scratch for the calls (status word zeroed at creation)."""

    def __init__(self, nbytes: int, device=None):
        if nbytes <= 0:
            raise ValueError("workspace size must be positive (unsupported shape?)")
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + nbytes]
        self.view[:256].zero_()
        self.nbytes = nbytes

    @property
    def ptr(self) -> int:
        return self.view.data_ptr()

    @classmethod
    def for_shape(cls, Bt, n_q, T, Hq, Hkv, d, d_idx, block, K, device=None,
                  kv_group=None) -> "Workspace":
        return cls(workspace_size(Bt, n_q, T, Hq, Hkv, d, d_idx, block, K, kv_group), device)


def index_topk(q_idx: torch.Tensor, k_idx: torch.Tensor, block: int, K: int, ws: Workspace,
               ids: torch.Tensor | None = None, stream=None, events=None) -> torch.Tensor:
    """q_idx [Bt, n_q, d_idx], k_idx [Bt, T, d_idx] bf16 -> ids [Bt, n_q, K] int32.
    events: optional {stage: (start, stop)} torch.cuda.Event pairs (msa_index_topk_ev)."""
    _dev(q_idx, torch.bfloat16, "q_idx")
    _dev(k_idx, torch.bfloat16, "k_idx")
    Bt, n_q, d_idx = q_idx.shape
    T = k_idx.shape[1]
    if k_idx.shape != (Bt, T, d_idx):
        raise ValueError(f"k_idx shape {tuple(k_idx.shape)} does not match q_idx")
    if ids is None:
        ids = torch.empty((Bt, n_q, K), dtype=torch.int32, device=q_idx.device)
    _dev(ids, torch.int32, "ids")
    lib = load_library()
    _check("msa_index_topk", lib.msa_index_topk_ev(q_idx.data_ptr(), k_idx.data_ptr(),
                                                   ids.data_ptr(), Bt, n_q, T, d_idx, block, K,
                                                   ws.ptr, ws.nbytes, _stream(stream),
                                                   _stage_events(events)))
    return ids


def index_topk_i8(q_idx: torch.Tensor, k_idx: torch.Tensor, block: int, K: int, ws: Workspace,
                  ids: torch.Tensor | None = None, stream=None, events=None) -> torch.Tensor:
    """Index branch on signed 8-bit index keys (msa_index_topk_i8):
    q_idx [Bt, n_q, d_idx], k_idx [Bt, T, d_idx] int8 -> ids [Bt, n_q, K] int32,
    the same selection msa_index_topk makes on the same integer values."""
    _dev(q_idx, torch.int8, "q_idx")
    _dev(k_idx, torch.int8, "k_idx")
    Bt, n_q, d_idx = q_idx.shape
    T = k_idx.shape[1]
    if k_idx.shape != (Bt, T, d_idx):
        raise ValueError(f"k_idx shape {tuple(k_idx.shape)} does not match q_idx")
    if ids is None:
        ids = torch.empty((Bt, n_q, K), dtype=torch.int32, device=q_idx.device)
    _dev(ids, torch.int32, "ids")
    lib = load_library()
    _check("msa_index_topk_i8", lib.msa_index_topk_i8_ev(q_idx.data_ptr(), k_idx.data_ptr(),
                                                         ids.data_ptr(), Bt, n_q, T, d_idx, block,
                                                         K, ws.ptr, ws.nbytes, _stream(stream),
                                                         _stage_events(events)))
    return ids


def select_invert(ids: torch.Tensor, T: int, block: int, ws: Workspace, stream=None):
    """ids [Bt, n_q, K] int32 -> (row_ptr [Bt*N+1], entries [Bt*n_q*K]) int32 (CSR)."""
    _dev(ids, torch.int32, "ids")
    Bt, n_q, K = ids.shape
    N = (T + block - 1) // block
    row_ptr = torch.empty(Bt * N + 1, dtype=torch.int32, device=ids.device)
    entries = torch.empty(max(Bt * n_q * K, 1), dtype=torch.int32, device=ids.device)
    lib = load_library()
    _check("msa_select_invert", lib.msa_select_invert(ids.data_ptr(), row_ptr.data_ptr(),
                                                      entries.data_ptr(), Bt, n_q, T, block, K,
                                                      ws.ptr, ws.nbytes, _stream(stream)))
    return row_ptr, entries


def sparse_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, ids: torch.Tensor, block: int,
                ws: Workspace, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                stream=None, events=None):
    """q [Bt, n_q, Hq, d], k/v [Bt, T, Hkv, d] bf16, ids [Bt, n_q, K] int32
    -> (out [Bt, n_q, Hq, d] fp32, lse [Bt, n_q, Hq] fp32).
    events: optional {stage: (start, stop)} torch.cuda.Event pairs (msa_sparse_attn_ev)."""
    _dev(q, torch.bfloat16, "q")
    _dev(k, torch.bfloat16, "k")
    _dev(v, torch.bfloat16, "v")
    _dev(ids, torch.int32, "ids")
    Bt, n_q, Hq, d = q.shape
    T, Hkv = k.shape[1], k.shape[2]
    if k.shape != (Bt, T, Hkv, d) or v.shape != k.shape:
        raise ValueError("k/v shapes do not match q")
    K = ids.shape[-1]
    if ids.shape != (Bt, n_q, K):
        raise ValueError("ids shape does not match q")
    if out is None:
        out = torch.empty((Bt, n_q, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((Bt, n_q, Hq), dtype=torch.float32, device=q.device)
    _dev(out, torch.float32, "out")
    _dev(lse, torch.float32, "lse")
    lib = load_library()
    _check("msa_sparse_attn", lib.msa_sparse_attn_ev(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                     ids.data_ptr(), out.data_ptr(),
                                                     lse.data_ptr(), Bt, n_q, T, Hq, Hkv, d,
                                                     block, K, ws.ptr, ws.nbytes,
                                                     _stream(stream), _stage_events(events)))
    return out, lse


def index_topk_paged(q_idx: torch.Tensor, k_idx_pages: torch.Tensor, page_table: torch.Tensor,
                     T: int, K: int, ws: Workspace, ids: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Decode index branch over paged index keys (msa_index_topk_paged):
    q_idx [Bt, 1, d_idx], k_idx_pages [num_pages, block, d_idx] bf16,
    page_table [Bt, page_stride] int32 -> ids [Bt, 1, K] int32."""
    _dev(q_idx, torch.bfloat16, "q_idx")
    _dev(k_idx_pages, torch.bfloat16, "k_idx_pages")
    _dev(page_table, torch.int32, "page_table")
    Bt, n_q, d_idx = q_idx.shape
    num_pages, block, d2 = k_idx_pages.shape
    if n_q != 1 or d2 != d_idx or page_table.dim() != 2 or page_table.shape[0] != Bt:
        raise ValueError("paged index: q_idx [Bt, 1, d_idx], k_idx_pages [pages, block, d_idx], "
                         "page_table [Bt, stride]")
    if ids is None:
        ids = torch.empty((Bt, 1, K), dtype=torch.int32, device=q_idx.device)
    _dev(ids, torch.int32, "ids")
    _check("msa_index_topk_paged", load_library().msa_index_topk_paged(
        q_idx.data_ptr(), k_idx_pages.data_ptr(), page_table.data_ptr(), page_table.shape[1],
        num_pages, ids.data_ptr(), Bt, T, d_idx, block, K, ws.ptr, ws.nbytes, _stream(stream)))
    return ids


def sparse_attn_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                      page_table: torch.Tensor, T: int, ids: torch.Tensor, ws: Workspace,
                      out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                      stream=None):
    """Decode sparse branch over paged K/V (msa_sparse_attn_paged): q [Bt, 1, Hq, d],
    k_pages/v_pages [num_pages, block, Hkv, d] bf16, page_table [Bt, page_stride]
    int32, ids [Bt, 1, K] -> (out [Bt, 1, Hq, d], lse [Bt, 1, Hq]) fp32."""
    for t, name in ((q, "q"), (k_pages, "k_pages"), (v_pages, "v_pages")):
        _dev(t, torch.bfloat16, name)
    _dev(page_table, torch.int32, "page_table")
    _dev(ids, torch.int32, "ids")
    Bt, n_q, Hq, d = q.shape
    num_pages, block, Hkv, d2 = k_pages.shape
    K = ids.shape[-1]
    if n_q != 1 or d2 != d or v_pages.shape != k_pages.shape or ids.shape != (Bt, 1, K) or \
            page_table.dim() != 2 or page_table.shape[0] != Bt:
        raise ValueError("paged attention: shapes do not match")
    if out is None:
        out = torch.empty((Bt, 1, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((Bt, 1, Hq), dtype=torch.float32, device=q.device)
    _dev(out, torch.float32, "out")
    _dev(lse, torch.float32, "lse")
    _check("msa_sparse_attn_paged", load_library().msa_sparse_attn_paged(
        q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), page_table.data_ptr(),
        page_table.shape[1], num_pages, ids.data_ptr(), out.data_ptr(), lse.data_ptr(), Bt, T, Hq,
        Hkv, d, block, K, ws.ptr, ws.nbytes, _stream(stream)))
    return out, lse


def sparse_attn_decode_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                               ids: torch.Tensor, block: int, out: torch.Tensor | None = None,
                               lse: torch.Tensor | None = None, status: torch.Tensor | None = None,
                               stream=None):
    """Decode attention (n_q = 1) whose scratch is the library's static device
    array (msa_sparse_attn_decode_noalloc): no workspace is passed and the
    library allocates nothing.  q [Bt, 1, Hq, d], k/v [Bt, T, Hkv, d] bf16,
    ids [Bt, 1, K] int32 -> (out [Bt, 1, Hq, d], lse [Bt, 1, Hq]) fp32.
    status: optional int32 CUDA tensor of one element that receives error bits."""
    _dev(q, torch.bfloat16, "q")
    _dev(k, torch.bfloat16, "k")
    _dev(v, torch.bfloat16, "v")
    _dev(ids, torch.int32, "ids")
    Bt, n_q, Hq, d = q.shape
    if n_q != 1:
        raise ValueError("the no-allocation entry point serves decode steps (n_q == 1)")
    T, Hkv = k.shape[1], k.shape[2]
    K = ids.shape[-1]
    if out is None:
        out = torch.empty((Bt, 1, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((Bt, 1, Hq), dtype=torch.float32, device=q.device)
    sp = 0
    if status is not None:
        _dev(status, torch.int32, "status")
        sp = status.data_ptr()
    lib = load_library()
    _check("msa_sparse_attn_decode_noalloc",
           lib.msa_sparse_attn_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                              ids.data_ptr(), out.data_ptr(), lse.data_ptr(), Bt,
                                              T, Hq, Hkv, d, block, K, sp or None,
                                              _stream(stream)))
    return out, lse


def device_status(ws: Workspace, stream=None) -> int:
    """Synchronise the stream, read and clear the workspace's device status."""
    return int(load_library().msa_device_status(ws.ptr, _stream(stream)))


def status_string(code: int) -> str:
    return load_library().msa_status_string(int(code)).decode()


def selftest_umma(A: torch.Tensor, B: torch.Tensor, b_mn_major: bool, a_tmem: bool = False,
                  stream=None):
    """C[128, N] = A[128, Kd] @ B with B as [N, Kd] (K-major) or [Kd, N] (MN-major);
    a_tmem: the MMA reads A from tensor memory."""
    _dev(A, torch.bfloat16, "A")
    _dev(B, torch.bfloat16, "B")
    Kd = A.shape[1]
    N = B.shape[1] if b_mn_major else B.shape[0]
    C = torch.empty((128, N), dtype=torch.float32, device=A.device)
    status = torch.zeros(1, dtype=torch.int32, device=A.device)
    lib = load_library()
    flags = int(b_mn_major) | (2 if a_tmem else 0)
    _check("msa_selftest_umma", lib.msa_selftest_umma(A.data_ptr(), B.data_ptr(), C.data_ptr(), N,
                                                      Kd, flags, status.data_ptr(),
                                                      _stream(stream)))
    return C, status
