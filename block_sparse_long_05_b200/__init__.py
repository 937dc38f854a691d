"""MiniMax Sparse Attention (MSA) hot path on one B200 (sm_100a).

The work runs in libmsa.so (C ABI: include/msa.h); ``msa`` is its thin
Python binding, ``inputs`` the seeded synthetic workloads, ``build`` the nvcc
build of the library.
"""
from .msa import (MSAError, Workspace, device_status, index_topk, index_topk_i8,  # noqa: F401
                  index_topk_paged, load_library, select_invert, selftest_umma, sparse_attn,
                  sparse_attn_decode_noalloc, sparse_attn_paged, status_string, workspace_size)
