"""MiniMax Sparse Attention (MSA) hot path on one B200 (sm_100a).

The work runs in libmsa.so (C ABI: include/msa.h); ``msa`` is its thin
Python binding, ``inputs`` the seeded synthetic workloads, ``build`` the nvcc
build of the library.
"""
from .msa import (MSAError, Workspace, device_status, index_topk, load_library,  # noqa: F401
                  select_invert, selftest_umma, sparse_attn, sparse_attn_decode_noalloc,
                  status_string, workspace_size)
