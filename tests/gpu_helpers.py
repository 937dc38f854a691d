"""Shared helpers of the GPU parity tests (CUDA library vs CPU oracle)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances on the fp32 attention output and lse against the fp64 oracle
# (bf16 inputs, fp32 accumulation): max-abs 2e-2 and mean-abs 2e-3.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def lib_ready():
    from block_sparse_long_05_b200 import build, msa
    build.build()
    return msa.load_library()


def assert_close(got: np.ndarray, exp: np.ndarray, what: str):
    got = np.asarray(got, dtype=np.float64)
    exp = np.asarray(exp, dtype=np.float64)
    assert got.shape == exp.shape, (what, got.shape, exp.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - exp)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e}, mean-abs {mean:.3e}"
    return mx, mean


def host(t: torch.Tensor) -> torch.Tensor:
    return t.detach().to("cpu")


def run_index(w, x, ws):
    from block_sparse_long_05_b200 import msa
    ids = msa.index_topk(x["q_idx"], x["k_idx"], w.block, w.K, ws)
    assert msa.device_status(ws) == 0
    return ids


def run_attn(w, x, ids, ws):
    from block_sparse_long_05_b200 import msa
    out, lse = msa.sparse_attn(x["q"], x["k"], x["v"], ids, w.block, ws)
    assert msa.device_status(ws) == 0
    return out, lse


def rows_of(t: torch.Tensor, rows: torch.Tensor, width: int) -> torch.Tensor:
    """Select flattened query rows of a [Bt, n_q, ...] tensor."""
    flat = t.reshape(-1, *t.shape[2:]) if t.dim() > 2 else t.reshape(-1)
    return flat[rows.to(flat.device)]
