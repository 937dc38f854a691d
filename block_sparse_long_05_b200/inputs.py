"""Seeded synthetic inputs for the MSA hot path.

This module holds the workload shapes and the random-number recipe only; it
contains none of the method's arithmetic.  The tests feed its tensors both to
the CUDA library and to the CPU oracle, and the benchmark times the library
on them.

Recipe (one torch generator per call, seeded, drawn in the order
q, k, v, q_idx, k_idx):
  * q, k, v  ~ N(0, 1) drawn in fp32, rounded to bf16 (round to nearest even);
  * q_idx, k_idx: integers uniform over {-3, ..., 3}, stored as bf16 (exact).
Shapes (row-major, contiguous):
  q [Bt, n_q, Hq, d], k and v [Bt, T, Hkv, d], q_idx [Bt, n_q, d_idx],
  k_idx [Bt, T, d_idx].  The n_q queries are the last n_q positions of each
  length-T context (prefill: n_q = T; decode: n_q = 1).
Large tensors are drawn in fixed-size chunks so that the temporary fp32
buffer stays small; the chunking is part of the recipe (same seed and device
give the same bytes).
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import torch

_CHUNK = 1 << 26  # elements per fp32 draw


@dataclass(frozen=True)
class Workload:
    name: str
    Bt: int
    n_q: int
    T: int
    Hq: int
    Hkv: int
    d: int
    block: int
    K: int
    d_idx: int
    seed: int = 0

    @property
    def n_blocks(self) -> int:
        return (self.T + self.block - 1) // self.block

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def is_decode(self) -> bool:
        return self.n_q == 1

    def as_dict(self) -> dict:
        return asdict(self)


# The five workloads of the hot path (sizes as the pages' setting fixes them).
TINY_PREFILL = Workload("tiny_prefill_T4096", 1, 4096, 4096, 8, 2, 64, 64, 8, 64)
PREFILL_64K = Workload("prefill_T65536", 1, 65536, 65536, 32, 8, 128, 128, 16, 128)
DECODE_128K = Workload("decode_32x131072", 32, 1, 131072, 64, 8, 128, 128, 16, 128)
PREFILL_256K = Workload("long_prefill_T262144", 1, 262144, 262144, 64, 8, 128, 512, 8, 128)
DECODE_1M = Workload("decode_4x1048576", 4, 1, 1048576, 64, 8, 128, 512, 8, 128)

# Smaller cases with the same head layout, for profiler captures (inputs still
# larger than the 126 MB L2, a few GB on the device in total).
PROFILE_PREFILL = Workload("profile_prefill_T16384", 1, 16384, 16384, 32, 8, 128, 128, 16, 128)
PROFILE_LONG_PREFILL = Workload("profile_long_prefill_T32768", 1, 32768, 32768, 64, 8, 128, 512,
                                8, 128)
PROFILE_DECODE = Workload("profile_decode_4x131072", 4, 1, 131072, 64, 8, 128, 512, 8, 128)

WORKLOADS = {w.name: w for w in (TINY_PREFILL, PREFILL_64K, DECODE_128K, PREFILL_256K, DECODE_1M,
                                 PROFILE_PREFILL, PROFILE_LONG_PREFILL, PROFILE_DECODE)}


def _fill_normal(out: torch.Tensor, gen: torch.Generator) -> None:
    flat = out.view(-1)
    for s in range(0, flat.numel(), _CHUNK):
        n = min(_CHUNK, flat.numel() - s)
        flat[s:s + n].copy_(torch.randn(n, generator=gen, device=out.device,
                                        dtype=torch.float32))


def _fill_small_ints(out: torch.Tensor, gen: torch.Generator) -> None:
    flat = out.view(-1)
    for s in range(0, flat.numel(), _CHUNK):
        n = min(_CHUNK, flat.numel() - s)
        flat[s:s + n].copy_(torch.randint(-3, 4, (n,), generator=gen, device=out.device,
                                          dtype=torch.int32))


def make_inputs(w: Workload, device="cpu", seed: int | None = None,
                index_values: str = "int3") -> dict:
    """Draw q, k, v, q_idx, k_idx for workload ``w`` on ``device``.

    index_values: "int3" (integers in [-3, 3], the workloads' setting),
    "zeros" (all-zero index keys: every score ties) or "normal" (N(0,1)
    rounded to bf16; exactness of the index scores is then not guaranteed).
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed if seed is None else seed)
    bf = torch.bfloat16
    q = torch.empty((w.Bt, w.n_q, w.Hq, w.d), dtype=bf, device=dev)
    k = torch.empty((w.Bt, w.T, w.Hkv, w.d), dtype=bf, device=dev)
    v = torch.empty((w.Bt, w.T, w.Hkv, w.d), dtype=bf, device=dev)
    q_idx = torch.empty((w.Bt, w.n_q, w.d_idx), dtype=bf, device=dev)
    k_idx = torch.empty((w.Bt, w.T, w.d_idx), dtype=bf, device=dev)
    _fill_normal(q, gen)
    _fill_normal(k, gen)
    _fill_normal(v, gen)
    if index_values == "int3":
        _fill_small_ints(q_idx, gen)
        _fill_small_ints(k_idx, gen)
    elif index_values == "zeros":
        q_idx.zero_()
        k_idx.zero_()
    elif index_values == "normal":
        _fill_normal(q_idx, gen)
        _fill_normal(k_idx, gen)
    else:
        raise ValueError(index_values)
    return {"q": q, "k": k, "v": v, "q_idx": q_idx, "k_idx": k_idx}


def sample_rows(w: Workload, n: int, seed: int = 1) -> torch.Tensor:
    """Flattened query rows (b * n_q + i) for sampled checks at full size.

    n rows drawn uniformly without replacement (generator seed ``seed``),
    always including each sequence's first and last query and, for every
    sequence, one query whose own block index is below K (the regime where
    every eligible block is selected).  Returned sorted, int64, on CPU.
    """
    total = w.Bt * w.n_q
    if n >= total:
        return torch.arange(total, dtype=torch.int64)
    gen = torch.Generator().manual_seed(seed)
    picked = set(torch.randperm(total, generator=gen)[:n].tolist())
    for b in range(w.Bt):
        base = b * w.n_q
        picked.add(base)
        picked.add(base + w.n_q - 1)
        t0 = w.T - w.n_q  # position of query 0
        t_early = min(w.T - 1, (w.K - 1) * w.block)  # own block = K - 1 (< K) when it exists
        if t_early >= t0:
            picked.add(base + (t_early - t0))
    return torch.tensor(sorted(picked), dtype=torch.int64)


def random_selection(w: Workload, device="cpu", seed: int = 2) -> torch.Tensor:
    """A synthetic selection with the structure of the index branch's output
    (own block always present, min(K, own+1) distinct blocks <= own, ascending,
    -1 padded) but drawn at random: used to test the sparse branch apart from
    the index branch.  Returns ids [Bt, n_q, K] int32 on ``device``."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    rows = w.Bt * w.n_q
    ids = torch.full((rows, w.K), -1, dtype=torch.int32, device=dev)
    t = (w.T - w.n_q) + torch.arange(rows, device=dev) % w.n_q
    own = torch.div(t, w.block, rounding_mode="floor")
    step = max(1, (1 << 24) // max(w.n_blocks, 1))
    for s in range(0, rows, step):
        e = min(rows, s + step)
        o = own[s:e]
        r = torch.rand((e - s, w.n_blocks), generator=gen, device=dev)
        cols = torch.arange(w.n_blocks, device=dev)[None, :]
        r = torch.where(cols < o[:, None], r, torch.full_like(r, -1.0))  # candidates j < own
        kk = min(w.K - 1, w.n_blocks)
        if kk > 0:
            val, idx = torch.topk(r, kk, dim=1)
            idx = torch.where(val >= 0, idx, torch.full_like(idx, -1))
        else:
            idx = torch.empty((e - s, 0), dtype=torch.int64, device=dev)
        sel = torch.cat([idx, o[:, None]], dim=1)
        big = torch.iinfo(torch.int64).max
        sel = torch.where(sel < 0, torch.full_like(sel, big), sel)
        sel, _ = torch.sort(sel, dim=1)
        sel = torch.where(sel == big, torch.full_like(sel, -1), sel)
        ids[s:e, :sel.shape[1]] = sel[:, :w.K].to(torch.int32)
    return ids.view(w.Bt, w.n_q, w.K)
