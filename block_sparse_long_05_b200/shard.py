"""Multi-GPU partitions of the MSA hot path (one process per GPU).

Two partitions, both exact: every rank computes a disjoint part of the same
result, and the parts together are the single-GPU result.

* Sequence sharding (decode, batched prefill): rank r takes its own
  sequences.  These are independent problems with no data-path collective
  (weak scaling).

* kv-head sharding of one long prefill.  "MiniMax M3 深度实战" section 2.2
  makes each (KV block, kv head) an independent unit of work, and the index
  branch of "MiniMax M3模型算力成本大幅降低原因深度解析" (索引分支) uses one
  index head shared by every query head.  So rank r holds kv heads
  [hk0, hk1) with their G query heads each, as a tensor-parallel attention
  layer produces them.  The index branch is split by query rows, balanced by
  candidate blocks per row.  The selected ids, T*K*4 bytes, are all-gathered
  (the one exchange step).  Each rank then runs the sparse branch for its
  heads over every query row.  Outputs stay head-sharded (strong scaling).

The functions take the index and attention steps as callables, so the same
partition logic drives the CUDA library (bench.py) and the CPU oracle (the
two-rank gloo test).
"""
from __future__ import annotations

from typing import Callable, List, Tuple

import torch


def head_range(Hkv: int, world: int, rank: int) -> Tuple[int, int]:
    """kv heads [hk0, hk1) of `rank`: contiguous, equal shares."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if Hkv % world != 0:
        raise ValueError(f"{Hkv} kv heads do not split over {world} ranks")
    per = Hkv // world
    return rank * per, (rank + 1) * per


def index_row_ranges(n_q: int, T: int, block: int, world: int,
                     align: int = 128) -> List[Tuple[int, int]]:
    """Split the n_q query rows into `world` contiguous ranges of about equal
    index-branch work.  Row i (position t = T - n_q + i) scores own(t) whole
    candidate blocks.  One more block per row stands for its fixed cost
    (query tile, top-K, ids store).  Boundaries are multiples of `align` rows
    (the index kernel's query tile) except the last.  Ranges may be empty
    when there are fewer tiles than ranks."""
    if world < 1:
        raise ValueError("world must be >= 1")
    t0 = T - n_q
    cost = torch.arange(n_q, dtype=torch.float64).add_(t0).div_(block).floor_().add_(1.0)
    cum = torch.cumsum(cost, 0)
    total = float(cum[-1]) if n_q > 0 else 0.0
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        i = int(torch.searchsorted(cum, torch.tensor([target], dtype=torch.float64))[0]) + 1
        i = min(n_q, max(bounds[-1], (i + align // 2) // align * align))
        bounds.append(i)
    bounds.append(n_q)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def row_slice_args(q_idx: torch.Tensor, k_idx: torch.Tensor, T: int, r0: int, r1: int):
    """The index-branch call for query rows [r0, r1) of one sequence: the
    queries are the last r1 - r0 positions of a context cut at
    T - n_q + r1, so the same entry point serves (its query i sits at
    t = T' - n_q' + i).  Returns (q_idx rows, k_idx prefix, T')."""
    if q_idx.shape[0] != 1:
        raise ValueError("row ranges split one sequence (Bt = 1)")
    n_q = q_idx.shape[1]
    T_cut = T - n_q + r1
    return q_idx[:, r0:r1], k_idx[:, :T_cut], T_cut


def gather_rows(local: torch.Tensor, ranges: List[Tuple[int, int]], group=None) -> torch.Tensor:
    """All-gather the per-rank row blocks [rows_r, ...] into the full
    [sum rows, ...] tensor on every rank (padded to the longest block for
    the collective, then unpadded)."""
    import torch.distributed as dist
    world = len(ranges)
    if world == 1:
        return local
    longest = max(r1 - r0 for r0, r1 in ranges)
    pad = torch.zeros((longest, *local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]].copy_(local)
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([parts[r][:r1 - r0] for r, (r0, r1) in enumerate(ranges)], 0)


def prefill_head_sharded(q_idx: torch.Tensor, k_idx: torch.Tensor, T: int, block: int,
                         world: int, rank: int,
                         index_fn: Callable[[torch.Tensor, torch.Tensor, int], torch.Tensor],
                         attn_fn: Callable[[torch.Tensor], object], group=None):
    """One kv-head-sharded prefill step of one sequence (Bt = 1).

    index_fn(q_idx_rows, k_idx_prefix, T_cut) -> ids [rows, K] for this
    rank's query rows; attn_fn(ids [n_q, K]) -> this rank's attention result
    over all rows (its own heads).  Returns (ids of every row, attn_fn's
    result)."""
    n_q = q_idx.shape[1]
    ranges = index_row_ranges(n_q, T, block, world)
    r0, r1 = ranges[rank]
    qi, ki, T_cut = row_slice_args(q_idx, k_idx, T, r0, r1)
    local = index_fn(qi, ki, T_cut) if r1 > r0 else None
    if local is None:
        K = _k_of(index_fn)
        local = torch.empty((0, K), dtype=torch.int32, device=q_idx.device)
    ids = gather_rows(local.reshape(r1 - r0, -1), ranges, group)
    return ids, attn_fn(ids)


def _k_of(index_fn) -> int:
    k = getattr(index_fn, "K", None)
    if k is None:
        raise ValueError("an empty row range needs index_fn.K (ids per row)")
    return int(k)
