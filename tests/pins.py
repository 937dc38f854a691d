"""Checks that pin the CPU oracle to facts other than itself.

Each check takes an oracle object (``oracle.oracle`` or a mutated copy) and
raises AssertionError when the oracle disagrees with:
  * the hand-worked examples under tests/golden/ (cited there);
  * brute force written a different way (numpy integer matmul, Python sort);
  * library routines (torch scaled_dot_product_attention in fp64 with the
    library's own GQA mapping, scipy logsumexp);
  * closed forms and invariants of the definition.
The checks are shared by the pin tests and by the tests that plant mistakes
in copies of the oracle.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# small helpers (independent of the oracle)
# --------------------------------------------------------------------------
def bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def rand_case(Bt, n_q, T, Hq, Hkv, d, d_idx, seed, index_values="int3"):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Bt, n_q, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(Bt, T, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(Bt, T, Hkv, d, generator=g).to(torch.bfloat16)
    if index_values == "int3":
        qi = torch.randint(-3, 4, (Bt, n_q, d_idx), generator=g).to(torch.bfloat16)
        ki = torch.randint(-3, 4, (Bt, T, d_idx), generator=g).to(torch.bfloat16)
    else:
        qi = torch.zeros(Bt, n_q, d_idx, dtype=torch.bfloat16)
        ki = torch.zeros(Bt, T, d_idx, dtype=torch.bfloat16)
    return q, k, v, qi, ki


def brute_ids(qi, ki, Bt, n_q, T, block, K):
    """Index branch by brute force: full integer score matrix, then a Python
    sort on (-score, j)."""
    Q = qi.float().numpy().astype(np.int64)
    Kk = ki.float().numpy().astype(np.int64)
    rows = []
    for b in range(Bt):
        S = Q[b] @ Kk[b].T  # [n_q, T], exact integers
        for i in range(n_q):
            t = T - n_q + i
            own = t // block
            cand = []
            for j in range(own):
                seg = S[i, j * block: min((j + 1) * block, t + 1, T)]
                cand.append((-int(seg.max()), j))
            cand.sort()
            m = min(K, own + 1) - 1
            sel = sorted([j for _, j in cand[:m]] + [own])
            rows.append(sel + [-1] * (K - len(sel)))
    return np.array(rows, dtype=np.int32).reshape(Bt * n_q, K)


def sdpa_reference(q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block):
    """Masked softmax attention by torch SDPA in fp64 (GQA by the library's
    enable_gqa), mask = key's block among the row's ids and key <= query."""
    ids = np.asarray(ids).reshape(Bt, n_q, -1)
    mask = torch.zeros(Bt, n_q, T, dtype=torch.bool)
    key_blk = torch.arange(T) // block
    for b in range(Bt):
        for i in range(n_q):
            t = T - n_q + i
            sel = torch.zeros(T, dtype=torch.bool)
            for j in ids[b, i]:
                if j >= 0:
                    sel |= key_blk == int(j)
            sel &= torch.arange(T) <= t
            mask[b, i] = sel
    qd = q.double().permute(0, 2, 1, 3)  # [Bt, Hq, n_q, d]
    kd = k.double().permute(0, 2, 1, 3)
    vd = v.double().permute(0, 2, 1, 3)
    out = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask[:, None], enable_gqa=True)
    # lse by scipy on explicitly expanded logits
    G = Hq // Hkv
    kx = kd.repeat_interleave(G, dim=1)
    logits = (qd @ kx.transpose(-1, -2)).numpy() / math.sqrt(d)
    logits = np.where(mask[:, None].numpy(), logits, -np.inf)
    lse = logsumexp(logits, axis=-1)  # [Bt, Hq, n_q]
    return (out.permute(0, 2, 1, 3).reshape(Bt * n_q, Hq, d).numpy(),
            np.transpose(lse, (0, 2, 1)).reshape(Bt * n_q, Hq))


def _read_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.rstrip("\n") for ln in f if ln.strip() and not ln.startswith("#")]


# --------------------------------------------------------------------------
# checks
# --------------------------------------------------------------------------
def check_index_golden(o):
    lines = _read_golden("index_worked_example.txt")
    kv = {}
    ids_exp = {}
    scores_exp = {}
    for ln in lines:
        tag, rest = ln.split(None, 1)
        if tag in ("k_idx", "q_idx"):
            kv[tag] = [[float(x) for x in p.split(",")] for p in rest.split()]
        elif tag == "scores":
            for item in rest.split():
                tj, s = item.split("=")
                t, j = tj.split(":")
                scores_exp[(int(t), int(j))] = float(s)
        elif tag == "ids":
            kpart, vals = rest.split(None, 1)
            K = int(kpart.split("=")[1])
            ids_exp[K] = np.array([[int(x) for x in p.split(",") if x != ""]
                                   for p in vals.split()], dtype=np.int32)
    T, block, d_idx = 8, 2, 2
    qi = bf16(kv["q_idx"]).reshape(1, T, d_idx)
    ki = bf16(kv["k_idx"]).reshape(1, T, d_idx)
    sc = o.index_scores(qi, ki, 1, T, T, d_idx, block)
    for (t, j), s in scores_exp.items():
        assert sc[t, j] == s, (t, j, sc[t, j], s)
    assert np.isnan(sc[0]).all() and np.isnan(sc[1]).all()
    for K, exp in ids_exp.items():
        got = o.index_topk(qi, ki, 1, T, T, d_idx, block, K)
        assert np.array_equal(got, exp.reshape(T, K)), (K, got, exp)


def check_attention_golden(o):
    lines = _read_golden("attention_closed_form.txt")
    vals = {}
    for ln in lines:
        tag, rest = ln.split(None, 1)
        vals[tag] = rest
    k = bf16([[float(x) for x in p.split(",")] for p in vals["k"].split()]).reshape(1, 2, 1, 4)
    v = bf16([[float(x) for x in p.split(",")] for p in vals["v"].split()]).reshape(1, 2, 1, 4)
    q = bf16([[float(x) for x in p.split(",")] for p in vals["q"].split()]).reshape(1, 2, 1, 4)
    ids = np.array([[0, -1], [0, 1]], dtype=np.int32)
    out, lse = o.sparse_attn(q, k, v, ids, 1, 2, 2, 1, 1, 4, 1, 2)
    for t in (0, 1):
        exp_out = np.array([float(x) for x in vals[f"out{t}"].split()])
        exp_lse = float(vals[f"lse{t}"])
        assert np.allclose(out[t, 0], exp_out, rtol=0, atol=1e-12), (t, out[t, 0], exp_out)
        assert abs(lse[t, 0] - exp_lse) < 1e-12, (t, lse[t, 0], exp_lse)


INDEX_SHAPES = [  # (Bt, n_q, T, block, K, d_idx)
    (1, 7, 7, 4, 2, 3),
    (2, 64, 64, 8, 3, 8),
    (1, 100, 100, 16, 4, 5),      # ragged tail
    (2, 5, 77, 8, 3, 4),          # last queries of a longer context
    (3, 1, 129, 16, 5, 8),        # decode shape
    (1, 40, 40, 4, 1, 2),         # own block only
    (1, 33, 33, 8, 9, 4),         # K above the number of blocks: dense
]


def check_index_bruteforce(o):
    for n, (Bt, n_q, T, block, K, d_idx) in enumerate(INDEX_SHAPES):
        _, _, _, qi, ki = rand_case(Bt, n_q, T, 1, 1, 1, d_idx, seed=100 + n)
        got = o.index_topk(qi, ki, Bt, n_q, T, d_idx, block, K)
        exp = brute_ids(qi, ki, Bt, n_q, T, block, K)
        assert np.array_equal(got, exp), (Bt, n_q, T, block, K, d_idx)
        # sampled rows give the same answer as the full run
        rows = np.array(sorted({0, Bt * n_q - 1, (Bt * n_q) // 2}), dtype=np.int64)
        got_r = o.index_topk(qi, ki, Bt, n_q, T, d_idx, block, K, rows=rows)
        assert np.array_equal(got_r, exp[rows])


def check_index_scores_bruteforce(o):
    """s(t, j) equals the maximum of the exact integer dot products over the
    keys of block j (NaN for j >= own(t)), including blocks whose products
    are all negative."""
    cases = [(Bt, n_q, T, block, d_idx, 200 + n, None)
             for n, (Bt, n_q, T, block, _, d_idx) in enumerate(INDEX_SHAPES)]
    cases.append((1, 20, 20, 4, 3, 0, "negative"))  # every product is -3
    for Bt, n_q, T, block, d_idx, seed, kind in cases:
        if kind == "negative":
            qi = bf16(np.ones((Bt, n_q, d_idx)))
            ki = bf16(-np.ones((Bt, T, d_idx)))
        else:
            _, _, _, qi, ki = rand_case(Bt, n_q, T, 1, 1, 1, d_idx, seed=seed)
        sc = o.index_scores(qi, ki, Bt, n_q, T, d_idx, block)
        Q = qi.float().numpy().astype(np.int64)
        Kk = ki.float().numpy().astype(np.int64)
        for b in range(Bt):
            S = Q[b] @ Kk[b].T
            for i in range(n_q):
                t = T - n_q + i
                own = t // block
                row = sc[b * n_q + i]
                for j in range((T + block - 1) // block):
                    if j < own:
                        assert row[j] == S[i, j * block:(j + 1) * block].max(), (b, i, j)
                    else:
                        assert np.isnan(row[j]), (b, i, j)


def check_index_invariants(o):
    Bt, n_q, T, block, K, d_idx = 2, 200, 200, 8, 5, 6
    _, _, _, qi, ki = rand_case(Bt, n_q, T, 1, 1, 1, d_idx, seed=7)
    ids = o.index_topk(qi, ki, Bt, n_q, T, d_idx, block, K)
    sc = o.index_scores(qi, ki, Bt, n_q, T, d_idx, block)
    for r in range(Bt * n_q):
        t = T - n_q + r % n_q
        own = t // block
        sel = [int(j) for j in ids[r] if j >= 0]
        assert own in sel
        assert len(sel) == min(K, own + 1)
        assert sel == sorted(set(sel))
        assert all(j == -1 for j in ids[r][len(sel):])
        chosen = [j for j in sel if j != own]
        rest = [j for j in range(own) if j not in chosen]
        for a in chosen:
            for c in rest:
                assert sc[r, a] > sc[r, c] or (sc[r, a] == sc[r, c] and a < c), (r, a, c)


def check_index_ties(o):
    # all-zero index keys: every score is 0, so the lowest blocks win
    Bt, n_q, T, block, K, d_idx = 1, 90, 90, 8, 4, 4
    _, _, _, qi, ki = rand_case(Bt, n_q, T, 1, 1, 1, d_idx, seed=3, index_values="zeros")
    ids = o.index_topk(qi, ki, Bt, n_q, T, d_idx, block, K)
    for t in range(T):
        own = t // block
        m = min(K, own + 1) - 1
        exp = sorted(list(range(m)) + [own])
        exp += [-1] * (K - len(exp))
        assert list(ids[t]) == exp, (t, ids[t], exp)
    # K = 1: only the own block
    ids1 = o.index_topk(qi, ki, Bt, n_q, T, d_idx, block, 1)
    assert np.array_equal(ids1[:, 0], np.arange(T) // block)


ATTN_SHAPES = [  # (Bt, n_q, T, Hq, Hkv, d, block, K)
    (1, 40, 40, 4, 2, 8, 8, 2),
    (2, 37, 37, 6, 3, 4, 4, 3),   # ragged tail, G = 2
    (1, 6, 50, 8, 2, 16, 8, 3),   # last queries only, G = 4
    (2, 1, 70, 4, 1, 8, 16, 2),   # decode, G = 4
]


def check_attention_sdpa_sparse(o):
    for n, (Bt, n_q, T, Hq, Hkv, d, block, K) in enumerate(ATTN_SHAPES):
        q, k, v, qi, ki = rand_case(Bt, n_q, T, Hq, Hkv, d, 8, seed=200 + n)
        ids = o.index_topk(qi, ki, Bt, n_q, T, 8, block, K)
        out, lse = o.sparse_attn(q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block, K)
        ref_out, ref_lse = sdpa_reference(q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block)
        assert np.allclose(out, ref_out, rtol=0, atol=1e-10), np.abs(out - ref_out).max()
        assert np.allclose(lse, ref_lse, rtol=0, atol=1e-10), np.abs(lse - ref_lse).max()


def check_attention_dense_limit(o):
    # K >= number of blocks: every eligible block is selected, which is dense
    # causal attention (torch SDPA is_causal, fp64, library GQA).
    Bt, T, Hq, Hkv, d, block = 2, 45, 4, 2, 8, 8
    K = (T + block - 1) // block
    q, k, v, qi, ki = rand_case(Bt, T, T, Hq, Hkv, d, 4, seed=11)
    ids = o.index_topk(qi, ki, Bt, T, T, 4, block, K)
    out, _ = o.sparse_attn(q, k, v, ids, Bt, T, T, Hq, Hkv, d, block, K)
    ref = F.scaled_dot_product_attention(q.double().permute(0, 2, 1, 3),
                                         k.double().permute(0, 2, 1, 3),
                                         v.double().permute(0, 2, 1, 3),
                                         is_causal=True, enable_gqa=True)
    ref = ref.permute(0, 2, 1, 3).reshape(Bt * T, Hq, d).numpy()
    assert np.allclose(out, ref, rtol=0, atol=1e-10), np.abs(out - ref).max()


def check_attention_special_cases(o):
    Bt, n_q, T, Hq, Hkv, d, block, K = 1, 24, 24, 4, 2, 8, 4, 3
    q, k, v, qi, ki = rand_case(Bt, n_q, T, Hq, Hkv, d, 4, seed=5)
    ids = o.index_topk(qi, ki, Bt, n_q, T, 4, block, K)
    # V == 1 gives out == 1
    ones = torch.ones_like(v)
    out1, _ = o.sparse_attn(q, k, ones, ids, Bt, n_q, T, Hq, Hkv, d, block, K)
    assert np.allclose(out1, 1.0, rtol=0, atol=1e-12)
    # K = 1 and t at the start of its block: the only key is t itself
    ids1 = o.index_topk(qi, ki, Bt, n_q, T, 4, block, 1)
    out, lse = o.sparse_attn(q, k, v, ids1, Bt, n_q, T, Hq, Hkv, d, block, 1)
    G = Hq // Hkv
    for t in range(0, T, block):
        for h in range(Hq):
            assert np.allclose(out[t, h], v[0, t, h // G].double().numpy(), atol=1e-12)
            exp_lse = float((q[0, t, h].double() @ k[0, t, h // G].double()) / math.sqrt(d))
            assert abs(lse[t, h] - exp_lse) < 1e-12


def check_partials_combine(o):
    # merging the per-slot partials equals the direct result (associativity)
    Bt, n_q, T, Hq, Hkv, d, block, K = 1, 30, 30, 4, 2, 8, 4, 3
    q, k, v, qi, ki = rand_case(Bt, n_q, T, Hq, Hkv, d, 4, seed=9)
    ids = o.index_topk(qi, ki, Bt, n_q, T, 4, block, K)
    out, lse = o.sparse_attn(q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block, K)
    po, pl = o.sparse_attn_partials(q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block, K)
    # a padded slot yields an empty partial
    pad = ids == -1
    assert np.all(np.isneginf(pl[pad])) and np.all(~np.isneginf(pl[~pad]))
    co, cl = o.lse_combine(po, pl)
    assert np.allclose(co, out, rtol=0, atol=1e-12)
    assert np.allclose(cl, lse, rtol=0, atol=1e-12)
    # each single-slot partial is itself the SDPA result for that block alone
    for s in range(K):
        one = np.where(np.arange(K)[None, :] == s, ids, -1)
        ok = ids[:, s] >= 0
        ro, rl = sdpa_reference(q, k, v, one, Bt, n_q, T, Hq, Hkv, d, block)
        assert np.allclose(po[ok, s], ro[ok], rtol=0, atol=1e-10)
        assert np.allclose(pl[ok, s], rl[ok], rtol=0, atol=1e-10)


def check_decode_position(o):
    # a decode query is the newest position: same answer as the last prefill row
    Bt, T, Hq, Hkv, d, block, K, d_idx = 2, 50, 4, 2, 8, 8, 3, 4
    q, k, v, qi, ki = rand_case(Bt, T, T, Hq, Hkv, d, d_idx, seed=13)
    ids_p = o.index_topk(qi, ki, Bt, T, T, d_idx, block, K).reshape(Bt, T, K)
    ids_d = o.index_topk(qi[:, -1:].contiguous(), ki, Bt, 1, T, d_idx, block, K)
    assert np.array_equal(ids_d, ids_p[:, -1])
    out_p, lse_p = o.sparse_attn(q, k, v, ids_p.reshape(-1, K), Bt, T, T, Hq, Hkv, d, block, K)
    out_d, lse_d = o.sparse_attn(q[:, -1:].contiguous(), k, v, ids_d, Bt, 1, T, Hq, Hkv, d,
                                 block, K)
    assert np.array_equal(out_d, out_p.reshape(Bt, T, Hq, d)[:, -1])
    assert np.array_equal(lse_d, lse_p.reshape(Bt, T, Hq)[:, -1])


def check_invert(o):
    Bt, n_q, T, block, K = 2, 60, 60, 8, 3
    _, _, _, qi, ki = rand_case(Bt, n_q, T, 1, 1, 1, 4, seed=17)
    ids = o.index_topk(qi, ki, Bt, n_q, T, 4, block, K)
    row_ptr, entries = o.select_invert(ids, Bt, n_q, T, block, K)
    N = (T + block - 1) // block
    lists = {(b, j): [] for b in range(Bt) for j in range(N)}
    for r in range(Bt * n_q):
        for s in range(K):
            j = int(ids[r, s])
            if j >= 0:
                lists[(r // n_q, j)].append(r * K + s)
    exp_ptr = [0]
    exp_entries = []
    for b in range(Bt):
        for j in range(N):
            exp_entries += lists[(b, j)]
            exp_ptr.append(len(exp_entries))
    assert np.array_equal(row_ptr, np.array(exp_ptr, dtype=np.int32))
    assert np.array_equal(entries, np.array(exp_entries, dtype=np.int32))


ALL_CHECKS = [
    check_index_golden,
    check_attention_golden,
    check_index_bruteforce,
    check_index_scores_bruteforce,
    check_index_invariants,
    check_index_ties,
    check_attention_sdpa_sparse,
    check_attention_dense_limit,
    check_attention_special_cases,
    check_partials_combine,
    check_decode_position,
    check_invert,
]
