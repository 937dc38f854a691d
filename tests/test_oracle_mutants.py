"""Plant plausible mistakes in copies of the oracle (on the CPU) and check
that the pins reject every one of them."""
import os

import pytest

import pins

# (name, text in the oracle source, replacement, how many occurrences)
MUTANTS = [
    ("mean_pool_instead_of_max", "if (dot > best) best = dot;",
     "best = (best == -INFINITY ? 0.0 : best) + dot / block;", 1),
    ("tie_to_higher_block", "return j_a < j_b;", "return j_a > j_b;", 1),
    ("k_excludes_own_block", "int m = (K < eligible ? K : eligible) - 1;",
     "int m = (K - 1 < own ? K - 1 : own) - (K > 1 && own > 0 ? 1 : 0);", 1),
    ("gqa_head_modulo", "t, T, Hkv, d, h / G, block, uniq", "t, T, Hkv, d, h % Hkv, block, uniq",
     1),
    ("scale_one_over_d", "return dot / sqrt((double)d);", "return dot / (double)d;", 1),
    ("causal_off_by_one", "if (hi > t + 1) hi = t + 1;", "if (hi > t) hi = t;", 3),
    ("lse_drops_max", "double l = mx + log(sum);", "double l = log(sum);", 1),
    ("index_scores_negated", "dot += bf16_bits_to_double(q_idx_row[c]) * bf16_bits_to_double(krow[c]);",
     "dot -= bf16_bits_to_double(q_idx_row[c]) * bf16_bits_to_double(krow[c]);", 1),
    ("combine_weight_sign", "double w = exp(l - L);", "double w = exp(L - l);", 1),
    ("query_position_from_sequence_start", "*t = (int64_t)T - n_q + (r % n_q);",
     "*t = (r % n_q);", 1),
    ("index_max_starts_at_zero", "double best = -INFINITY;", "double best = 0.0;", 1),
    ("own_block_one_late", "int own = (int)(t / block);", "int own = (int)((t + 1) / block);", 2),
    ("own_block_not_forced", "sel[n_sel++] = own;", "(void)own;", 1),
    ("softmax_not_normalised", "double p = exp(x[n++] - l);", "double p = exp(x[n++] - mx);", 1),
    ("combine_lse_drops_max", "double L = mx + log(sum);", "double L = log(sum);", 1),
    ("invert_unsorted", "for (int i = 0; i < n_q; ++i)\n            for (int s = 0; s < K; ++s) {\n                int64_t r",
     "for (int i = n_q - 1; i >= 0; --i)\n            for (int s = 0; s < K; ++s) {\n                int64_t r", 1),
]


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new, count):
    from oracle import oracle
    src = oracle.source_text()
    assert src.count(old) == count, (name, src.count(old))
    mutant = oracle.compile_variant(src.replace(old, new), os.path.join(tmp_path, name + ".so"))
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(mutant)
        except Exception:  # AssertionError, or a crash-free error from the mutant
            failed.append(check.__name__)
    assert failed, f"no pin rejects the planted mistake {name}"
