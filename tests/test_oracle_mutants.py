"""The oracle pins must catch plausible slips in the oracle.

Each case below plants one mistake in a temporary copy of the oracle source
(on the CPU, in a scratch directory), compiles it, and runs the pins that
should reject it.  The committed oracle is never modified.
"""
import os

import pytest

from oracle import oracle as O
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "ksa_oracle.c")

# (name, text to replace, replacement, occurrence to replace, pins that must fail)
MUTANTS = [
    ("mean divides by bs on the tail", "out[d] /= (double)n;", "out[d] /= (double)bs;", 0,
     [lambda o: pins.test_summaries_arithmetic_series(o)]),
    ("mean drops the last token", "t < j * bs + n;", "t < j * bs + n - 1;", 0,
     [lambda o: pins.test_summaries_constant_blocks(o, 16)]),
    ("wrong head->group map in scores", "for (int h = g * G; h < (g + 1) * G; ++h)",
     "for (int h = g; h < Hq; h += Hkv)", 0,
     [pins.test_scores_basis_queries_pick_components]),
    ("ties go to the higher index", "if (best < 0 || s[j] > s[best])",
     "if (best < 0 || s[j] >= s[best])", 0, [pins.test_topk_bruteforce_with_ties]),
    ("softmax scale dropped", "z[i] = scale * acc;", "z[i] = acc;", 0,
     [lambda o: pins.test_dense_attention_equals_sdpa(o, 2, 64, 300)]),
    ("tokens past L kept", "if (t < L) tok[n_tok++]", "if (t < T) tok[n_tok++]", 0,
     [pins.test_block_selection_attention_equals_sdpa_on_gathered]),
    ("wrong kv-head for a query head in attention", "const int g = h / G;",
     "const int g = h % Hkv;", 0,
     [lambda o: pins.test_dense_attention_equals_sdpa(o, 2, 64, 300)]),
    ("lse without the log", "zmax + log(denom)", "zmax + denom", 0,
     [pins.test_golden_attention]),
    ("weights not normalised", "const double w = exp(z[i] - zmax) / denom;",
     "const double w = exp(z[i] - zmax);", 0, [pins.test_attention_convex_hull_and_weights]),
    ("voted part may overlap the window", "const int n_cand = L - R;",
     "const int n_cand = L;", 0, [pins.test_unified_window_excluded_from_voted_part]),
    ("unified ties go to the higher token", "return (x->t > y->t) - (x->t < y->t);",
     "return (x->t < y->t) - (x->t > y->t);", 0, [pins.test_unified_bruteforce_small]),
    ("wrong kv-head for a query head in recall", "const int g = h / G;",
     "const int g = h % Hkv;", 1, [pins.test_recall_is_the_lse_difference]),
    ("recall without the max subtraction", "w[t] = exp(w[t] - zmax);", "w[t] = exp(w[t]);", 0,
     [pins.test_recall_with_huge_logits]),
    ("recall weights not divided by the dense sum", "if (sel[t]) mass += w[t] / denom;",
     "if (sel[t]) mass += w[t];\n      denom = mass;", 0, [pins.test_golden_recall]),
    ("wrong kv-head for a query head in per-head top-k", "const int g = h / G;",
     "const int g = h % Hkv;", 2, [pins.test_tokens_per_head_rank_counting]),
    ("wrong kv-head for a query head in voting", "const int g = h / G;",
     "const int g = h % Hkv;", 3, [pins.test_unified_bruteforce_small]),
    ("recency window shifted by one", "for (int t = L - R; t < L; ++t) pick[n++] = t;",
     "for (int t = L - R - 1; t < L - 1; ++t) pick[n++] = t;", 0,
     [pins.test_unified_closed_forms]),
    ("bf16 ties rounded away from zero",
     "if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;",
     "if (frac >= 0.5) r += 1.0;", 0,
     [lambda o: pins.test_round_bf16_format_values(o, 1.0 + 2.0 ** -8, 0x3F80)]),
    ("bf16 grid one bit too coarse", "int q = e - 8;", "int q = e - 7;", 0,
     [pins.test_round_bf16_matches_torch_on_binary32]),
    ("bf16 subnormal spacing of the normal range", "if (q < -133) q = -133;",
     "if (q < -126) q = -126;", 0,
     [lambda o: pins.test_round_bf16_format_values(o, 2.0 ** -133, 0x0001)]),
    ("bf16 summary storage never applied", "if (summary_fmt == 1) {", "if (0) {", 0,
     [pins.test_select_blocks_bf16_storage_tie]),
    ("e4m3 ties rounded away from zero",
     "if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;\n  double v = ldexp(r, q);",
     "if (frac >= 0.5) r += 1.0;\n  double v = ldexp(r, q);", 0,
     [lambda o: pins.test_round_e4m3_format_values(o, 1.0625, 1.0)]),
    ("e4m3 spacing one bit too fine", "int q = e - 4; /* spacing", "int q = e - 5; /* spacing", 0,
     [pins.test_round_e4m3_matches_torch]),
    ("e4m3 scale one binade too small", "while (amax > ldexp(448.0, e)) ++e;",
     "while (amax > ldexp(448.0, e + 1)) ++e;", 0, [pins.test_e4m3_scale_exponent]),
    ("fp8 summary storage never applied", "  } else if (summary_fmt == 2) {",
     "  } else if (0) {", 0, [pins.test_select_blocks_fp8_storage]),
    ("page row ignores the kv-head",
     "pages + (((size_t)page * Hkv + g) * bs + t % bs) * D;",
     "pages + (((size_t)page * Hkv) * bs + t % bs) * D;", 0,
     [pins.test_gather_pages_identity_table]),
    ("token offset within a page off by one",
     "pages + (((size_t)page * Hkv + g) * bs + t % bs) * D;",
     "pages + (((size_t)page * Hkv + g) * bs + (t + 1) % bs) * D;", 0,
     [pins.test_gather_pages_scatter_roundtrip_and_bad_pages]),
    ("random head: always head 0",
     "memcpy(token_idx + (size_t)b * k, all + ((size_t)b * Hq + h) * k,",
     "memcpy(token_idx + (size_t)b * k, all + ((size_t)b * Hq) * k,", 0,
     [pins.test_one_head_set_is_that_heads_brute_force_topk]),
    ("window one block early", "row[i] = i < n ? nb - n + i : -1;",
     "row[i] = i < n ? nb - n + i - 1 : -1;", 0,
     [pins.test_select_window_is_topk_of_a_recency_score]),
]


def _replace_nth(text, old, new, n):
    start = -1
    for _ in range(n + 1):
        start = text.index(old, start + 1)
    return text[:start] + new + text[start + len(old):]


@pytest.mark.parametrize("name,old,new,nth,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new, nth, catchers):
    src = open(SRC).read()
    assert src.count(old) > nth, f"mutation site vanished: {old!r}"
    mutated = _replace_nth(src, old, new, nth)
    path = tmp_path / "ksa_oracle_mutant.c"
    path.write_text(mutated)
    # a distinct file per mutant, kept until the session ends: the dynamic
    # loader reuses an already-loaded library whose file has the same inode
    so = str(tmp_path / f"libksa_oracle_mutant_{abs(hash(name))}.so")
    O.build(force=True, src=str(path), out=so)
    mutant = O.Oracle(so)
    caught = 0
    for pin in catchers:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin rejected the mutant: {name}"
