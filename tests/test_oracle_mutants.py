"""The oracle's pins must catch plausible mistakes.  Each case below compiles
a copy of the oracle's C source with one mistake planted (on the CPU only),
points the oracle wrapper at that build, and checks that at least one pin
from tests/test_oracle_pins.py now fails."""
import os

import pytest

import oracle
import test_oracle_pins as pins

SRC = open(oracle.SRC).read()

# (name, original text, planted mistake, first occurrence only)
MUTANTS = [
    ("means_divide_by_block_size",
     "      means[(int64_t)i * D + d] = s / (double)(t1 - t0);\n    }\n  }\n}\n\n/* Block scores",
     "      means[(int64_t)i * D + d] = s / (double)bs;\n    }\n  }\n}\n\n/* Block scores"),
    ("scores_drop_scale", "    scores[i] = scale * s;", "    scores[i] = s;"),
    ("scores_first_head_only", "      s += dot;", "      if (j == 0) s += dot;"),
    ("select_ties_to_higher_index",
     "  if (sc[ia] < sc[ib]) return 1;\n  return (ia > ib) - (ia < ib);",
     "  if (sc[ia] < sc[ib]) return 1;\n  return (ia < ib) - (ia > ib);"),
    ("select_forgets_current_block", "  sel[1] = nb - 1;", "  sel[1] = cand[k - 2];"),
    ("select_ascending_scores",
     "  if (sc[ia] > sc[ib]) return -1;\n  if (sc[ia] < sc[ib]) return 1;",
     "  if (sc[ia] < sc[ib]) return -1;\n  if (sc[ia] > sc[ib]) return 1;"),
    ("attend_value_transposed",
     "oj[d] += w * kin_oracle_bf16_to_f64(V[(int64_t)t * D + d]);",
     "oj[d] += w * kin_oracle_bf16_to_f64(V[(int64_t)(d % L) * D + (t % D)]);"),
    ("attend_missing_scale", "        z[c] = scale * dot;", "        z[c] = dot;"),
    ("merge_sign_flipped", "      double w = exp(m_parts[s * g + j] - M);", "      double w = exp(M - m_parts[s * g + j]);"),
    ("update_refreshes_last_block_only",
     "  for (int i = L0 / bs; i <= (L - 1) / bs; ++i) {",
     "  for (int i = (L - 1) / bs; i <= (L - 1) / bs; ++i) {"),
]


def _run_pins():
    """The pins, on small fixed parameters; returns the names that failed."""
    checks = [
        ("dense", lambda: pins.test_full_budget_is_dense_attention(4, 16, (83, 130))),
        ("dense_bs32", lambda: pins.test_full_budget_is_dense_attention(1, 32, (64, 31))),
        ("brute_force", lambda: [pins.test_select_maximises_summed_score(t) for t in range(40)]),
        ("all_equal", pins.test_select_all_equal_prefers_low_indices),
        ("topk_property", pins.test_select_large_topk_property),
        ("linearity", lambda: pins.test_scores_equal_group_sum_of_mean_token_logits(150, 16, 5)),
        ("onehot", pins.test_onehot_values_expose_softmax_weights),
        ("hull", pins.test_output_in_convex_hull_and_constant_values),
        ("merge", lambda: pins.test_chunked_merge_equals_single_pass(7)),
        ("update", lambda: pins.test_incremental_update_equals_build_from_scratch(16)),
        ("means", pins.test_means_are_plain_averages),
        ("planted", pins.test_planted_block_is_selected_and_dominates),
    ]
    failed = []
    for name, fn in checks:
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


@pytest.mark.parametrize("name,orig,bad", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, orig, bad, tmp_path):
    assert SRC.count(orig) >= 1, name
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(orig, bad, 1))
    lib = tmp_path / "libmutant.so"
    oracle.build(src=str(src), out=str(lib))
    saved = oracle._lib
    try:
        oracle._lib = oracle.load(str(lib))
        failed = _run_pins()
    finally:
        oracle._lib = saved
    assert failed, f"no pin caught the planted mistake {name}"


def test_unmodified_oracle_passes_the_same_pins():
    assert _run_pins() == []


# The oracle's Python parts (token top-k, paged gather, bf16 rounding): the
# same check, with the mistake planted in a copy of the function's source
# that replaces it for the duration of the test.
PY_MUTANTS = [
    ("token_ties_to_higher_index", "token_topk_attend",
     "np.lexsort((np.arange(L), -z[j]))", "np.lexsort((-np.arange(L), -z[j]))"),
    ("token_keeps_smallest_logits", "token_topk_attend",
     "np.lexsort((np.arange(L), -z[j]))", "np.lexsort((np.arange(L), z[j]))"),
    ("token_drops_scale", "token_topk_attend", "z = scale * (q @ Kf.T)", "z = q @ Kf.T"),
    ("token_kept_set_not_ascending", "token_topk_attend", "s = np.sort(order[:n])", "s = order[:n]"),
    ("token_normalises_over_every_token", "token_topk_attend",
     "/ w.sum())", "/ np.exp(z[j] - m).sum())"),
    ("token_lse_over_every_token", "token_topk_attend",
     "lses.append(m + np.log(w.sum()))", "lses.append(m + np.log(np.exp(z[j] - m).sum()))"),
    ("paged_ignores_the_table", "gather_paged", "pages[int(table_row[i]), h]", "pages[i, h]"),
    ("paged_reads_head_zero", "gather_paged", "pages[int(table_row[i]), h]", "pages[int(table_row[i]), 0]"),
    ("bf16_truncates", "round_bf16", "np.round(m * 256.0)", "np.floor(m * 256.0)"),
    ("bf16_seven_bits", "round_bf16", "np.round(m * 256.0) / 256.0", "np.round(m * 128.0) / 128.0"),
]


def _run_py_pins():
    checks = [
        ("token_dense", pins.test_token_topk_full_budget_is_dense_attention),
        ("token_brute_force", lambda: [pins.test_token_topk_keeps_the_best_set(t) for t in range(20)]),
        ("token_weights", pins.test_token_topk_weights_are_softmax_of_kept_logits_only),
        ("paged", pins.test_gather_paged_follows_the_block_table),
        ("bf16", pins.test_round_bf16_matches_torch_conversion),
    ]
    failed = []
    for name, fn in checks:
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


@pytest.mark.parametrize("name,func,orig,bad", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_python_pins_catch_planted_mistake(name, func, orig, bad, monkeypatch):
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(getattr(oracle, func)))
    assert src.count(orig) == 1, (name, "the original text must occur once")
    ns = dict(vars(oracle))
    exec(compile(src.replace(orig, bad), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setattr(oracle, func, ns[func])
    failed = _run_py_pins()
    assert failed, f"planted mistake {name!r} passed every pin"


def test_unmodified_python_oracle_passes_the_same_pins():
    assert _run_py_pins() == []
