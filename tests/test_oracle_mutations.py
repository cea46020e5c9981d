"""Each plausible mistake planted in a copy of the oracle (on the CPU) must fail at
least one pin.  A mistake is planted at every place the same expression occurs.  This
shows the pins constrain every step the oracle takes: scale, softmax denominator,
column index, head mapping, query indexing, the delta's sign, the pooling window, the
mask, the tie-break (signed zeros included), the budget clamp, the output order and the
compaction source row."""
import os

import pytest

import oracle
from oracle_pins import PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "focus_oracle.c")

MUTATIONS = {
    "scale_dropped": ("s[j] = scale * dot;", "s[j] = dot;"),
    "prefix_left_out_of_denominator": (
        "for (int j = 0; j < N; ++j)\n                    Z += exp",
        "for (int j = L; j < N; ++j)\n                    Z += exp"),
    "prefix_column_read": ("exp(s[L + j] - m) / Z", "exp(s[j] - m) / Z"),
    "head_mapping_modulo": ("for (int h = g * G; h < (g + 1) * G; ++h)",
                            "for (int h = g; h < Hq; h += Hkv)"),
    "query_index_transposed": ("q + (((size_t)r * B + i) * Hq + h) * d",
                               "q + (((size_t)r * Hq + h) * B + i) * d"),
    "delta_sign": ("delta[j] = i1[(size_t)r * B + j] - i0[(size_t)r * B + j];",
                   "delta[j] = i0[(size_t)r * B + j] - i1[(size_t)r * B + j];"),
    "pool_window_asymmetric": ("t <= j + half", "t < j + half"),
    "mask_dropped": ("decoded[(size_t)r * B + j] ? -INFINITY : best", "best"),
    "tie_break_reversed": ("    return a < b;", "    return a > b;"),
    "signed_zeros_ordered": ("    if (va < vb)\n        return 0;\n    return a < b;",
                             "    if (va < vb)\n        return 0;\n    if (signbit(va) != signbit(vb))\n"
                             "        return signbit(vb) != 0;\n    return a < b;"),
    "negative_budget_not_clamped": ("int k = budget[r] < 0 ? 0 : budget[r];", "int k = budget[r];"),
    "output_not_ascending": ("while (t > 0 && chosen[t - 1] > x)", "while (0)"),
    "compact_wrong_source": ("hidden + ((size_t)r * B + j) * H",
                             "hidden + ((size_t)r * B + (row - cu_seqlens[r])) * H"),
    "successor_instead_of_predecessor": ("keep[cand[t] - 1] = 1;", "keep[cand[t] + 1 < B ? cand[t] + 1 : cand[t]] = 1;"),
    "predecessor_only_if_masked": ("                if (cand[t] >= 1)\n                    keep[cand[t] - 1] = 1;",
                                   "                if (cand[t] >= 1 && !decoded[(size_t)r * B + cand[t] - 1])\n                    keep[cand[t] - 1] = 1;"),
    "rightmost_rule_keeps_decoded": ("                if (decoded[(size_t)r * B + j] == 0)\n                    keep[j] = 1;",
                                     "                keep[j] = 1;"),
    "rightmost_rule_uses_leftmost": ("            if (cand[t] > rightmost)", "            if (rightmost < 0 || cand[t] < rightmost)"),
    "lse_sign": ("acc += exp(scale * dot - lse[row]);", "acc += exp(scale * dot + lse[row]);"),
    "lse_wrong_head_index": ("const size_t row = ((size_t)r * B + i) * Hq + h;",
                             "const size_t row = ((size_t)r * B + i) * Hq + g;"),
    "paged_slot_ignored": ("src = k_pages + ((page * page_size + (size_t)(j % page_size)) * Hkv + g) * d;",
                           "src = k_pages + ((page * page_size) * Hkv + g) * d;"),
    "paged_wrong_page": ("page_table[(size_t)r * max_pages + j / page_size]",
                         "page_table[(size_t)r * max_pages + j % page_size]"),
    "budget_threshold_mean_only": ("if (!dec[j] && D[j] > mu + sigma)", "if (!dec[j] && D[j] > mu)"),
    "budget_alpha_dropped": ("double want = ceil(alpha * (decode_avg[r]", "double want = ceil(1.0 * (decode_avg[r]"),
    "budget_sample_std": ("const double sigma = sqrt(ss / m);", "const double sigma = sqrt(ss / (m > 1 ? m - 1 : 1));"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))  # every occurrence: the same slip everywhere
    lib = oracle.build(force=True, src=str(mut), out=str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(lib)
    failed = []
    for pin in PINS:
        try:
            pin(orc)
        except (AssertionError, oracle.OracleError):
            failed.append(pin.__name__)
    assert failed, f"no pin catches mutation {name}"
