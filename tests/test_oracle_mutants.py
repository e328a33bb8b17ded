"""Plausible slips in the oracle are caught by the pins.

Each mutant is a copy of the oracle's C source with one deliberate mistake
(a dropped term, a wrong sign or index, a transposed operand, a flipped
tie-break ...).  It is compiled into a temporary directory on the CPU and the
pin suite must report at least one failure for it (or the mutant must
crash, which a pin run would also expose).  The real oracle source is
never modified.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_routing_oracle.c")

MUTANTS = {
    "bias_sign": ("s[e] = p[e] + (bias ? bias[e] : 0.0);", "s[e] = p[e] - (bias ? bias[e] : 0.0);"),
    "gather_biased": ("weights[i * (int64_t)k + j] = p[admissible[j].index];",
                      "weights[i * (int64_t)k + j] = s[admissible[j].index];"),
    "drop_second_in_top2": ("return best + second;", "return best;"),
    "tie_higher_index": ("if (a->index < b->index) return -1;\n    if (a->index > b->index) return 1;",
                         "if (a->index < b->index) return 1;\n    if (a->index > b->index) return -1;"),
    "sigmoid_sign": ("p[e] = 1.0 / (1.0 + exp(-x[e]));", "p[e] = 1.0 / (1.0 + exp(x[e]));"),
    "skip_best_group": ("for (int t = 0; t < TG; ++t) group_kept", "for (int t = 1; t < TG; ++t) group_kept"),
    "no_renorm": ("if (renorm) w = w / wsum;", "if (0) w = w / wsum;"),
    "scale_divides": ("weights[i * (int64_t)k + j] = w * rsf;", "weights[i * (int64_t)k + j] = w / rsf;"),
    "softmax_sign": ("p[e] = exp(x[e] - mx);", "p[e] = exp(mx - x[e]);"),
    "softmax_unnormalised": ("for (int e = 0; e < E; ++e) p[e] = p[e] / sum;", ";"),
    "interleaved_groups": ("if (group_kept[e / S]) {", "if (group_kept[e % G]) {"),
    "transposed_weight": ("double wv = (w_layout == 0) ? w[(int64_t)c * E + e] : w[(int64_t)e * K + c];",
                          "double wv = (w_layout == 0) ? w[(int64_t)e * K + c] : w[(int64_t)c * E + e];"),
    "ascending_order": ("if (a->value > b->value) return -1;\n    if (a->value < b->value) return 1;",
                        "if (a->value > b->value) return 1;\n    if (a->value < b->value) return -1;"),
    "group_max_is_min": ("if (s[first + j] > m) m = s[first + j];", "if (s[first + j] < m) m = s[first + j];"),
    "perm_unstable": ("for (int64_t i = 0; i < n; ++i) {       /* pairs in ascending index: stable */",
                      "for (int64_t i = n - 1; i >= 0; --i) {       /* reversed: not stable */"),
    "perm_inclusive_offsets": ("for (int e = 0; e < E; ++e) cursor[e] = offsets[e];",
                               "for (int e = 0; e < E; ++e) cursor[e] = offsets[e + 1] - 1;"),
    "perm_scatter_is_gather": ("        scatter[i] = p;\n", "        scatter[p] = (int32_t)i;\n"),
    "shared_weight_times_rsf": ("weights[i * (int64_t)k + (k - 1)] = sum / rsf;",
                                "weights[i * (int64_t)k + (k - 1)] = sum * rsf;"),
    "shared_id_offset": ("ids[i * (int64_t)k + (k - 1)] = E + pick[i];", "ids[i * (int64_t)k + (k - 1)] = pick[i];"),
    "sort_unstable": ("while (b >= 0 && id[b] > ka) {", "while (b >= 0 && id[b] >= ka) {"),
    "softcap_unscaled": ("out[i] = c * tanh(x[i] / c);", "out[i] = tanh(x[i] / c);"),
    "softcap_times_inside": ("out[i] = c * tanh(x[i] / c);", "out[i] = c * tanh(x[i] * c);"),
    "softcap_zero_clears": ("            out[i] = x[i];\n", "            out[i] = 0.0;\n"),
    "router_skips_last_term": ("for (int c = 0; c < K; ++c) {", "for (int c = 0; c < K - 1; ++c) {"),
    "gate_by_sorted_position": ("if (weights && gate) gate[p] = weights[i];",
                                "if (weights && gate) gate[p] = weights[p];"),
    "top2_second_skips_first_slot": ("if (j != best_j && s[first + j] > second) second = s[first + j];",
                                     "if (s[first + j] > second && j != 0) second = s[first + j];"),
    "renorm_epsilon": ("if (renorm) w = w / wsum;", "if (renorm) w = w / (wsum + 1e-9);"),
    "shared_sum_includes_own_slot": ("for (int j = 0; j < k - 1; ++j) sum += weights[i * (int64_t)k + j];",
                                     "for (int j = 0; j < k; ++j) sum += weights[i * (int64_t)k + j];"),
    "perm_counts_high_ids": ("        if (ids[i] >= 0 && ids[i] < E) counts[ids[i]] += 1;",
                             "        if (ids[i] >= 0 && ids[i] <= E) counts[ids[i] < E ? ids[i] : E - 1] += 1;"),
    "philox_no_key_bump": ("            k0 += W0;\n", "            k0 += 0;\n"),
    "philox_words_swapped": ("y0 = hi1 ^ x1 ^ k0, y1 = lo1, y2 = hi0 ^ x3 ^ k1, y3 = lo0;",
                             "y0 = hi0 ^ x1 ^ k0, y1 = lo0, y2 = hi1 ^ x3 ^ k1, y3 = lo1;"),
    "pick_low_bits": ("pick[i] = (int32_t)(uint64_t)(((unsigned __int128)out[0] * (uint64_t)num_shared) >> 64);",
                      "pick[i] = (int32_t)(out[0] % (uint64_t)num_shared);"),
    "pick_no_carry": ("const uint64_t ctr[4] = {c0, c0 < offset ? 1u : 0u, 0, 0};",
                      "const uint64_t ctr[4] = {c0, 0, 0, 0};"),
    "sigmoid_half_slope": ("p[e] = 1.0 / (1.0 + exp(-x[e]));", "p[e] = 1.0 / (1.0 + exp(-0.5 * x[e]));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_src = tmp_path / f"mutant_{name}.c"
    mutant_src.write_text(src.replace(old, new))
    so = oracle.compile_oracle(str(mutant_src), str(tmp_path / f"libmutant_{name}.so"))
    # Run the pins in a child process: a mutant may also crash (an index
    # slip can read out of bounds), which counts as caught.
    code = ("import sys, oracle; from tests import oracle_pins; "
            f"f = oracle_pins.run_all(oracle.load({str(so)!r})); "
            "print(len(f)); sys.exit(0 if f else 3)")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                         timeout=300)
    assert res.returncode != 3, f"mutant {name} passed every pin"
