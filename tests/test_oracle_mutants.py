"""Pin strength: copies of the oracle with one plausible mistake each must fail a pin.

Each mutant is the oracle's C source with one textual change (a dropped term,
a wrong index, a reversed comparison, a swapped operand), compiled to a
temporary library on the CPU.  The clean oracle passes every pin
(test_oracle_pins.py); every mutant must fail at least one."""
import os
import subprocess

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "drop_score_scale": ("s_out[i] = scale * dot;", "s_out[i] = dot;"),
    "gqa_modulo_mapping": ("int32_t g = h / group;\n    const uint16_t *qh = q + (int64_t)h * d;\n    for (int64_t i = 0;",
                           "int32_t g = h % h_kv;\n    const uint16_t *qh = q + (int64_t)h * d;\n    for (int64_t i = 0;"),
    "softmax_no_max_shift": ("    double m = s[0];\n    for (int64_t i = 1; i < n; ++i)\n        if (s[i] > m)\n            m = s[i];\n",
                             "    double m = 0.0;\n"),
    "softmax_sign_flip": ("z += exp(s[i] - m);", "z += exp(m - s[i]);"),
    "vote_first_head_only": ("    for (int32_t h = 0; h < h_q; ++h) {\n        oracle_head_logits(",
                             "    for (int32_t h = 0; h < 1; ++h) {\n        oracle_head_logits("),
    "tie_to_higher_id": ("if (a->i < b->i) return -1;\n    if (a->i > b->i) return 1;",
                         "if (a->i > b->i) return -1;\n    if (a->i < b->i) return 1;"),
    "no_local_window": ("int64_t l0 = n - n_local;", "int64_t l0 = n;"),
    "sink_overlaps_candidates": ("e[j].v = v[s_end + j];\n            e[j].i = s_end + j;",
                                 "e[j].v = v[j];\n            e[j].i = j;"),
    "attn_reads_k_as_v": ("const uint16_t *vj = v + (int64_t)ids[j]", "const uint16_t *vj = k + (int64_t)ids[j]"),
    "attn_drop_scale": ("            s[j] = scale * dot;", "            s[j] = dot;"),
    "channel_shift": ("dot += widen_bf16(qh[c]) * widen_bf16(ki[c]);",
                      "dot += widen_bf16(qh[c]) * widen_bf16(ki[(c + 1) % d]);"),
    "stride_swap": ("const uint16_t *ki = k + i * stride_tok + (int64_t)g * stride_head;",
                    "const uint16_t *ki = k + i * stride_head + (int64_t)g * stride_tok;"),
    "cosine_strict": ("reuse = (c >= theta) ? 1 : 0;", "reuse = (c > theta) ? 1 : 0;"),
    "cosine_no_norm": ("return ab / (sqrt(aa) * sqrt(bb));", "return ab / sqrt(aa * aa);"),
    "qprev_not_updated": ("    memcpy(q_prev, q, (size_t)len * sizeof(uint16_t));\n", "\n"),
    "reuse_windows_of_old_length": ("oracle_windows(n_new, n_sink, n_local, &s_new, &l0_new);",
                                    "oracle_windows(n_old, n_sink, n_local, &s_new, &l0_new);"),
    "reuse_keeps_old_local_window": ("if (id >= s_old && id < l0_old && id >= s_new && id < l0_new)",
                                     "if (id >= s_old && id >= s_new && id < l0_new)"),
    "reuse_drops_topk_part": ("if (id >= s_old && id < l0_old && id >= s_new && id < l0_new)\n            chosen[id] = 1;",
                              "if (id < 0)\n            chosen[id] = 1;"),
    # page-level comparator
    "quest_meta_skips_last_token": ("for (int64_t t = t0 + 1; t < t1; ++t) {", "for (int64_t t = t0 + 1; t < t1 - 1; ++t) {"),
    "quest_meta_page_off_by_one": ("int64_t t1 = t0 + P < n ? t0 + P : n;", "int64_t t1 = t0 + P + 1 < n ? t0 + P + 1 : n;"),
    "quest_bound_takes_smaller_product": ("u += a > b ? a : b;", "u += a < b ? a : b;"),
    "quest_bound_max_key_only": ("u += a > b ? a : b;", "u += b;"),
    "quest_scores_drop_scale": ("total += scale * u;", "total += u;"),
    "quest_scores_gqa_modulo": ("int32_t g = h / group;\n            const uint16_t *qh = q + (int64_t)h * d;\n            const uint16_t *mn",
                                "int32_t g = h % h_kv;\n            const uint16_t *qh = q + (int64_t)h * d;\n            const uint16_t *mn"),
    "quest_scores_max_over_heads": ("            total += scale * u;", "            total = total > scale * u ? total : scale * u;"),
    "quest_budget_rounds_up": ("int64_t kp = k / P;", "int64_t kp = (k + P - 1) / P;"),
    "quest_candidates_ignore_windows": ("        int64_t lo = j * P > s_end ? j * P : s_end;\n        int64_t hi = (j + 1) * P < l_begin ? (j + 1) * P : l_begin;\n        if (lo < hi) {",
                                        "        int64_t lo = j * P;\n        int64_t hi = (j + 1) * P;\n        if (lo < hi) {"),
    "quest_drops_pages_overlapping_the_sink": ("        if (lo < hi) {\n            e[nc].v = score[j];",
                                               "        if (lo < hi && j * P >= s_end) {\n            e[nc].v = score[j];"),
}


@pytest.fixture(scope="module")
def clean_source():
    with open(os.path.join(os.path.dirname(oracle.__file__), "ts_oracle.c")) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, clean_source, tmp_path):
    old, new = MUTANTS[name]
    assert clean_source.count(old) == 1, "mutation site not unique: %s" % name
    src = tmp_path / ("%s.c" % name)
    src.write_text(clean_source.replace(old, new))
    so = tmp_path / ("%s.so" % name)
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(src), "-lm"])
    failed = []
    with oracle.using_library(str(so)):
        for pin in oracle_pins.ALL_PINS:
            if pin is oracle_pins.pin_select_brute_force:
                args = (150,)
            elif pin is oracle_pins.pin_quest_select_brute_force:
                args = (150,)
            else:
                args = ()
            try:
                pin(*args)
            except (AssertionError, ValueError, FloatingPointError):
                failed.append(pin.__name__)
    assert failed, "mutant %s passed every pin" % name
