"""The pins catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), compiles it, and checks that at least one pin
fails on the broken copy.  This shows the pins are sharp enough to catch a
dropped term, a wrong sign or index, a swapped operand, a wrong alignment or
a reversed tie-break.  Every mutant stays memory-safe.
"""
import os
import subprocess

import pytest

import oracle as orc
from tests import oracle_pins as pins

SRC = os.path.join(os.path.dirname(orc.__file__), "msa_oracle.c")

MUTANTS = {
    "tie_break_reversed": ("return (x->id < y->id) ? -1 : (x->id > y->id);",
                           "return (x->id > y->id) ? -1 : (x->id < y->id);"),
    "index_not_causal_in_block": ("for (int64_t j = j0; j < j1 && j <= p; ++j) {",
                                  "for (int64_t j = j0; j < j1; ++j) {"),
    "min_pool_instead_of_max": ("if (dot > best) best = dot;",
                                "if (best == -INFINITY || dot < best) best = dot;"),
    "index_dot_drops_a_term": ("for (int64_t i = 0; i < d_idx; ++i)",
                               "for (int64_t i = 1; i < d_idx; ++i)"),
    "one_block_too_few": ("const int64_t take = (cb < topk - 1) ? cb : topk - 1;",
                          "const int64_t take = (cb < topk - 1) ? cb : topk - 2;"),
    "top_left_alignment": ("return S - T + t;", "return t;"),
    "attention_not_causal": ("j < S && j <= p;", "j < S;"),
    "wrong_default_scale": ("scale = 1.0 / sqrt((double)d);", "scale = 1.0 / (double)d;"),
    "lse_drops_max": ("lse[ri * Hq + h] = m + log(denom);", "lse[ri * Hq + h] = log(denom);"),
    "wrong_group_of_head": ("const int64_t g = h / R;", "const int64_t g = h % Hkv;"),
    "values_read_from_keys": ("o[c] += w * widen(V, dtype,", "o[c] += w * widen(K, dtype,"),
    "bf16_widening_shift": ("<< 16;", "<< 15;"),
    "softmax_sign": ("const double w = exp(s[q] - m);", "const double w = exp(m - s[q]);"),
    "mass_not_head_averaged": ("out[i] = head_sum / (double)R;", "out[i] = head_sum;"),
    "mass_not_causal": ("if (j > p) break;                   /* causal tokens only */",
                        "if (j > S) break;"),
    "mass_wrong_head_of_group": ("const int64_t h = g * R + hh;", "const int64_t h = hh * Hkv + g;"),
    "mass_unscaled_scores": ("head_sum += exp(scale * dot - l);", "head_sum += exp(dot - l);"),
    "hier_one_candidate_too_few": ("const int64_t nc = (cb < kc - 1) ? cb : kc - 1;",
                                   "const int64_t nc = (cb < kc - 2) ? cb : kc - 2;"),
    "hier_coarse_drops_a_term": ("dot += widen(q_idx_rows, dtype, q0 + ii) * mean[ii];",
                                 "dot += (ii == 0) ? 0.0 : widen(q_idx_rows, dtype, q0 + ii) * mean[ii];"),
    "hier_no_fine_rescoring": ("                    cand[c].score = best;\n",
                               "                    (void)best;\n"),
    "paged_offset_in_page": ("const int64_t src = pg * page_size + j % page_size;",
                             "const int64_t src = pg * page_size + (j + 1) % page_size;"),
    "paged_wrong_table_entry": ("block_table[b * max_pages + j / page_size];\n",
                                "block_table[b * max_pages + (j / page_size + 1) % max_pages];\n"),
}
# "current_block_not_forced" needs a two-part edit: candidates include cb and
# the forced append is dropped.
FORCED_EDIT = [
    ("for (int64_t n = 0; n < cb; ++n) {\n                    cand[n].score",
     "for (int64_t n = 0; n <= cb; ++n) {\n                    cand[n].score"),
    ("qsort(cand, (size_t)cb, sizeof(cand_t), cand_better_first);",
     "qsort(cand, (size_t)(cb + 1), sizeof(cand_t), cand_better_first);"),
    ("const int64_t take = (cb < topk - 1) ? cb : topk - 1;",
     "const int64_t take = (cb + 1 < topk) ? cb + 1 : topk;"),
    ("out[take] = (int32_t)cb;\n                for (int64_t i = take + 1;",
     "for (int64_t i = take;"),
]


def _build(tmp_path, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert old in src, f"mutation anchor not found: {old!r}"
        src = src.replace(old, new)
    c = tmp_path / "mutant.c"
    c.write_text(src)
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-std=c11", "-shared", "-fPIC", str(c),
                           "-o", str(so), "-lm"])
    return orc.bind(str(so))


@pytest.mark.parametrize("name", sorted(MUTANTS) + ["current_block_not_forced"])
def test_pins_catch_mutant(name, tmp_path):
    edits = FORCED_EDIT if name == "current_block_not_forced" else [MUTANTS[name]]
    lib = _build(tmp_path, edits)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake '{name}'"
