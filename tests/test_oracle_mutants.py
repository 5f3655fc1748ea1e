"""Planted mistakes in the oracle, each caught by one of its pins.

Every case copies the oracle package into a scratch folder inside the
repository (`_build/oracle_mutants/`, ignored by git), replaces one line of
the C source with a plausible mistake -- a dropped term or factor, a wrong
sign, swapped counter words, a transposed operand, a wrong constant, a
reversed bit or sort order -- builds that copy, and runs the named pin of
test_oracle_pins.py against it: the pin must fail.  The real oracle is never
touched.  This shows the pins are tight enough that an error of these kinds
anywhere in the oracle's arithmetic would not go unnoticed.

The smallest-index rule of the argmax scan is pinned on planted exact ties
through the oracle's argmax test entry point (perturbed scores of distinct
tokens tie with probability about 2^-32 per pair, so random sampler inputs
cannot show it).  Not covered, on purpose: the choice of counter tag for the
group noise (a reading of the pages, not arithmetic; the grouped GPU parity
tests compare the tag bit for bit).
"""
import importlib.util
import os
import shutil
import sys

import pytest

from tests import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRATCH = os.path.join(ROOT, "_build", "oracle_mutants")

# (name, line of fmms_oracle.c, its mistaken replacement, pin, pin arguments)
MUTANTS = [
    ("counter_row_step_swapped",
     "uint32_t r = oracle_noise_word(key, step, (uint32_t)b, (uint32_t)v, tag);",
     "uint32_t r = oracle_noise_word(key, (uint32_t)b, step, (uint32_t)v, tag);",
     "test_constant_rows_sample_the_noise_argmax", {}),
    ("temperature_dropped",
     "s[v] = l[v] / T + oracle_gumbel_from_u32(r);",
     "s[v] = l[v] + oracle_gumbel_from_u32(r);",
     "test_gumbel_max_matches_softmax", {"T": 0.7}),
    ("noise_scaled_by_temperature",
     "s[v] = l[v] / T + oracle_gumbel_from_u32(r);",
     "s[v] = (l[v] + oracle_gumbel_from_u32(r)) / T;",
     "test_gumbel_max_matches_softmax", {"T": 0.7}),
    ("gumbel_outer_sign",
     "return -log(t);",
     "return log(t);",
     "test_gumbel_high_precision", {}),
    ("uniform_map_off_by_one",
     "double u = ((double)r + 1.0) / denom;",
     "double u = ((double)r + 2.0) / denom;",
     "test_gumbel_high_precision", {}),
    ("upper_branch_wrong_complement",
     "double one_minus_u = (two32 - (double)r) / denom;",
     "double one_minus_u = (two32 - (double)r - 1.0) / denom;",
     "test_gumbel_high_precision", {}),
    ("philox_weyl_constant",
     "#define ORACLE_PHILOX_WEYL_B 0xBB67AE85u",
     "#define ORACLE_PHILOX_WEYL_B 0xBB67AE87u",
     "test_philox_matches_independent_implementation", {}),
    ("philox_multiplicands_swapped",
     "uint64_t pa = (uint64_t)ORACLE_PHILOX_MUL_A * (uint64_t)x0;",
     "uint64_t pa = (uint64_t)ORACLE_PHILOX_MUL_A * (uint64_t)x1;",
     "test_philox_matches_independent_implementation", {}),
    ("philox_nine_rounds",
     "for (int round = 0; round < 10; ++round) {",
     "for (int round = 0; round < 9; ++round) {",
     "test_philox_matches_independent_implementation", {}),
    ("dot_product_last_term_dropped",
     "for (int k = 0; k < d; ++k) acc += bf16_to_double(h[k]) * bf16_to_double(w[k]);",
     "for (int k = 0; k < d - 1; ++k) acc += bf16_to_double(h[k]) * bf16_to_double(w[k]);",
     "test_logits_match_library_matmul", {}),
    ("weight_operand_transposed",
     "for (int k = 0; k < d; ++k) acc += bf16_to_double(h[k]) * bf16_to_double(w[k]);",
     "for (int k = 0; k < d; ++k) acc += bf16_to_double(h[k]) * bf16_to_double(W[(int64_t)k * V + v]);",
     "test_logits_match_library_matmul", {}),
    ("mask_bit_order_reversed",
     "return (int)((mask[(int64_t)b * words + (v >> 5)] >> (v & 31)) & 1u);",
     "return (int)((mask[(int64_t)b * words + (v >> 5)] >> (31 - (v & 31))) & 1u);",
     "test_masked_tokens_never_drawn_and_rest_is_softmax", {}),
    ("group_lse_replaced_by_max",
     "return m + log(acc);",
     "return m;",
     "test_grouped_matches_softmax", {"G": 8}),
    ("group_boundaries_rounded_up",
     "return (int)(((int64_t)g * V) / G);",
     "return (int)(((int64_t)g * V + G - 1) / G);",
     "test_grouped_summary_identities", {"G": 3}),
    ("multi_sample_tags_shared",
     "2u * (uint32_t)k, mask, s);",
     "0u * (uint32_t)k, mask, s);",
     "test_multi_samples_are_softmax_draws", {}),
    ("argmax_ties_toward_the_larger_index",
     "if (arg < 0 || s[v] > b1) {\n      b2 = b1;",
     "if (arg < 0 || s[v] >= b1) {\n      b2 = b1;",
     "test_oracle_argmax_scan_ties_to_the_smallest_index", {}),
    ("argmax_second_best_dropped",
     "} else if (s[v] > b2) {\n      b2 = s[v];\n    }\n  }\n  if (best) *best = b1;",
     "}\n  }\n  if (best) *best = b1;",
     "test_oracle_argmax_scan_ties_to_the_smallest_index", {}),
    ("grouped_within_margin_from_the_wrong_scores",
     "out_margin[2 * i + 1] = (gstar < 0) ? INFINITY : in1 - in2;",
     "out_margin[2 * i + 1] = (gstar < 0) ? INFINITY : in1 - k2;",
     "test_grouped_summary_and_margins_match_the_scores", {"G": 3}),
    ("topk_ties_toward_the_larger_index",
     "return (x->v < y->v) ? -1 : (x->v > y->v);",
     "return (x->v > y->v) ? -1 : (x->v < y->v);",
     "test_topk_all_logits_tied_keeps_the_smallest_indices", {}),
    ("topk_keeps_smallest_logits",
     "if (x->l > y->l) return -1;\n  if (x->l < y->l) return 1;",
     "if (x->l < y->l) return -1;\n  if (x->l > y->l) return 1;",
     "test_topk_matches_truncated_softmax", {}),
]


def load_mutant(name, old, new):
    """Builds and imports a copy of the oracle with `old` replaced by `new`."""
    src_pkg = os.path.join(ROOT, "oracle")
    dst_pkg = os.path.join(SCRATCH, name, "oracle_" + name)
    shutil.rmtree(os.path.join(SCRATCH, name), ignore_errors=True)
    shutil.copytree(src_pkg, dst_pkg, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    c_path = os.path.join(dst_pkg, "fmms_oracle.c")
    with open(c_path) as f:
        text = f.read()
    assert text.count(old) == 1, "the line to change must occur exactly once: %r" % old
    with open(c_path, "w") as f:
        f.write(text.replace(old, new))
    mod_name = "oracle_mutant_" + name
    spec = importlib.util.spec_from_file_location(
        mod_name, os.path.join(dst_pkg, "__init__.py"), submodule_search_locations=[dst_pkg])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[mod_name] = mod
    spec.loader.exec_module(mod)
    mod._load()
    return mod


@pytest.mark.parametrize("name,old,new,pin,kwargs", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new, pin, kwargs):
    mutant = load_mutant(name, old, new)
    try:
        with pytest.raises(AssertionError):
            getattr(pins, pin)(mutant, **kwargs)
    finally:
        sys.modules.pop("oracle_mutant_" + name, None)
        shutil.rmtree(os.path.join(SCRATCH, name), ignore_errors=True)
