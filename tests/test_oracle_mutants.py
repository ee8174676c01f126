"""Planted mistakes in the oracle, on the CPU.  Each mutant is oracle/lsa_oracle.c with one
plausible slip (a wrong divisor, an off-by-one, a flipped comparison, a dropped term, a
quantifier over one row instead of all); it is compiled with gcc into the git-ignored
_build/mutants/ folder, swapped in for the real library, and the named pin must fail on
it.  This shows that the pins in test_oracle_pins.py tie the oracle to something other
than itself closely enough to catch such a slip.  CPU only."""
import ctypes
import functools
import os
import subprocess

import pytest
import torch

import oracle
from tests import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lsa_oracle.c")
OUT = os.path.join(ROOT, "_build", "mutants")

# (name, text in lsa_oracle.c, replacement, pin that must fail)
MUTANTS = [
    ("partial block averaged over 64 tokens",
     "for (int d = 0; d < D; ++d) out[d] /= n;",
     "for (int d = 0; d < D; ++d) out[d] /= (double)blk;",
     pins.test_summary_partial_block_closed_form),
    ("group score without the softmax scale",
     "*s = scale * acc;", "*s = acc;",
     pins.test_score_sign_and_scale),
    ("ties to the higher block index",
     "return (a->j < b->j) ? -1 : (a->j > b->j);",
     "return (a->j > b->j) ? -1 : (a->j < b->j);",
     pins.test_select_ties_go_to_lower_index_and_small_nb_takes_all),
    ("log-sum-exp without the max",
     "  *lse = m + log(l);\n}", "  *lse = log(l);\n}",
     pins.test_losa_step_all_blocks_equals_dense_attention_over_prefix_and_block),
    ("decode keeps tokens past the sequence end",
     "for (int t = j * blk; t < j * blk + blk && t < T; ++t) toks[ntok++] = t;",
     "for (int t = j * blk; t < j * blk + blk; ++t) toks[ntok++] = t;",
     pins.test_decode_subset_equals_masked_dense_and_ignores_tail),
    ("stable tokens join the union",
     "if (!active[(size_t)b * Tq + i]) {", "if (0) {",
     pins.test_blockquery_union_is_union_of_token_selections),
    ("prefill mask lets no token see itself",
     "if (t <= i && t < L) {", "if (t < i && t < L) {",
     functools.partial(pins.test_blasst_lambda_zero_is_dense_causal, L=200)),
    ("query change divided by D only",
     "sum / ((double)Hq * (double)D)", "sum / (double)D",
     pins.test_losa_classify_single_element_change),
    ("activity threshold not strict",
     "on = mi > tau;", "on = mi >= tau;",
     pins.test_losa_classify_constant_shift_closed_form),
    ("merge weights swapped",
     "wp * o_pre[row * D + d] + wi * o_in[d]", "wi * o_pre[row * D + d] + wp * o_in[d]",
     pins.test_losa_step_all_blocks_equals_dense_attention_over_prefix_and_block),
    ("decode skip decided by the first head only",
     "for (int hh = 0; hh < G; ++hh) {\n          double gi;",
     "for (int hh = 0; hh < 1; ++hh) {\n          double gi;",
     pins.test_decode_blasst_skips_only_blocks_every_head_finds_negligible),
    ("prefill skip decided by the first row only",
     "for (int ii = 0; ii < nrows; ++ii) {\n        double gi;",
     "for (int ii = 0; ii < 1; ++ii) {\n        double gi;",
     pins.test_blasst_skip_needs_every_row_negligible),
    ("compressed token divided by the full block length",
     "for (int d = 0; d < D; ++d) o[d] /= (double)(t1 - t0);",
     "for (int d = 0; d < D; ++d) o[d] /= (double)len;",
     pins.test_nsa_compress_is_avg_pool_with_clipped_tail),
    ("window one token short",
     "const int t0 = T - w > 0 ? T - w : 0;", "const int t0 = T - w + 1 > 0 ? T - w + 1 : 0;",
     pins.test_nsa_window_and_compressed_branches_are_sdpa),
    ("weighted score ignores the weights",
     "dot += w[d] * elem(q, dtype, qrow + d) * kb[d];", "dot += elem(q, dtype, qrow + d) * kb[d];",
     pins.test_fasa_weights_score_with_the_kept_chunks_only),
    ("local forced blocks shifted by one",
     "for (int j = NB - n_local; j < NB; ++j)", "for (int j = NB - n_local - 1; j < NB - 1; ++j)",
     functools.partial(pins.test_select_matches_brute_force, NB=10, k=4, ns=1, nl=2)),
    ("decode reads the query of another head",
     "const size_t qrow = ((size_t)b * Hq + h) * D;\n        attend_row(q, k, v, dtype, qrow, kvbase",
     "const size_t qrow = ((size_t)b * Hq + hh * Hkv + g) * D;\n        attend_row(q, k, v, dtype, qrow, kvbase",
     functools.partial(pins.test_decode_with_all_blocks_equals_dense, dtype=torch.float32)),
    ("prefill forgets to rescale the running sum",
     "        l[ii] *= alpha;\n", "",
     functools.partial(pins.test_blasst_lambda_zero_is_dense_causal, L=300)),
    ("stable rows attend instead of keeping the cache",
     "if (active[(size_t)b * Tq + i]) {", "if (1) {",
     pins.test_blockquery_all_stable_is_cache_bit_exact),
    ("activity ties to the higher token index",
     "(mj == mi && j < i)", "(mj == mi && j > i)",
     pins.test_losa_classify_unchanged_queries),
    ("attention inside the block made causal",
     "attend_row(q, k, v, dtype, row * D, kvbase, D, toks, Tq, scale, logits, o_in, &lse_in);",
     "attend_row(q, k, v, dtype, row * D, kvbase, D, toks, i + 1, scale, logits, o_in, &lse_in);",
     pins.test_losa_step_all_blocks_equals_dense_attention_over_prefix_and_block),
    ("compressed block as long as the stride",
     "const int t1 = (t0 + len < T) ? t0 + len : T;", "const int t1 = (t0 + stride < T) ? t0 + stride : T;",
     pins.test_nsa_compress_is_avg_pool_with_clipped_tail),
    ("sparse-decode rescale factor inverted",
     "exp(m[hh] - mn)", "exp(mn - m[hh])",
     pins.test_decode_blasst_lambda_zero_is_masked_dense),
    ("group score from the first head only",
     "          acc += dot;\n        }\n        *s = scale * acc;",
     "          acc += dot;\n          break;\n        }\n        *s = scale * acc;",
     pins.test_group_score_is_sum_of_single_head_scores),
    ("compressed-branch log-sum-exp without the max",
     "      lse[(size_t)b * Hq + h] = m + log(l);", "      lse[(size_t)b * Hq + h] = log(l);",
     pins.test_nsa_window_and_compressed_branches_are_sdpa),
    ("compressed-branch logits without the softmax scale",
     "        logit[t - t0] = scale * dot;", "        logit[t - t0] = dot;",
     pins.test_nsa_window_and_compressed_branches_are_sdpa),
]


def _build(i, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutant {i}: the text to replace must occur exactly once"
    os.makedirs(OUT, exist_ok=True)
    src = os.path.join(OUT, f"mutant{i}.c")
    lib = os.path.join(OUT, f"libmutant{i}.so")
    with open(src, "w") as f:
        f.write(text.replace(old, new))
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
                    "-o", lib, src, "-lm"], check=True)
    handle = ctypes.CDLL(lib)
    handle.oracle_num_threads.restype = ctypes.c_int
    return handle


@pytest.mark.parametrize("i", range(len(MUTANTS)), ids=[m[0] for m in MUTANTS])
def test_pin_catches_planted_mistake(i, monkeypatch):
    name, old, new, pin = MUTANTS[i]
    oracle._load()  # the real library is built and loaded first
    monkeypatch.setattr(oracle, "_lib", _build(i, old, new))
    with pytest.raises(AssertionError):
        pin()


def test_unmutated_oracle_passes_the_same_pins():
    for _, _, _, pin in MUTANTS:
        pin()
