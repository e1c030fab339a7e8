"""Pin sensitivity: plant one plausible mistake at a time in a copy of the oracle's
C source (on the CPU), build it, and require that at least one pin fails.  The
shipped oracle is never modified."""
import os
import tempfile

import pytest

import oracle
from tests import oracle_pins as pins

with open(oracle.SOURCE) as _fh:
    _SRC = _fh.read()

# (name, original text, planted mistake)
MUTANTS = [
    ("summary_min_flipped", "if (x < lo) lo = x;", "if (x > lo) lo = x;"),
    ("bound_takes_min", "u += (lo > hi) ? lo : hi;", "u += (lo < hi) ? lo : hi;"),
    ("bound_only_max_side", "u += (lo > hi) ? lo : hi;", "u += hi;"),
    ("group_sum_dropped", "total += u;", "total = u;"),
    ("wrong_head_row", "double lo = q[h * d + c] * smin", "double lo = q[c] * smin"),
    ("tie_to_higher_index", "return ia < ib;", "return ia > ib;"),
    ("ema_alpha_beta_swapped", "double decayed = alpha * e[b];", "double decayed = beta * e[b];"),
    ("ema_no_decay", "double decayed = alpha * e[b];", "double decayed = e[b];"),
    ("ema_contracted_fma", "e[b] = decayed + added;", "e[b] = fma(alpha, e[b], added);"),
    ("attention_scale_dropped", "double p = exp(scale * dot_q_k(q, k + (size_t)t * d, d) - m);",
     "double p = exp(dot_q_k(q, k + (size_t)t * d, d) - m);"),
    ("attention_tail_token_dropped",
     "int t0 = blocks[i] * bs, t1 = t0 + bs < n ? t0 + bs : n;\n        for (int t = t0; t < t1; ++t) {\n            double p",
     "int t0 = blocks[i] * bs, t1 = t0 + bs < n ? t0 + bs : n - 1;\n        for (int t = t0; t < t1; ++t) {\n            double p"),
    ("merge_unweighted", "double w = exp(m[j] - ms);", "double w = 1.0;"),
    ("merge_lse_without_max", "*lse = ms + log(ls);", "*lse = log(ls);"),
    ("missed_set_inverted", "if (!contains(pred, npred, sel[i])) missed[nm++]",
     "if (contains(pred, npred, sel[i])) missed[nm++]"),
    ("partial_no_max_shift", "double p = exp(scale * dot_q_k(q, k + (size_t)t * d, d) - mm);",
     "double p = exp(scale * dot_q_k(q, k + (size_t)t * d, d));"),
    ("variant_max_takes_min", "if (h == 0 || u > best) best = u;", "if (h == 0 || u < best) best = u;"),
    ("variant_first_sink_skipped", "for (int b = 0; b < n_sink", "for (int b = 1; b < n_sink"),
    ("variant_local_from_oldest", "int b = nb - 1 - i;", "int b = i;"),
    ("rep_offset_ignored", "const uint16_t *krow = k + ((size_t)b * bs + off) * d;",
     "const uint16_t *krow = k + ((size_t)b * bs) * d;"),
    ("paged_wrong_head", "((size_t)table[t / bs] * Hkv + h) * bs", "((size_t)table[t / bs] * Hkv) * bs"),
    ("paged_block_not_mapped", "((size_t)table[t / bs] * Hkv + h) * bs", "((size_t)(t / bs) * Hkv + h) * bs"),
    ("rep_tail_not_clamped", "if (off > valid - 1) off = valid - 1;", "if (off > bs - 1) off = bs - 1;"),
    ("rep_first_head_only", "total += q[h * d + c] * bf16_val(krow[c]);", "total += q[c] * bf16_val(krow[c]);"),
    ("rep_last_token_only", "for (int j = 0; j < r; ++j) {\n                int off = rep",
     "for (int j = r - 1; j < r; ++j) {\n                int off = rep"),
    ("step_tail_summary_skipped",
     "oracle_block_summary(ku, n, d, bs, tail, mn + (size_t)tail * d, mx + (size_t)tail * d);", ";"),
    ("step_predicts_before_update",
     "oracle_ema_update(e, nb, su, nsel, D->alpha);\n        for (int j = 0; j < D->P; ++j) pn[j] = -1;\n"
     "        oracle_top_ranked(e, nb, D->P, pn);",
     "for (int j = 0; j < D->P; ++j) pn[j] = -1;\n        oracle_top_ranked(e, nb, D->P, pn);\n"
     "        oracle_ema_update(e, nb, su, nsel, D->alpha);"),
    ("prr_reuses_dropped_partials", "if (!keep[j]) continue;", "if (0 && !keep[j]) continue;"),
    ("prr_repair_skipped", "for (int i = 0; i < nm; ++i) {\n        oracle_block_partial",
     "for (int i = 0; i < 0; ++i) {\n        oracle_block_partial"),
    ("step_wrong_query_group", "qg[h * d + c] = bf16_val(q[((size_t)b * D->Hq + kvh * G + h) * d + c]);",
     "qg[h * d + c] = bf16_val(q[((size_t)b * D->Hq + h) * d + c]);"),
]


@pytest.mark.parametrize("name,orig,bad", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, orig, bad):
    assert _SRC.count(orig) >= 1, f"mutation anchor for {name} not found"
    src = _SRC.replace(orig, bad, 1)
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "mutant.c")
        so = os.path.join(tmp, "libmutant.so")
        with open(c, "w") as fh:
            fh.write(src)
        oracle.build(source=c, output=so, force=True)
        o = oracle.Oracle(so)
        failed = []
        for check in pins.ALL_CHECKS:
            try:
                check(o)
            except AssertionError:
                failed.append(check.__name__)
                break
        assert failed, f"no pin caught the planted mistake {name}"
