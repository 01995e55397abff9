"""Plant plausible mistakes in copies of the oracle and check that the pins catch each.

Every mutant is an edited copy of oracle/vx_oracle.c compiled into a temporary folder;
the real oracle is never modified.  A mutant that passes every pin would mean the pins
leave that part of the oracle unchecked.  CPU only.
"""
import os

import pytest

import oracle
from oracle import build as obuild
import pins

SRC = open(obuild.SRC).read()

# (name, exact snippet in the oracle source, replacement)
MUTANTS = [
    ("centroid_divides_by_page_size", "double mean = sum / (double)m;", "double mean = sum / (double)P;"),
    ("centroid_reads_past_length",
     "for (int32_t t = 0; t < m; ++t)\n                        sum +=",
     "for (int32_t t = 0; t < P; ++t)\n                        sum +="),
    ("centroid_ignores_row_start",
     "int64_t phys = page_indices[page_ptr[b] + j];\n            int32_t m = valid_in_page(seq_lens[b], P, j);",
     "int64_t phys = page_indices[j];\n            int32_t m = valid_in_page(seq_lens[b], P, j);"),
    ("narrow_via_float", "r = ldexp(nearbyint(ldexp(ax, 8 - e)), e - 8);",
     "r = ldexp(nearbyint(ldexp((double)(float)ax, 8 - e)), e - 8);"),
    ("narrow_truncates", "r = ldexp(nearbyint(ldexp(ax, 8 - e)), e - 8);",
     "r = ldexp(floor(ldexp(ax, 8 - e)), e - 8);"),
    ("scores_first_head_only", "for (int32_t g = h * G; g < (h + 1) * G; ++g) {\n                    const uint16_t *qg",
     "for (int32_t g = h * G; g < h * G + 1; ++g) {\n                    const uint16_t *qg"),
    ("scores_wrong_kv_head", "int64_t c0 = (phys * Hkv + h) * Dqk;", "int64_t c0 = (phys * Hkv + 0) * Dqk;"),
    ("scores_drop_last_dim", "for (int32_t d = 0; d < dims; ++d) {", "for (int32_t d = 0; d < dims - 1; ++d) {"),
    ("scores_ignore_score_dims", "int32_t dims = score_dims > 0 ? score_dims : Dqk;", "int32_t dims = Dqk;"),
    ("topk_ties_to_higher_index", "return (x->j > y->j) - (x->j < y->j);", "return (x->j < y->j) - (x->j > y->j);"),
    ("topk_one_short", "for (int32_t i = 0; i < k; ++i) out[i] = i < keff ? all[i].j : -1;",
     "for (int32_t i = 0; i < k; ++i) out[i] = i < keff - 1 ? all[i].j : -1;"),
    ("topk_ascending_scores", "if (x->s > y->s) return -1;\n    if (x->s < y->s) return 1;",
     "if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;"),
    ("splitmix_constant_typo", "0xbf58476d1ce4e5b9ULL", "0xbf58476d1ce4e5b8ULL"),
    ("prefill_slot_off_by_one", "int32_t in_page = pos % P;", "int32_t in_page = (pos + 1) % P;"),
    ("prefill_rows_restart_per_request", "if (L < 1 || L > max_len || fp < 0 || fp > L) continue;",
     "if (L < 1 || L > max_len || fp < 0 || fp > L) continue;\n        row = 0;"),
    ("prefill_ignores_row_start", "int64_t page = page_indices[page_ptr[b] + pos / P];",
     "int64_t page = page_indices[pos / P];"),
    ("approx_emits_boundary_bucket", "if (code[j] > bstar) out[filled++] = j;", "if (code[j] >= bstar) out[filled++] = j;"),
    ("approx_fill_not_rotated", "int32_t j = (o + i) % n;", "int32_t j = i;"),
    ("approx_clamp_off_by_one", "c = f >= (double)(nbins - 1) ? nbins - 1 : (int32_t)f;",
     "c = f >= (double)(nbins - 2) ? nbins - 2 : (int32_t)f;"),
    ("approx_scale_by_range_plus_one", "float scale = (float)nbins / range;", "float scale = (float)nbins / (range + 1.0f);"),
    ("attend_drops_scale", "logit[T] = sm_scale * dot;", "logit[T] = dot;"),
    ("attend_reads_past_length", "int32_t m = valid_in_page(L, P, j);\n                for (int32_t t = 0; t < m; ++t) {\n                    row_k[T]",
     "int32_t m = P;\n                for (int32_t t = 0; t < m; ++t) {\n                    row_k[T]"),
    ("attend_lse_log2", "lse[(int64_t)b * Hq + g] = mx + log(l);", "lse[(int64_t)b * Hq + g] = mx + log2(l);"),
    ("attend_value_slot_zero", "row_v[T] = mla_shared_kv ? row_k[T] : ((phys * Hkv + h) * P + t) * Dv;",
     "row_v[T] = mla_shared_kv ? row_k[T] : ((phys * Hkv + h) * P + 0) * Dv;"),
    ("attend_wrong_group", "int32_t h = g / G;", "int32_t h = g % Hkv;"),
    ("attend_ignores_sel", "int32_t j = sel ? sel[((int64_t)b * Hkv + h) * k + i] : i;",
     "int32_t j = sel ? i : i;"),
    ("append_wrong_slot", "int32_t slot = pos % P;", "int32_t slot = (pos + 1) % P;"),
]


def _run_pins():
    """Names of the pins that fail (stops after the first failure)."""
    for pin in pins.ALL_PINS:
        try:
            pin()
        except Exception:  # an assertion or a crash both count as caught
            return [pin.__name__]
    return []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    assert SRC.count(old) == 1, f"mutation anchor for {name} must be unique in the oracle source"
    lib = obuild.build_variant(SRC.replace(old, new), str(tmp_path), name)
    with oracle.using(lib):
        failed = _run_pins()
    assert failed, f"mutant {name} passed every pin"
