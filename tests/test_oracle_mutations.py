"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle's C source to a temporary directory, plants one
mistake (a dropped term, a wrong sign or index, a wrong divisor), compiles the
mutant with the same flags, points the oracle binding at it, and checks that at
least one pin test fails. The real oracle library is never modified.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_attention as t_attn
import tests.test_oracle_cag as t_cag
import tests.test_oracle_fp8 as t_fp8
import tests.test_oracle_ivf as t_ivf
import tests.test_oracle_pool as t_pool
import tests.test_oracle_select as t_sel

SRC = os.path.join(os.path.dirname(oracle.__file__), "lf_oracle.c")

PINS = [
    t_pool.test_pool_hand_worked,
    t_pool.test_pool_ramp_closed_form,
    t_pool.test_pool_constant_and_frame_identity,
    t_sel.test_select_hand_worked,
    lambda: [t_sel.test_select_brute_force_with_ties(s) for s in range(6)],
    lambda: [t_sel.test_select_invariants(*a) for a in [(2, 2, 2), (2, 9, 3), (2, 1, 99), (1, 2, 2)]],
    lambda: [t_sel.test_select_1d_brute_force_with_ties(s) for s in range(6)],
    lambda: [t_sel.test_select_1d_invariants(*a) for a in [(2, 1), (2, 7), (2, 10**6), (1, 3)]],
    t_sel.test_select_1d_forces_no_frame,
    t_sel.test_select_1d_matches_two_level_on_frame_structured_scores,
    lambda: [t_ivf.test_ivf_full_probe_equals_exact_selection(*a) for a in [(0, 4, 3), (1, 1, 2), (2, 7, 5), (3, 10, 1)]],
    lambda: [t_ivf.test_ivf_kmeans_matches_sklearn(s) for s in range(4)],
    lambda: [t_ivf.test_ivf_probing_invariants(*a) for a in [(0, 5, 1, 2), (1, 5, 2, 6), (2, 8, 3, 4), (3, 3, 1, 9)]],
    t_ivf.test_ivf_dense_first_chunk,
    t_fp8.test_e4m3_matches_torch_on_values_midpoints_and_random,
    t_fp8.test_e4m3_saturates,
    t_fp8.test_quant_rows_hand_worked,
    t_fp8.test_quant_cols_hand_worked_per_head,
    lambda: [t_fp8.test_quant_keeps_the_largest_magnitude_and_the_error_bound(s) for s in range(3)],
    t_fp8.test_attention_f64_equals_attention_on_bf16_inputs,
    t_fp8.test_quant_rows_f32_hand_worked,
    lambda: [t_fp8.test_quant_rows_f32_matches_torch(s) for s in range(3)],
    lambda: [t_attn.test_all_keep_equals_dense_sdpa(*a) for a in [(100, 64, 16), (64, 64, 8)]],
    t_attn.test_single_block_and_partial_block,
    t_attn.test_rows_subset_and_empty_list,
    t_attn.test_value_is_convex_combination,
    t_attn.test_per_query_block_lists,
    t_cag.test_cag_hand_worked,
    t_cag.test_blocks_for_sparsity_hand_worked,
    lambda: [t_cag.test_cag_budget_identity_and_growth(s) for s in range(20)],
]

# (name, text to find, replacement[, how many occurrences; default all]).
MUTATIONS = [
    ("partial block mean divides by block size", "out[d] = s / (double)(t1 - t0);", "out[d] = s / (double)bt;"),
    ("frame mean divides by padded length", "fo[d] = s / (double)F;", "fo[d] = s / (double)(bpf * bt);"),
    ("blocks straddle frame end", "*t1 = (j + 1) * bt < F ? (j + 1) * bt : F;", "*t1 = (j + 1) * bt;"),
    ("kv head stride ignored", "const uint16_t* kh = k + bh * kv_stride * D;", "const uint16_t* kh = k + bh * (long)NF * F * D;", 1),
    ("ties go to the higher index", "return (a->idx > b->idx) - (a->idx < b->idx);", "return (a->idx < b->idx) - (a->idx > b->idx);"),
    ("bottom-k instead of top-k", "if (a->score > b->score) return -1;", "if (a->score > b->score) return 1;"),
    ("recent frame dropped", "for (int t = NF - n_recent - n_cur; t < NF; ++t) out[n++] = t;", "for (int t = NF - n_cur; t < NF; ++t) out[n++] = t;"),
    ("sink frame dropped", "for (int t = 0; t < n_sink; ++t) out[n++] = t;", "for (int t = 1; t < n_sink; ++t) out[n++] = t;"),
    ("frame scored against a neighbour", "cand[m].score = dot(qr, k_frame + (bh * NF + n_sink + m) * (long)D, D);", "cand[m].score = dot(qr, k_frame + (bh * NF + n_sink + m + 1) * (long)D, D);"),
    ("block score ignores last dim", "for (int d = 0; d < D; ++d) s += a[d] * b[d];", "for (int d = 0; d + 1 < D; ++d) s += a[d] * b[d];"),
    ("softmax scale dropped", "z[s] = scale * acc;", "z[s] = acc;"),
    ("query block index ignores frames", "int r = (int)(t / F) * bpf + (int)((t % F) / bt);", "int r = (int)(t / bt);"),
    ("softmax denominator dropped", "for (int d = 0; d < D; ++d) o[d] /= denom;", ""),
    ("CAG sign flipped", "s_out[i] = s_base - beta / sqrt(T[i]);", "s_out[i] = s_base + beta / sqrt(T[i]);"),
    ("CAG alpha = 1/T", "double alpha = 1.0 / sqrt(T[i]);", "double alpha = 1.0 / T[i];"),
    ("CAG dense chunk weight dropped", "if (target_over_all) W += w[i];", ""),
    ("1-D keeps one block too few", "for (int t = 0; t < keep; ++t) kept[t] = cand[t].idx;", "for (int t = 0; t + 1 < keep; ++t) kept[t] = cand[t].idx;"),
    ("1-D scores the neighbouring block", "cand[g].score = dot(qr, k_pool + (bh * (long)Nkv + g) * D, D);", "cand[g].score = dot(qr, k_pool + (bh * (long)Nkv + (g + 1) % Nkv) * D, D);"),
    ("1-D list left in score order", "qsort(kept, (size_t)keep, sizeof(int), by_int);", ""),
    ("1-D first chunk not dense", "int keep = (chunk_index == 1 || topk_blocks > Nkv) ? Nkv : topk_blocks;", "int keep = topk_blocks > Nkv ? Nkv : topk_blocks;"),
    ("IVF ranks clusters by the negated score", "cl[j].score = dot(qr, cent + (long)j * D, D);", "cl[j].score = -dot(qr, cent + (long)j * D, D);"),
    ("IVF centroids never move", "for (int d = 0; d < D; ++d) cent[(long)j * D + d] = sum[(long)j * D + d] / (double)cnt[j];", "for (int d = 0; d < D; ++d) cent[(long)j * D + d] += 0.0 * sum[(long)j * D + d];"),
    ("IVF distance drops the last coordinate", "                    for (int d = 0; d < D; ++d) {\n                        double t = km", "                    for (int d = 0; d + 1 < D; ++d) {\n                        double t = km"),
    ("IVF probes one cluster too few", "if (t >= np_min && have >= kf) break;", "if (t + 1 >= np_min && have >= kf) break;"),
    ("e4m3 keeps four mantissa bits", "step = ldexp(1.0, e - 4);", "step = ldexp(1.0, e - 5);"),
    ("e4m3 truncates", "double qv = nearbyint(a / step) * step;", "double qv = floor(a / step) * step;"),
    ("e4m3 subnormal step halved", "step = ldexp(1.0, -9);", "step = ldexp(1.0, -10);"),
    ("row scale from the first element", "double t = fabs(bf16_to_f64(x[i * D + d]));", "double t = fabs(bf16_to_f64(x[i * D]));"),
    ("column scale from the first row", "double t = fabs(bf16_to_f64(x[(g * stride + i) * D + d]));", "double t = fabs(bf16_to_f64(x[(g * stride) * D + d]));"),
    ("fp64 attention drops the last coordinate", "for (int d = 0; d < D; ++d) acc += qt[d] * kh[tok[s] * D + d];", "for (int d = 0; d + 1 < D; ++d) acc += qt[d] * kh[tok[s] * D + d];"),
    ("k_b truncates instead of rounding", "double x = floor((1.0 - s) * (double)n_kv_blocks / (double)n_sel + 0.5);", "double x = floor((1.0 - s) * (double)n_kv_blocks / (double)n_sel);"),
    ("fp32 quantiser scale divides by 447", "float sc = amax > 0.0f ? amax / 448.0f : 1.0f;",
     "float sc = amax > 0.0f ? amax / 447.0f : 1.0f;"),
    ("fp32 quantiser multiplies by the scale", "float y = (float)bf16_to_f64(x[i * D + d]) / sc;",
     "float y = (float)bf16_to_f64(x[i * D + d]) * sc;"),
    ("fp32 quantiser amax of signed values", "float t = (float)fabs(bf16_to_f64(x[i * D + d]));",
     "float t = (float)bf16_to_f64(x[i * D + d]);"),
]


def _build_mutant(tmp_path, find, repl, count=-1):
    src = open(SRC).read()
    assert find in src, f"mutation anchor not found: {find}"
    mutant = src.replace(find, repl, count)
    c = tmp_path / "mutant.c"
    c.write_text(mutant)
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                    "-ffp-contract=off", "-w", "-o", str(so), str(c), "-lm"], check=True)
    return oracle.configure(ctypes.CDLL(str(so)))


def _some_pin_fails():
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError):
            return True
    return False


@pytest.mark.parametrize("mutation", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(tmp_path, monkeypatch, mutation):
    name = mutation[0]
    lib = _build_mutant(tmp_path, *mutation[1:])
    monkeypatch.setattr(oracle, "_lib", lib)
    assert _some_pin_fails(), f"no pin caught the planted mistake: {name}"


def test_unmutated_copy_passes_all_pins(tmp_path, monkeypatch):
    lib = _build_mutant(tmp_path, "#include <math.h>", "#include <math.h>")
    monkeypatch.setattr(oracle, "_lib", lib)
    assert not _some_pin_fails()
