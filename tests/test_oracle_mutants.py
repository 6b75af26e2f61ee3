"""Planted mistakes: each mutant is a copy of the oracle's C source with one
plausible error (a dropped term, a wrong sign or index, a swapped operand),
built into its own library; the pins of tests/test_oracle.py must reject
every one of them.  The mistakes are planted only in temporary copies, on the
CPU; the oracle's own source is never modified."""
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
import test_golden as G
import test_oracle as T

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")

# (name, exact text in pa_oracle.c, replacement) -- or (name, [(text, replacement), ...], None)
MUTANTS = [
    ("pool_sum_not_mean", "double mq = sq / n, mk = sk / n;", "double mq = sq, mk = sk;"),
    ("pool_wrong_kv_head", "k[b * ksb + i * kss + (int64_t)kv_of(h, H, Hkv) * ksh + c]",
     "k[b * ksb + i * kss + (int64_t)(h % Hkv) * ksh + c]"),
    ("pool_no_rounding", "if (qp_bf16) qp_bf16[o] = pa_oracle_f64_to_bf16(mq);",
     "if (qp_bf16) qp_bf16[o] = pa_oracle_f64_to_bf16(mq * 1.001);"),
    ("rne_ties_away", "double r = nearbyint(x / q) * q;", "double r = round(x / q) * q;"),
    ("scores_no_causal_mask", "            if (causal && j > i) continue;\n            double s = 0.0;",
     "            double s = 0.0;"),
    ("scores_min_not_max", "\n            if (s > best) best = s;", "\n            if (best == -INFINITY || s < best) best = s;"),
    ("scores_no_scale", "            s *= scale;\n            if (s > best) best = s;", "            if (s > best) best = s;"),
    ("mass_not_mean_over_rows", "m[j / BLK] += p / BLK;", "m[j / BLK] += p;"),
    ("mass_no_causal", "int jhi = causal ? i + 1 : N;", "int jhi = N;"),
    ("rank_ascending", "    if (a->s > b->s) return -1;\n    if (a->s < b->s) return 1;",
     "    if (a->s < b->s) return -1;\n    if (a->s > b->s) return 1;"),
    ("rank_ties_high_index_first", "return (a->kb < b->kb) ? -1 : (a->kb > b->kb);",
     "return (a->kb > b->kb) ? -1 : (a->kb < b->kb);"),
    ("rank_no_forced_diagonal", "if (qb > 0) out[1] = qb;", "if (qb > 0) out[1] = qb - 1 > 0 ? qb - 1 : qb;"),
    ("budget_off_by_one", "if (t + 1 >= forced(nb - 1) && cum >= gfx) { kh = t + 1; break; }",
     "if (t + 1 >= forced(nb - 1) && cum >= gfx) { kh = t + 2 > nb ? nb : t + 2; break; }"),
    ("budget_strict", "cum >= gfx) { kh = t + 1; break; }", "cum > gfx) { kh = t + 1; break; }"),
    ("budget_floor_not_ceil", "clampi(((int64_t)kh * (qb + 1) + nb - 1) / nb, forced(qb), qb + 1)",
     "clampi(((int64_t)kh * (qb + 1)) / nb, forced(qb), qb + 1)"),
    ("fixed_floor_not_ceil", "clampi(((int64_t)frac_permille * (qb + 1) + 999) / 1000, forced(qb), qb + 1)",
     "clampi(((int64_t)frac_permille * (qb + 1)) / 1000, forced(qb), qb + 1)"),
    ("sparse_unnormalised", "                    double p = exp(zz - zmax) / den;", "                    double p = exp(zz - zmax);"),
    ("sparse_no_causal", "                    if (!causal || j <= i) {\n                        s = 0.0;",
     "                    if (1) {\n                        s = 0.0;"),
    ("sparse_v_from_q_head", "o[c] += p * bf16_to_f64(v[b * vsb + (int64_t)j * vss + kvh * vsh + c]);\n                }\n            if (lse)",
     "o[c] += p * bf16_to_f64(v[b * vsb + (int64_t)j * vss + (h % Hkv) * vsh + c]);\n                }\n            if (lse)"),
    ("dense_wrong_scale", "            z[j] = scale * s;", "            z[j] = s;"),
    ("stride_first_row_of_window", "for (int ii = stride - 1; ii < BLK; ii += stride) {",
     "for (int ii = 0; ii < BLK; ii += stride) {"),
    ("stride_ignored", "for (int ii = stride - 1; ii < BLK; ii += stride) {",
     "for (int ii = 0; ii < BLK; ii++) {"),
    ("skip_when_any_row_below", "                    if (e > worst) worst = e;",
     "                    if (worst == -INFINITY || e < worst) worst = e;"),
    ("skip_running_max_frozen", "                if (mt[ii * n + t] > row_max[ii]) row_max[ii] = mt[ii * n + t];",
     "                if (t == 0) row_max[ii] = mt[ii * n + t];"),
    ("skip_block_still_counted", "            use[t] = skip_in ? !skip_in[base + blk[t]] : !own;",
     "            use[t] = skip_in ? !skip_in[base + blk[t]] : 1;"),
    ("xattn_main_diagonal", "q[b * qsb + (int64_t)(R * S + S - 1 - t) * qss + h * qsh + e]",
     "q[b * qsb + (int64_t)(R * S + t) * qss + h * qsh + e]"),
    ("xattn_no_causal", "int cend = causal ? R + 1 : ncol;", "int cend = ncol;"),
    ("xattn_scale_without_stride", "double scale = 1.0 / (sqrt((double)d) * S);", "double scale = 1.0 / sqrt((double)d);"),
    ("find_blocks_strict", "if (cum >= tfx) { n = t + 1; break; }", "if (cum > tfx) { n = t + 1; break; }"),
    ("find_blocks_ascending", "while (u > 0 && (m[out[u - 1]] < m[t] ||", "while (u > 0 && (m[out[u - 1]] > m[t] ||"),
    ("noncausal_budget_row_scaled", ": clampi(kh, forced(qb), nb);",
     ": clampi(((int64_t)kh * (qb + 1) + nb - 1) / nb, forced(qb), nb);"),
    ("noncausal_dense_still_causal", "int nkeys = causal ? i + 1 : N;", "int nkeys = i + 1;"),
    ("noncausal_rank_keeps_only_lower_blocks", "int len = row_len(causal, nb, qb);\n                out[0] = 0;",
     "int len = qb + 1;\n                out[0] = 0;"),
    ("skip_threshold_log2", "double lnl = (lambda > 0.0) ? log(lambda) : -INFINITY;",
     "double lnl = (lambda > 0.0) ? log2(lambda) : -INFINITY;"),
]

# The pins each mutant runs against (all of them are cheap).
PINS = [
    T.test_bf16_rne_exact_and_midpoints,
    T.test_pool_closed_form,
    T.test_pool_one_head_per_group_is_identity,
    T.test_pool_matches_numpy_mean_and_head_permutation,
    T.test_scores_one_head_per_group_equal_per_head_scores,
    T.test_scores_planted_pair_and_causal_mask,
    lambda: T.test_strided_scores_planted_rows(4),
    T.test_mass_rows_sum_to_one_and_match_scipy_softmax,
    lambda: T.test_rank_brute_force_with_ties(0),
    lambda: T.test_budget_brute_force_and_invariants(0),
    T.test_budget_is_find_blocks_when_ranking_follows_mass,
    T.test_fixed_and_all_counts_closed_form,
    T.test_dense_matches_torch_sdpa,
    T.test_sparse_all_equals_dense,
    T.test_sparse_matches_sdpa_with_block_mask,
    lambda: T.test_skip_brute_force(0.2),
    T.test_skip_planted_running_max,
    T.test_skip_sweep_skips_some_and_nests,
    lambda: T.test_xattn_mass_is_the_antidiagonal_sum_softmax(8),
    T.test_xattn_stride_one_is_the_exact_mass,
    T.test_find_blocks_brute_force,
    T.test_noncausal_dense_and_sparse_all_match_sdpa,
    T.test_noncausal_scores_mass_rank_budget,
    G.test_golden_rank,
    G.test_golden_budget,
]


def build_mutant(src_text: str, old, new, workdir: str) -> str:
    edits = old if isinstance(old, list) else [(old, new)]
    for a, b in edits:
        assert src_text.count(a) == 1, f"mutation anchor not unique: {a[:50]!r}"
        src_text = src_text.replace(a, b)
    path = os.path.join(workdir, "m.c")
    with open(path, "w") as f:
        f.write(src_text)
    lib = os.path.join(workdir, "libm.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-o", lib, path, "-lm"])
    return lib


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, monkeypatch):
    import ctypes
    src = open(SRC).read()
    d = tempfile.mkdtemp(prefix="pa_mutant_")
    try:
        libpath = build_mutant(src, old, new, d)
        L = ctypes.CDLL(libpath)
        L.pa_oracle_f64_to_bf16.restype = ctypes.c_uint16
        L.pa_oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        L.pa_oracle_num_threads.restype = ctypes.c_int
        monkeypatch.setattr(oracle, "_lib", L)
        caught = []
        for pin in PINS:
            try:
                pin()
            except AssertionError:
                caught.append(getattr(pin, "__name__", "pin"))
                break
        assert caught, f"no pin rejects the planted mistake {name}"
    finally:
        shutil.rmtree(d, ignore_errors=True)
