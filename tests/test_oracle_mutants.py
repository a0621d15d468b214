"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of the oracle source (a dropped term, a wrong sign, a
wrong divisor, a dropped index, a flipped comparison), builds it with gcc, and runs the pin
suite against that build in a subprocess: the suite has to fail. CPU only.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ekv_oracle.c")

MUTANTS = {
    "bound_takes_min": ("acc += a > b ? a : b;", "acc += a < b ? a : b;"),
    "variance_divides_by_n_minus_1": ("var[(size_t)j * d + c] = ss / n;",
                                      "var[(size_t)j * d + c] = ss / (n > 1 ? n - 1 : 1);"),
    "meta_ignores_head": ("return (((size_t)block * H_kv + h) * P + t) * d + c;",
                          "return (((size_t)block * H_kv) * P + t) * d + c; (void)h;"),
    "entmax15_wrong_root": ("tk = mean - sqrt(disc);", "tk = mean + sqrt(disc);"),
    "sparsemax_wrong_sign": ("tk = (sum - 1.0) / k;", "tk = (sum + 1.0) / k;"),
    "trunc_moment_drops_pdf_term": ("return r * Phi + b * phi;", "return r * Phi;"),
    "trunc_moment15_drops_variance": ("return (r * r + b * b) * Phi + r * b * phi;",
                                      "return (r * r) * Phi + r * b * phi;"),
    "topk_ties_to_higher_index": ("return a < b ? -1 : (a > b);\n}\n\nstatic int cmp_int_asc",
                                  "return a > b ? -1 : (a < b);\n}\n\nstatic int cmp_int_asc"),
    "gauss_v_not_squared": ("b += qc * qc * var[(size_t)j * d + c];",
                            "b += qc * var[(size_t)j * d + c];"),
    "gauss_select_not_strict": ("ub[(size_t)g * n_pages + j] > tau_hat[g] - delta)",
                                "ub[(size_t)g * n_pages + j] >= tau_hat[g] - delta)"),
    "est_max_uncapped": ("return e < ub ? e : ub;", "return e;"),
    "est_max_wrong_quantile": ("sqrt(2.0 * log((double)n))", "sqrt(log((double)n))"),
    "softmax_stat_drops_max": ("stat[g] = mx + log(l);", "stat[g] = log(l);"),
    "moment_drops_cross_moment_term": ("fE[a] = vbar[a] + scale / n_e * acc;", "fE[a] = vbar[a];"),
    "moment_cross_moment_uncentred": (
        "cache_off(pt_row[j], h, t, c, H_kv, P, d)) - kbar[c];\n"
        "                dv[c] = elem(v_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d)) - vbar[c];",
        "cache_off(pt_row[j], h, t, c, H_kv, P, d));\n"
        "                dv[c] = elem(v_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d));"),
    "moment_cross_moment_without_scale": ("fE[a] = vbar[a] + scale / n_e * acc;",
                                          "fE[a] = vbar[a] + acc / n_e;"),
    "moment_jensen_drops_count": ("const double logZE = log((double)n_e) + sbar;",
                                  "const double logZE = sbar;"),
    "moment_mix_weights_swapped": ("og[a] = wR * og[a] + (1.0 - wR) * fE[a];",
                                   "og[a] = (1.0 - wR) * og[a] + wR * fE[a];"),
    "token_score_first_query_only": ("            for (int g = 0; g < G; ++g) {\n                double sg = 0.0;",
                                     "            for (int g = 0; g < 1; ++g) {\n                double sg = 0.0;"),
    "token_candidates_past_the_sequence_end": (
        "        int n = seq_len - j * P < P ? seq_len - j * P : P;\n        for (int t = 0; t < n; ++t) {\n            double acc",
        "        int n = P;\n        for (int t = 0; t < n; ++t) {\n            double acc"),
    "token_attention_ignores_position": ("        blk[i] = pt_row[j];\n        pos[i] = t;",
                                         "        blk[i] = pt_row[j];\n        pos[i] = 0;"),
    "moment_sums_transposed": ("                    S[(size_t)a * d + c] += va * elem(",
                               "                    S[(size_t)c * d + a] += va * elem("),
    "bound_drops_scale": ("            acc *= scale;\n", "            (void)scale;\n"),
    "gauss_mean_drops_scale": ("m[(size_t)g * n_pages + j] = scale * a;", "m[(size_t)g * n_pages + j] = a;"),
    "gauss_variance_scale_not_squared": ("v[(size_t)g * n_pages + j] = scale * scale * b;",
                                         "v[(size_t)g * n_pages + j] = scale * b;"),
    "topk_keeps_one_page_too_many": ("int cnt = k < n ? k : n;", "int cnt = k < n ? k + 1 : n;"),
    "meta_max_takes_min": ("                if (x > hi) hi = x;", "                if (x < hi) hi = x;"),
    "meta_mean_divides_by_page_size": ("            double mu = sum / n;", "            double mu = sum / P;"),
    "gauss_F_ignores_token_counts": ("F += (double)cnt[j] * ora_trunc_moment(a, b, tau, alpha);",
                                     "F += ora_trunc_moment(a, b, tau, alpha); (void)cnt;"),
    "gauss_F_drops_alpha_factor_on_b": ("        double b = (alpha - 1.0) * sqrt(v[j] > 0.0 ? v[j] : 0.0);\n        F +=",
                                        "        double b = sqrt(v[j] > 0.0 ? v[j] : 0.0);\n        F +="),
    "gauss_tau_bisects_the_wrong_way": ("            lo = mid;\n        else\n            hi = mid;",
                                        "            hi = mid;\n        else\n            lo = mid;"),
    "gauss_select_needs_every_query": (
        "        int keep = 0;\n        for (int g = 0; g < G; ++g)\n            if ((alpha - 1.0) * ub[(size_t)g * n_pages + j] > tau_hat[g] - delta)\n                keep = 1;",
        "        int keep = 1;\n        for (int g = 0; g < G; ++g)\n            if (!((alpha - 1.0) * ub[(size_t)g * n_pages + j] > tau_hat[g] - delta))\n                keep = 0;"),
    "gauss_select_margin_sign": ("ub[(size_t)g * n_pages + j] > tau_hat[g] - delta)\n                keep = 1;",
                                 "ub[(size_t)g * n_pages + j] > tau_hat[g] + delta)\n                keep = 1;"),
    "entmax15_weights_not_squared": ("p[i] = r > 0.0 ? (alpha == 2.0 ? r : r * r) : 0.0;",
                                     "p[i] = r > 0.0 ? r : 0.0;"),
    "softmax_not_normalised": ("            for (int i = 0; i < n_tok; ++i)\n                p[i] /= l;\n",
                               "            (void)0;\n"),
    "attention_reads_invalid_tokens": (
        "n_tok += seq_len - j * P < P ? seq_len - j * P : P;", "n_tok += P;"),
    "quality_sums_the_kept_mass": ("            if (!in_sel[i]) dsum += p;", "            if (in_sel[i]) dsum += p;"),
    "quality_given_stat_ignored": ("                    p = exp(s - stat[g]);", "                    p = exp(s);"),
    "quality_counts_every_token_as_support": ("            int member = mode == ORA_SOFTMAX ? 1 : p > 0.0;",
                                              "            int member = 1;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found: " + name
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-D_DEFAULT_SOURCE", "-O2", "-fPIC", "-shared",
                           "-o", str(lib), str(mut), "-lm"])
    env = dict(os.environ, EKV_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "planted mistake %s went unnoticed:\n%s" % (name, r.stdout[-2000:])
