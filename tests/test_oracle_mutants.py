"""Planted mistakes in copies of the oracle must each fail at least one pin (CPU only).

Each mutant is a text substitution in a temporary copy of oracle/oracle.c -- a dropped
term, a wrong sign, index or order, a wrong rounding -- compiled on its own.  The real
oracle source is never modified.
"""
import os

import pytest

import oracle
import pins

MUTANTS = {
    "rms_drops_eps": ("sqrt(sumsq / (double)D + eps)", "sqrt(sumsq / (double)D)"),
    "rms_sum_not_mean": ("sqrt(sumsq / (double)D + eps)", "sqrt(sumsq + eps)"),
    "rms_weight_reversed": ("double wj = w ? widen(w, dt, j) : 1.0;\n        y[j] = x[j] / denom",
                            "double wj = w ? widen(w, dt, D - 1 - j) : 1.0;\n        y[j] = x[j] / denom"),
    "rms_null_weight_is_zero": ("double wj = w ? widen(w, dt, j) : 1.0;\n        y[j] = x[j] / denom",
                                "double wj = w ? widen(w, dt, j) : 0.0;\n        y[j] = x[j] / denom"),
    "rms_multiplies_by_denom": ("y[j] = x[j] / denom * wj;", "y[j] = x[j] * denom * wj;"),
    "add_normalises_unrounded_h": ("row[j] = widen(h, dt, i);", "row[j] = (double)sum;"),
    "add_drops_residual": ("float sum = (float)widen(x, dt, i) + (float)widen(r, dt, i);",
                           "float sum = (float)widen(x, dt, i);"),
    "allreduce_float_accumulation": ("double s = 0.0;\n            for (int p = 0; p < nparts; ++p)",
                                     "float s = 0.0f;\n            for (int p = 0; p < nparts; ++p)"),
    "allreduce_drops_last_part": ("for (int p = 0; p < nparts; ++p) s +=",
                                  "for (int p = 0; p < nparts - 1; ++p) s +="),
    "allreduce_rounds_through_binary32": ("((uint16_t*)xb)[o] = oracle_bf16_from_f64(s);",
                                          "((uint16_t*)xb)[o] = oracle_bf16_from_f64((double)(float)s);"),
    "allreduce_skips_residual": ("int rc = oracle_add_rms_norm(xb, (const char*)r + off * esz,",
                                 "int rc = oracle_add_rms_norm(xb, (const char*)xb,"),
    "llama3_thresholds_swapped": ("if (wavelen < orig / high_freq_factor) {",
                                  "if (wavelen < orig / low_freq_factor) {"),
    "llama3_ramp_reversed": ("const double s = (orig / wavelen - low_freq_factor) / (high_freq_factor - low_freq_factor);",
                             "const double s = (high_freq_factor - orig / wavelen) / (high_freq_factor - low_freq_factor);"),
    "llama3_multiplies_by_factor": ("            out[i] = theta / factor;\n",
                                    "            out[i] = theta * factor;\n"),
    "llama3_theta_over_dims_half": ("const double theta = pow(base, -(double)(2 * i) / (double)dims);",
                                    "const double theta = pow(base, -(double)i / (double)dims);"),
    "yarn_ramp_reversed": ("gamma = (r - alpha) / (beta - alpha);",
                           "gamma = (beta - r) / (beta - alpha);"),
    "yarn_multiplies_by_s": ("out[d] = (1.0 - gamma) * theta_d / s + gamma * theta_d;",
                             "out[d] = (1.0 - gamma) * theta_d * s + gamma * theta_d;"),
    "yarn_ramp_roles_swapped": ("out[d] = (1.0 - gamma) * theta_d / s + gamma * theta_d;",
                                "out[d] = gamma * theta_d / s + (1.0 - gamma) * theta_d;"),
    "yarn_turns_inverted": ("const double r = L / lambda_d;", "const double r = lambda_d / L;"),
    "yarn_temperature_log10": ("*mscale = 0.1 * log(s) + 1.0;", "*mscale = 0.1 * log10(s) + 1.0;"),
    "suscaled_multiplies_by_factor": ("out[i] = theta_i / lambda[i];", "out[i] = theta_i * lambda[i];"),
    "suscaled_long_from_L": ("const double* lambda = seq_len > orig ? long_factors : short_factors;",
                             "const double* lambda = seq_len >= orig ? long_factors : short_factors;"),
    "suscaled_factor_sets_swapped": ("const double* lambda = seq_len > orig ? long_factors : short_factors;",
                                     "const double* lambda = seq_len > orig ? short_factors : long_factors;"),
    "suscaled_factor_index_reversed": ("out[i] = theta_i / lambda[i];",
                                       "out[i] = theta_i / lambda[dims / 2 - 1 - i];"),
    "suscaled_attention_no_sqrt": ("*mscale = s > 1.0 ? sqrt(1.0 + log(s) / log(orig)) : 1.0;",
                                   "*mscale = s > 1.0 ? 1.0 + log(s) / log(orig) : 1.0;"),
    "suscaled_attention_ratio_inverted": ("*mscale = s > 1.0 ? sqrt(1.0 + log(s) / log(orig)) : 1.0;",
                                          "*mscale = s > 1.0 ? sqrt(1.0 + log(orig) / log(s)) : 1.0;"),
    "suscaled_attention_log_of_max": ("*mscale = s > 1.0 ? sqrt(1.0 + log(s) / log(orig)) : 1.0;",
                                      "*mscale = s > 1.0 ? sqrt(1.0 + log(max_pos) / log(orig)) : 1.0;"),
    "yarn_temperature_squared": ("*mscale = 0.1 * log(s) + 1.0;",
                                 "*mscale = (0.1 * log(s) + 1.0) * (0.1 * log(s) + 1.0);"),
    "layer_mean_over_D_minus_1": ("double mean = sum / (double)D;\n    double sqdev = 0.0;\n    for (int64_t j = 0; j < D; ++j) sqdev +=",
                                  "double mean = sum / (double)(D - 1);\n    double sqdev = 0.0;\n    for (int64_t j = 0; j < D; ++j) sqdev +="),
    "layer_eps_outside_sqrt": ("double denom = sqrt(var + eps);", "double denom = sqrt(var) + eps;"),
    "rms_eps_outside_sqrt": ("sqrt(sumsq / (double)D + eps)", "(sqrt(sumsq / (double)D) + eps)"),
    "rms_no_sqrt": ("sqrt(sumsq / (double)D + eps)", "(sumsq / (double)D + eps)"),
    "rms_weight_squared": ("y[j] = x[j] / denom * wj;", "y[j] = x[j] / denom * wj * wj;"),
    "rope_theta_index_shifted": ("double theta = freqs ? freqs[i] : pow(base, -2.0 * (double)i / (double)dims);",
                                 "double theta = freqs ? freqs[i] : pow(base, -2.0 * (double)(i + 1) / (double)dims);"),
    "rms_vjp_dw_weighted": ("dw[j] += gj * xj * r;", "dw[j] += gj * wj * xj * r;"),
    "layer_unbiased_variance": ("double var = sqdev / (double)D;",
                                "double var = sqdev / (double)(D - 1);"),
    "layer_drops_mean_in_output": ("y[j] = (x[j] - mean) / denom * wj + bj;",
                                   "y[j] = x[j] / denom * wj + bj;"),
    "layer_drops_bias": ("y[j] = (x[j] - mean) / denom * wj + bj;",
                         "y[j] = (x[j] - mean) / denom * wj;"),
    "layer_drops_eps": ("double denom = sqrt(var + eps);", "double denom = sqrt(var);"),
    "layer_bias_before_scale": ("y[j] = (x[j] - mean) / denom * wj + bj;",
                                "y[j] = ((x[j] - mean) / denom + bj) * wj;"),
    "rope_wrong_sign": ("y[p] = x[p] * c - x[q] * s;", "y[p] = x[p] * c + x[q] * s;"),
    "rope_clockwise": ("y[q] = x[p] * s + x[q] * c;", "y[q] = -x[p] * s + x[q] * c;"),
    "rope_theta_factor": ("pow(base, -2.0 * (double)i / (double)dims)",
                          "pow(base, -1.0 * (double)i / (double)dims)"),
    "rope_theta_over_D": ("pow(base, -2.0 * (double)i / (double)dims)",
                          "pow(base, -2.0 * (double)i / (double)D)"),
    "rope_halves_over_D": ("int64_t q = traditional ? 2 * i + 1 : i + half;",
                           "int64_t q = traditional ? 2 * i + 1 : i + D / 2;"),
    "rope_traditional_swapped": ("int64_t p = traditional ? 2 * i : i;",
                                 "int64_t p = traditional ? 2 * i + 1 : i;\n        if (traditional) { int64_t t_ = 2 * i; (void)t_; }"),
    "rope_ignores_scale": ("double phi = pos * scale * theta;", "double phi = pos * theta;"),
    "rope_inverse_not_negated": ("if (!forward) phi = -phi;", "(void)forward;"),
    "rope_ignores_offset": ("double pos = (double)offset + (double)(k % L);\n        rope_row(x + k * D",
                            "double pos = (double)(k % L);\n        rope_row(x + k * D"),
    "norm_rope_ignores_offset": ("double pos = (double)offset + (double)(k % L);\n        rope_row(nrm",
                                 "double pos = (double)(k % L);\n        rope_row(nrm"),
    "norm_rope_position_k_div_L": ("double pos = (double)offset + (double)(k % L);\n        rope_row(nrm",
                                   "double pos = (double)offset + (double)(k / L);\n        rope_row(nrm"),
    "norm_rope_skips_normalise": ("if (normalize)\n            rms_row(row, w, dt, D, (double)eps, nrm);\n        else\n            memcpy(nrm, row, (size_t)D * sizeof(double));\n        double pos",
                                  "if (0)\n            rms_row(row, w, dt, D, (double)eps, nrm);\n        else\n            memcpy(nrm, row, (size_t)D * sizeof(double));\n        double pos"),
    "rope_ex_skips_normalise": ("if (normalize)\n            rms_row(row, w, dt, D, (double)eps, nrm);\n        else\n            memcpy(nrm, row, (size_t)D * sizeof(double));\n        int64_t l",
                                "if (0)\n            rms_row(row, w, dt, D, (double)eps, nrm);\n        else\n            memcpy(nrm, row, (size_t)D * sizeof(double));\n        int64_t l"),
    "rope_ex_freqs_ignored": ("double theta = freqs ? freqs[i] : pow(base, -2.0 * (double)i / (double)dims);",
                              "double theta = pow(base, -2.0 * (double)i / (double)dims);"),
    "rope_ex_cache_row_ignores_offset": ("int64_t out = y_len > 0 ? (k / L) * y_len + offset + l : k;",
                                         "int64_t out = y_len > 0 ? (k / L) * y_len + l : k;"),
    "rope_ex_cache_row_uses_L": ("int64_t out = y_len > 0 ? (k / L) * y_len + offset + l : k;",
                                 "int64_t out = y_len > 0 ? (k / L) * L + offset + l : k;"),
    "rms_vjp_drops_projection": ("dx[k * D + j] = r * wj * gj - xj * r * r * r * c / (double)D;",
                                 "dx[k * D + j] = r * wj * gj;"),
    "rms_vjp_r_squared": ("dx[k * D + j] = r * wj * gj - xj * r * r * r * c / (double)D;",
                          "dx[k * D + j] = r * wj * gj - xj * r * r * c / (double)D;"),
    "rms_vjp_sum_not_mean": ("dx[k * D + j] = r * wj * gj - xj * r * r * r * c / (double)D;",
                             "dx[k * D + j] = r * wj * gj - xj * r * r * r * c;"),
    "rms_vjp_dw_without_r": ("dw[j] += gj * xj * r;", "dw[j] += gj * xj;"),
    "layer_vjp_drops_mean_a": ("dx[k * D + j] = r * (a - sa / (double)D - xh * sax / (double)D);",
                               "dx[k * D + j] = r * (a - xh * sax / (double)D);"),
    "layer_vjp_drops_xh_term": ("dx[k * D + j] = r * (a - sa / (double)D - xh * sax / (double)D);",
                                "dx[k * D + j] = r * (a - sa / (double)D);"),
    "layer_vjp_dw_uses_x": ("dw[j] += gj * xh;", "dw[j] += gj * widen(x, dt, k * D + j);"),
    "layer_vjp_db_weighted": ("db[j] += gj;", "db[j] += a;"),
    "round_truncates": ("double n = rint(ldexp(a, -qexp));", "double n = trunc(ldexp(a, -qexp));"),
    "round_ties_away": ("double n = rint(ldexp(a, -qexp));", "double n = round(ldexp(a, -qexp));"),
    "round_subnormal_quantum": ("int qexp = (e < -125 ? -125 : e) - 8;", "int qexp = e - 8;"),
}


@pytest.fixture(scope="module")
def source():
    with open(oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / "oracle_mutant.c"
    src.write_text(source.replace(old, new))
    lib = oracle.compile_oracle(str(src), str(tmp_path / "liboracle_mutant.so"))
    mutant = oracle.Oracle(lib)
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(mutant)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"planted mistake {name!r} passed every pin"
