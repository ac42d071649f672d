"""Planted mistakes: each mutant is a copy of the oracle's C source with one
plausible error (a dropped term, a wrong sign, index or divisor, a transposed
operand).  It is compiled on the CPU into a temporary library and the whole
battery of oracle pins runs against it: at least one pin must fail.  This is
the evidence that the pins constrain every part of the oracle."""
import importlib
import inspect
import os
import subprocess

import pytest

from conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "dit_oracle.c")

MUTANTS = {
    "ln_unbiased_variance": ("var /= (double)D;", "var /= (double)(D - 1);"),
    "ln_eps_outside_root": ("1.0 / sqrt(var + eps)", "1.0 / (sqrt(var) + eps)"),
    "ln_scale_without_one": ("(1.0 + scale[d])", "scale[d]"),
    "ln_shift_scale_swapped": ("(1.0 + scale[d]) + shift[d]", "(1.0 + shift[d]) + scale[d]"),
    "ln_mean_dropped": ("(x[d] - mu) * inv", "x[d] * inv"),
    "gate_adds_instead_of_multiplies": ("+ g[d] * dito_bf16_to_f64(r[row + d])",
                                        "+ g[d] + dito_bf16_to_f64(r[row + d])"),
    "gate_ln_reads_unrounded": ("x_out[row + d] = h;\n                work[d] = dito_bf16_to_f64(h);",
                                "x_out[row + d] = h;\n                work[d] = v;"),
    "tok_gate_ln_reads_unrounded": ("x_out[tok * D + d] = h;\n                work[d] = dito_bf16_to_f64(h);",
                                    "x_out[tok * D + d] = h;\n                work[d] = v;"),
    "tok_set_ignored": ("int64_t m = b * mod_batch_stride + set * mod_set_stride;",
                        "int64_t m = b * mod_batch_stride;"),
    "tok_set_strided_as_sample": ("int64_t m = b * mod_batch_stride + set * mod_set_stride;",
                                  "int64_t m = (b + set) * mod_set_stride;"),
    "tok_gated_index_per_token_of_sample": ("int sg = set_index[tok];", "int sg = set_index[n];"),
    "tok_gated_gate_from_set0": ("gate[mg + d]", "gate[b * mod_batch_stride + d]"),
    "store_operands_swapped": ("dito_f64_to_bf16(dito_bf16_to_f64(after[i]) - dito_bf16_to_f64(before[i]))",
                               "dito_f64_to_bf16(dito_bf16_to_f64(before[i]) - dito_bf16_to_f64(after[i]))"),
    "apply_subtracts": ("dito_f64_to_bf16(dito_bf16_to_f64(h[i]) + dito_bf16_to_f64(residual[i]))",
                        "dito_f64_to_bf16(dito_bf16_to_f64(h[i]) - dito_bf16_to_f64(residual[i]))"),
    "apply_ties_away": ("dito_f64_to_bf16(dito_bf16_to_f64(h[i]) + dito_bf16_to_f64(residual[i]))",
                        "dito_f64_to_bf16(nextafter(dito_bf16_to_f64(h[i]) + dito_bf16_to_f64(residual[i]), 1e300))"),
    "gemm_gate_reads_linear_half": ("const uint16_t* wg = w + (int64_t)j * K;",
                                    "const uint16_t* wg = w + ((int64_t)F + j) * K;"),
    "gemm_weight_transposed": ("double tg = xv * dito_bf16_to_f64(wg[k]);",
                               "double tg = xv * dito_bf16_to_f64(w[(int64_t)k * 2 * F + j]);"),
    "gemm_last_term_dropped": ("for (int k = 0; k < K; ++k) {\n                double xv",
                               "for (int k = 0; k < K - 1; ++k) {\n                double xv"),
    "gemm_silu_sign": ("out[r * F + j] = g / (1.0 + exp(-g)) * u;",
                       "out[r * F + j] = g / (1.0 + exp(g)) * u;"),
    "down_gate_by_row": ("const double* g = gate + (m / N) * mod_batch_stride;",
                         "const double* g = gate + (m % N) * mod_batch_stride;"),
    "down_weight_column": ("const uint16_t* wn = w + (int64_t)n * K;",
                           "const uint16_t* wn = w + (int64_t)n;"),
    "down_gate_added": ("dito_bf16_to_f64(x[m * (int64_t)D + n]) + g[n] * s);",
                        "dito_bf16_to_f64(x[m * (int64_t)D + n]) + g[n] + s);"),
    "router_mean_over_full_block": ("qm[j * hd + d] = sq / (double)(t1 - t0);",
                                    "qm[j * hd + d] = sq / (double)block;"),
    "router_keeps_lowest": ("if (sc[oc] > sc[ob] || (sc[oc] == sc[ob] && oc < ob)) best = c;",
                            "if (sc[oc] < sc[ob] || (sc[oc] == sc[ob] && oc < ob)) best = c;"),
    "router_ties_to_higher_index": ("if (sc[oc] > sc[ob] || (sc[oc] == sc[ob] && oc < ob)) best = c;",
                                    "if (sc[oc] > sc[ob] || (sc[oc] == sc[ob] && oc > ob)) best = c;"),
    "router_scores_q_with_q": ("for (int d = 0; d < hd; ++d) s += qm[i * hd + d] * km[j * hd + d];",
                               "for (int d = 0; d < hd; ++d) s += qm[i * hd + d] * qm[j * hd + d];"),
    "router_keep_floor": ("double want = ceil((1.0 - sparsity) * (double)n_blocks - 1e-9);",
                          "double want = floor((1.0 - sparsity) * (double)n_blocks);"),
    "attn_scale_dropped": ("                    s *= scale;\n", "\n"),
    "attn_not_normalised": ("double pw = work[n++] / l;", "double pw = work[n++];"),
    "attn_values_from_k": ("const uint16_t* vu = v + ((int64_t)b * N + u) * row_stride",
                           "const uint16_t* vu = k + ((int64_t)b * N + u) * row_stride"),
    "swiglu_exp_sign": ("a / (1.0 + exp(-a))", "a / (1.0 + exp(a))"),
    "swiglu_halves_swapped": ("double a = dito_bf16_to_f64(in[m * 2 * (int64_t)F + j]);",
                              "double a = dito_bf16_to_f64(in[m * 2 * (int64_t)F + F + j]);"),
    "swiglu_row_stride": ("double b = dito_bf16_to_f64(in[m * 2 * (int64_t)F + F + j]);",
                          "double b = dito_bf16_to_f64(in[m * (int64_t)F + F + j]);"),
    "rms_mean_over_half_head": ("ms /= (double)hd;\n    double inv = 1.0 / sqrt(ms + eps);",
                                "ms /= (double)(hd / 2);\n    double inv = 1.0 / sqrt(ms + eps);"),
    "rms_eps_outside_root": ("double inv = 1.0 / sqrt(ms + eps);",
                             "double inv = 1.0 / (sqrt(ms) + eps);"),
    "ex_head_eps_outside_root": ("                inv = 1.0 / sqrt(ms + eps);",
                                 "                inv = 1.0 / (sqrt(ms) + eps);"),
    "rms_weight_index": ("double u1 = x[2 * p + 1] * inv * w[2 * p + 1];",
                         "double u1 = x[2 * p + 1] * inv * w[2 * p];"),
    "rope_rotation_sign": ("out[2 * p]     = u0 * cos(phi) - u1 * sin(phi);",
                           "out[2 * p]     = u0 * cos(phi) + u1 * sin(phi);"),
    "ex_rotation_sign": ("oh[a] = u0 * cos(phi) - u1 * sin(phi);",
                         "oh[a] = u0 * cos(phi) + u1 * sin(phi);"),
    "rope_rotate_half_layout": ("double u1 = x[2 * p + 1] * inv * w[2 * p + 1];",
                                "double u1 = x[(p + hd / 2) % hd] * inv * w[(p + hd / 2) % hd];"),
    "rope_axis_h_w_swapped": ("axis = 1; i = p - pt;", "axis = 2; i = p - pt;"),
    "rope_frequency_over_head": ("\n        double omega = pow(theta, -2.0 * (double)i / (2.0 * (double)P));",
                                 "\n        double omega = pow(theta, -2.0 * (double)i / (double)hd);"),
    "ex_frequency_over_head": ("\n                double omega = pow(theta, -2.0 * (double)i / (2.0 * (double)P));",
                               "\n                double omega = pow(theta, -2.0 * (double)i / (double)hd);"),
    "rope_pos_axis_index": ("\n        double phi = (double)p3[axis] * omega;",
                            "\n        double phi = (double)p3[0] * omega;"),
    "ex_pos_axis_index": ("\n                double phi = (double)p3[axis] * omega;",
                          "\n                double phi = (double)p3[0] * omega;"),
    "ex_half_partner_index": ("int b = layout == 0 ? 2 * q + 1 : q + hd / 2;",
                              "int b = layout == 0 ? 2 * q + 1 : hd - 1 - q;"),
    "ex_half_rotation_sign": ("oh[b] = u0 * sin(phi) + u1 * cos(phi);",
                              "oh[b] = -u0 * sin(phi) + u1 * cos(phi);"),
    "ex_row_norm_over_head": ("ms /= (double)width;", "ms /= (double)hd;"),
    "ex_row_weight_per_head": ("const double* wh = norm == 1 ? w + (int64_t)h * hd : w;",
                               "const double* wh = w;"),
    "grid_h_w_confused": ("pos[3 * n + 1] = (int32_t)((g / Wg) % Hg);",
                          "pos[3 * n + 1] = (int32_t)((g / Hg) % Wg);"),
    "cache_denominator_uses_cur": ("s_den += fabs(p);", "s_den += fabs(c);"),
    "cache_not_strict": ("return q < threshold ? 1 : 0;", "return q <= threshold ? 1 : 0;"),
    "cache_zero_over_zero": ("q = (num == 0.0) ? 0.0 : INFINITY;", "q = num / den;"),
    "cache_sample_offset": ("int64_t off = (int64_t)b * N * D;", "int64_t off = (int64_t)b * N;"),
    "bf16_double_rounding": ("uint16_t sign = signbit(v) ? 0x8000u : 0u;",
                             "v = (double)(float)v; uint16_t sign = signbit(v) ? 0x8000u : 0u;"),
    "bf16_ties_away": ("double r = rint(k);", "double r = floor(k + 0.5);"),
    "bf16_subnormal_quantum": ("int qexp = (e - 1 >= -126) ? (e - 8) : -133;",
                               "int qexp = e - 8;"),
}

PIN_MODULES = ["test_oracle_bf16", "test_oracle_adaln", "test_oracle_swiglu", "test_oracle_qk",
               "test_oracle_cachedit", "test_oracle_cache_step", "test_oracle_swiglu_gemm",
               "test_oracle_gemm_residual", "test_oracle_subblock",
               "test_oracle_sparse_attention"]


def _pins():
    pins = []
    for modname in PIN_MODULES:
        mod = importlib.import_module(modname)
        for name, fn in inspect.getmembers(mod, inspect.isfunction):
            if name.startswith("test_") and list(inspect.signature(fn).parameters) == ["orc"]:
                pins.append((f"{modname}.{name}", fn))
    return pins


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_every_planted_mistake_is_caught(mutant, tmp_path):
    import oracle
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {mutant} not unique"
    path_c = tmp_path / "mutant.c"
    path_c.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                    "-o", str(lib), str(path_c), "-lm"], check=True)
    orc = oracle.Oracle(str(lib))
    caught = []
    for name, fn in _pins():
        try:
            fn(orc)
        except Exception:  # an assertion, or a crash of the mutant's arithmetic
            caught.append(name)
    assert caught, f"no pin catches the planted mistake {mutant}"
