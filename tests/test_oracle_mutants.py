"""Planted mistakes in the oracle must be caught by the pins.

Each case copies onebit_oracle.c to a temporary directory, plants one
plausible mistake (a dropped term, a wrong sign, a wrong index, an inverted
ratio, ...), builds it with the same flags, and checks that at least one pin
of tests/oracle_pins.py fails on it.  Where the oracle repeats a statement
(the same server average in the 1-bit and 2-bit stages, say), the mutant names
the occurrence it plants.  Every planted mistake keeps memory accesses in
bounds, so a mutant can only compute wrong values, never crash the run.  CPU only; nothing here touches the
product library.
"""

import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "onebit_oracle.c")

MUTANTS = {
    "error_sign": ("err_set(err, err_dtype, e0 + i, c[i] - dequantize(q, s, i))",
                   "err_set(err, err_dtype, e0 + i, c[i] + dequantize(q, s, i))"),
    "error_not_added": ("clip) + err_get(err, err_dtype, e0 + i);", "clip) + 0.0f;", 0),
    "sign_of_zero": ("if (c[i] >= 0.0f) words", "if (c[i] > 0.0f) words"),
    "bit_order": ("words[i / 32] |= 1u << (i % 32)", "words[i / 32] |= 1u << (31 - i % 32)"),
    "scale_no_sqrt": ("return (float)(sqrt(S) / sqrt((double)n));", "return (float)(S / (double)n);"),
    "scale_no_mean": ("return (float)(sqrt(S) / sqrt((double)n));", "return (float)sqrt(S);"),
    "server_sum_not_mean": ("float avg = acc / (float)W;", "float avg = acc;", 0),
    "server_error_dropped": ("c[i] = avg + err_get(srv_err, err_dtype, o + i);", "c[i] = avg;", 0),
    "server_error_sign": ("err_set(srv_err, err_dtype, o + i, c[i] - dequantize(q, s, i))",
                          "err_set(srv_err, err_dtype, o + i, dequantize(q, s, i) - c[i])"),
    "bf16_store_truncates": ("return (uint16_t)((u + 0x7fffu + lsb) >> 16);", "return (uint16_t)(u >> 16);"),
    "bf16_store_ties_up": ("return (uint16_t)((u + 0x7fffu + lsb) >> 16);",
                           "return (uint16_t)((u + 0x8000u) >> 16);"),
    "server_first_worker_only": ("for (int32_t w = 0; w < W; ++w)\n        acc +=",
                                 "for (int32_t w = 0; w < 1; ++w)\n        acc +=", 0),
    # (anchors of the scaled-sign update: the s_srv line above, 6-space indentation)
    "momentum_coeff": ("s_srv[k], i);\n      float mi = beta1 * m[o + i] + one_minus_b1 * g_hat;",
                       "s_srv[k], i);\n      float mi = one_minus_b1 * m[o + i] + beta1 * g_hat;"),
    "param_sign": ("\n      float pi = p[o + i] - lr * mi", "\n      float pi = p[o + i] + lr * mi"),
    "frozen_v_sqrt_dropped": ("\n      float pi = p[o + i] - lr * mi / (sqrtf(v[o + i]) + eps);",
                              "\n      float pi = p[o + i] - lr * mi / (v[o + i] + eps);"),
    "trust_ratio_inverted": ("return (float)(sqrt(P) / sqrt(U));", "return (float)(sqrt(U) / sqrt(P));"),
    "lamb_ratio_dropped": ("float pi = p[i] - lr * r * u;", "float pi = p[i] - lr * u;"),
    "warmup_v_not_squared": ("one_minus_b2 * (g * g)", "one_minus_b2 * g"),
    "warmup_first_worker_only": ("for (int32_t w = 0; w < W; ++w) acc += grad_at",
                                 "for (int32_t w = 0; w < 1; ++w) acc += grad_at"),
    "clip_ignored": ("if (g > clip) return clip;", "if (g > clip) return g;"),
    "bf16_shift": ("[idx] << 16;", "[idx] << 15;"),
    "chunk_word_base": ("wo[k + 1] = wo[k] + words_of(off[k + 1] - off[k]);",
                        "wo[k + 1] = wo[k] + (off[k + 1] - off[k]) / 32;"),
    "nan_not_flagged": ("static int is_nonfinite(float x) { return !isfinite(x); }",
                        "static int is_nonfinite(float x) { return isinf(x); }"),
    # the momentum-error rule
    "ternary_zero_is_positive": ("if (c > 0.0f) return 1;", "if (c >= 0.0f) return 1;"),
    "ternary_error_coeffs_swapped": ("float eps_new = beta1 * eps_old + one_minus_b1 * delta;",
                                     "float eps_new = one_minus_b1 * eps_old + beta1 * delta;"),
    "ternary_error_not_compensated": ("clip_grad(grad_at(grads, dtype, e), clip) + eps_old;",
                                      "clip_grad(grad_at(grads, dtype, e), clip) + 0.0f;"),
    "ternary_delta_sign": ("float delta = c - (float)q;", "float delta = (float)q - c;"),
    "ternary_error_is_delta": ("float eps_new = beta1 * eps_old + one_minus_b1 * delta;",
                               "float eps_new = delta;"),
    "ternary_server_first_worker_only": ("for (int32_t w = 0; w < W; ++w) sum += codes_w",
                                         "for (int32_t w = 0; w < 1; ++w) sum += codes_w"),
    "ternary_mean_not_divided": ("float g_hat = (float)codes_srv[4 * cw[k] + i] / (float)W;",
                                 "float g_hat = (float)codes_srv[4 * cw[k] + i];"),
    "ternary_code_word_base": ("cw[k + 1] = cw[k] + code_words_of(off[k + 1] - off[k]);",
                               "cw[k + 1] = cw[k] + (off[k + 1] - off[k]) / 4;"),
    "ternary_nan_check_dropped": ("if (is_nonfinite(eps_new)) flags |= ORC_STATUS_NONFINITE;", ""),
    "ternary_momentum_coeff": ("(float)W;\n      float mi = beta1 * m[o + i] + one_minus_b1 * g_hat;",
                               "(float)W;\n      float mi = one_minus_b1 * m[o + i] + beta1 * g_hat;"),
    "ternary_param_sign": ("\n        float pi = p[o + i] - lr * mi", "\n        float pi = p[o + i] + lr * mi", 0),
    # 2-bit Adam (a third entry: which occurrence of a shared statement is planted)
    "twobit_error_not_added": ("clip) + err_get(err, err_dtype, e0 + i);", "clip) + 0.0f;", 1),
    "twobit_server_sum_not_mean": ("float avg = acc / (float)W;", "float avg = acc;", 1),
    "twobit_server_error_dropped": ("c[i] = avg + err_get(srv_err, err_dtype, o + i);", "c[i] = avg;", 1),
    "twobit_server_first_worker_only": ("for (int32_t w = 0; w < W; ++w)\n        acc +=",
                                        "for (int32_t w = 0; w < 1; ++w)\n        acc +=", 1),
    "twobit_param_sign": ("\n        float pi = p[o + i] - lr * mi", "\n        float pi = p[o + i] + lr * mi", 1),
    "twobit_second_plane_of_c": ("  quantize_signs(r, nk, words + nw);", "  quantize_signs(c, nk, words + nw);"),
    "twobit_second_scale_of_c": ("  s[1] = quantize_scale(r, nk);", "  s[1] = quantize_scale(c, nk);"),
    "twobit_error_drops_first_plane": ("resid[i] = r[i] - dequantize(words + nw, s[1], i);",
                                       "resid[i] = c[i] - dequantize(words + nw, s[1], i);"),
    "twobit_dequantize_first_plane_only": ("return dequantize(words, s[0], i) + dequantize(words + nw, s[1], i);",
                                           "return dequantize(words, s[0], i);"),
    "twobit_second_plane_shifted": ("  quantize_signs(r, nk, words + nw);", "  quantize_signs(r, nk, words + nw - 1);"),
    "twobit_apply_word_step": ("    wo += 2 * nw;", "    wo += nw;"),
    # the quantisation rate
    "rates_count_padding": ("for (int64_t i = 0; i < nk; ++i) count += sign_bit(q, i);",
                            "for (int64_t i = 0; i < 32 * nw; ++i) count += sign_bit(q, i);"),
    "rates_plane_offset": ("const uint32_t* q = bits + base + pl * nw;", "const uint32_t* q = bits + base;"),
    "rates_divisor": ("(float)((double)count / (double)nk)", "(float)((double)count / (double)(32 * nw))"),
    "rates_row_stride": ("int64_t base = (int64_t)r * row_words;", "int64_t base = 0;"),
    # 0/1 Adam's local step
    "local_gradient_dropped": ("float kept = clip_grad(grad_at(grads, dtype, e), clip) + err_get(err, err_dtype, e);",
                               "float kept = 0.0f + err_get(err, err_dtype, e);"),
    "local_clip_ignored": ("float kept = clip_grad(grad_at(grads, dtype, e), clip) + err_get(err, err_dtype, e);",
                           "float kept = grad_at(grads, dtype, e) + err_get(err, err_dtype, e);"),
    "local_param_sign": ("float pi = p[o + i] - lr * m[o + i] / (sqrtf(v[o + i]) + eps);",
                         "float pi = p[o + i] + lr * m[o + i] / (sqrtf(v[o + i]) + eps);"),
    "local_lamb_skipped": ("      flags |= lamb_update_layer(p + o, m + o, v + o, lr, eps, nk);\n      continue;",
                           "      continue;"),
    "local_nan_not_flagged": ("if (is_nonfinite(kept)) flags |= ORC_STATUS_NONFINITE;", ""),
    "ternary_clip_after_error": ("float c = clip_grad(grad_at(grads, dtype, e), clip) + eps_old;",
                                 "float c = clip_grad(grad_at(grads, dtype, e) + eps_old, clip);"),
}


@pytest.fixture(scope="module")
def src_text():
    return open(SRC).read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, src_text, tmp_path):
    old, new, *nth = MUTANTS[name]
    if nth:       # a statement the oracle repeats: plant only its nth occurrence
        parts = src_text.split(old)
        assert len(parts) > nth[0] + 1, f"mutation anchor for {name} has no occurrence {nth[0]}"
        text = old.join(parts[: nth[0] + 1]) + new + old.join(parts[nth[0] + 1:])
    else:
        assert src_text.count(old) == 1, f"mutation anchor for {name} not unique/present"
        text = src_text.replace(old, new)
    mutated = tmp_path / "onebit_oracle.c"
    mutated.write_text(text)
    lib = oracle.build(force=True, src=str(mutated), out=str(tmp_path / f"lib_{name}.so"))
    o = oracle.Oracle(lib)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name!r} passed every pin"
