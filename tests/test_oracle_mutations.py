"""Planted mistakes in the oracle (on the CPU): each plausible slip, compiled into a copy
of i8_oracle.c, must make at least one pin fail.  Shows the pins are not self-confirming."""
import os
import subprocess

import pytest

from oracle import oracle as O
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "i8_oracle.c")

# (name, exact text in the oracle, replacement)
MUTATIONS = [
    ("round_half_even", "float c = roundf(v);", "float c = rintf(v);"),
    ("truncate", "float c = roundf(v);", "float c = truncf(v);"),
    ("strict_threshold", ">= threshold)", "> threshold)"),
    ("scale_128", "float s = 127.0f / amax;", "float s = 128.0f / amax;"),
    ("absmax_includes_outliers",
     "            if (skip && skip[k])\n                continue;\n            float a",
     "            float a"),
    ("outlier_part_dropped", "out_part += (double)", "out_part += 0.0 * (double)"),
    ("recovery_over_128", "* (double)SCB[n] / 127.0;", "* (double)SCB[n] / 128.0;"),
    ("dequant_missing_weight_scale",
     "(double)acc[i * N + n] * (double)SCx[t] * (double)SCB[n]",
     "(double)acc[i * N + n] * (double)SCx[t]"),
    ("transposed_weight_index", "const int8_t *b = B + n * K;",
     "const int8_t *b = B + (n * K) % (K * N > 0 ? K : 1);"),
    ("bias_sign", "C[i * N + n] = int_part + out_part + b;",
     "C[i * N + n] = int_part + out_part - b;"),
    ("mask_bit_order", "mask_words[k / 32] |= (uint32_t)1 << (k % 32);",
     "mask_words[k / 32] |= (uint32_t)1 << (31 - k % 32);"),
    ("subnormal_decode", "v = ldexpf((float)f, -24);", "v = ldexpf((float)f, -25);"),
    # e4m3 variant
    ("e4m3_scale_447", "float s = 448.0f / amax;", "float s = 447.0f / amax;"),
    ("e4m3_ties_away", "double r = nearbyint(a / step) * step;",
     "double r = round(a / step) * step;"),
    ("e4m3_exponent_bias_8", "v = ldexp(1.0 + m / 8.0, e - 7);",
     "v = ldexp(1.0 + m / 8.0, e - 8);"),
    ("e4m3_two_fraction_bits", "double step = ldexp(1.0, E - 3);",
     "double step = ldexp(1.0, E - 2);"),
    ("e4m3_dequant_127", "/ (448.0 * 448.0);", "/ (448.0 * 127.0);"),
    ("e4m3_recovery_127", "(double)SCB[n] / 448.0;", "(double)SCB[n] / 127.0;"),
    ("e4m3_outlier_dropped", "out_part += (double)oracle_half_to_float(X[t * K + k]) * w;\n"
     "            }\n            double b = bias ? (double)oracle_half_to_float(bias[n]) : 0.0;\n"
     "            C[i * N + n] = main_part",
     "out_part += 0.0;\n"
     "            }\n            double b = bias ? (double)oracle_half_to_float(bias[n]) : 0.0;\n"
     "            C[i * N + n] = main_part"),
    ("e4m3_subnormal_binade", "    if (E < -6)\n        E = -6;", "    if (E < -7)\n        E = -7;"),
    ("e4m3_decode_subnormal", "v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    ("e4m3_saturate_below_448", "    if (a >= 448.0)\n        return sign | 0x7E;",
     "    if (a >= 416.0)\n        return sign | 0x7E;"),
    ("e4m3_outlier_codes_kept",
     "            if (skip && skip[k]) {\n                qr[k] = 0;\n                continue;\n"
     "            }\n            float v = oracle_half_to_float(row[k]) * s;\n            qr[k]",
     "            float v = oracle_half_to_float(row[k]) * s;\n            qr[k]"),
    ("e4m3_act_scale_row_index", "main_part = acc[i * N + n] * (double)SCx[t]",
     "main_part = acc[i * N + n] * (double)SCx[i]"),
    # scan, index list and half decode
    ("idx_descending",
     "    for (int64_t k = 0; k < K; ++k)\n        if (is_outlier[k])\n            idx[count++]",
     "    for (int64_t k = K - 1; k >= 0; --k)\n        if (is_outlier[k])\n            idx[count++]"),
    ("scan_first_row_only",
     "    for (int64_t t = 0; t < T; ++t)\n        for (int64_t k = 0; k < K; ++k)\n"
     "            if (fabsf",
     "    for (int64_t t = 0; t < 1; ++t)\n        for (int64_t k = 0; k < K; ++k)\n"
     "            if (fabsf"),
    ("scan_signed", "if (fabsf(oracle_half_to_float(X[t * K + k])) >= threshold)",
     "if (oracle_half_to_float(X[t * K + k]) >= threshold)"),
    ("half_exponent_bias_14", "v = ldexpf((float)(f + 1024), e - 25);",
     "v = ldexpf((float)(f + 1024), e - 24);"),
    # int8 quantiser
    ("outlier_codes_kept",
     "            if (skip && skip[k]) {\n                qr[k] = 0;\n                continue;\n"
     "            }\n            float v = oracle_half_to_float(row[k]) * s;\n            float c",
     "            float v = oracle_half_to_float(row[k]) * s;\n            float c"),
    ("weight_absmax_half_row",
     "        for (int64_t k = 0; k < K; ++k) {\n            if (skip && skip[k])\n"
     "                continue;\n            float a = fabsf(oracle_half_to_float(row[k]));\n"
     "            if (a > amax)\n                amax = a;\n        }\n"
     "        scale[r] = amax;\n        int8_t",
     "        for (int64_t k = 0; k < (skip ? K : K / 2); ++k) {\n            if (skip && skip[k])\n"
     "                continue;\n            float a = fabsf(oracle_half_to_float(row[k]));\n"
     "            if (a > amax)\n                amax = a;\n        }\n"
     "        scale[r] = amax;\n        int8_t"),
    ("clamp_126", "if (c > 127.0f) c = 127.0f;", "if (c > 126.0f) c = 126.0f;"),
    # product and output
    ("matmul_drops_last_k",
     "            for (int64_t k = 0; k < K; ++k)\n                s += (int64_t)a[k] * (int64_t)b[k];",
     "            for (int64_t k = 0; k + 1 < K; ++k)\n                s += (int64_t)a[k] * (int64_t)b[k];"),
    ("act_scale_row_index", "(double)acc[i * N + n] * (double)SCx[t] * (double)SCB[n]",
     "(double)acc[i * N + n] * (double)SCx[i] * (double)SCB[n]"),
    ("outlier_part_wrong_column",
     "out_part += (double)oracle_half_to_float(X[t * K + k]) * w;\n            }\n"
     "            double b = bias ? (double)oracle_half_to_float(bias[n]) : 0.0;\n"
     "            C[i * N + n] = int_part",
     "out_part += (double)oracle_half_to_float(X[t * K + j]) * w;\n            }\n"
     "            double b = bias ? (double)oracle_half_to_float(bias[n]) : 0.0;\n"
     "            C[i * N + n] = int_part"),
    ("dequant_single_127", "                              / (127.0 * 127.0);",
     "                              / (127.0);"),
    # training-mode backward and the recovered weight
    ("backward_dx_wrong_weight_entry",
     "(double)oracle_half_to_float(W[n * K + k]);\n                dX[t * K + k] = s;",
     "(double)oracle_half_to_float(W[(k * N + n) % (N * K)]);\n                dX[t * K + k] = s;"),
    ("backward_dw_drops_last_row",
     "                for (int64_t t = 0; t < T; ++t)\n                    s += (double)oracle_half_to_float(dY[t * N + n]) *\n"
     "                         (double)oracle_half_to_float(X[t * K + k]);",
     "                for (int64_t t = 0; t + 1 < T; ++t)\n                    s += (double)oracle_half_to_float(dY[t * N + n]) *\n"
     "                         (double)oracle_half_to_float(X[t * K + k]);"),
    ("bias_grad_every_other_row",
     "            for (int64_t t = 0; t < T; ++t)\n                s += (double)oracle_half_to_float(dY[t * N + n]);",
     "            for (int64_t t = 0; t < T; t += 2)\n                s += (double)oracle_half_to_float(dY[t * N + n]);"),
    ("recovered_weight_over_128", "const float s = SCB[n] / (e4m3 ? 448.0f : 127.0f);",
     "const float s = SCB[n] / (e4m3 ? 448.0f : 128.0f);"),
    ("bias_index_row",
     "double b = bias ? (double)oracle_half_to_float(bias[n]) : 0.0;\n"
     "            C[i * N + n] = int_part",
     "double b = bias ? (double)oracle_half_to_float(bias[i % N]) : 0.0;\n"
     "            C[i * N + n] = int_part"),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) >= 1, "mutation anchor not found: %s" % name
    mut = src.replace(old, new)
    c = tmp_path / ("%s.c" % name)
    so = tmp_path / ("lib%s.so" % name)
    c.write_text(mut, encoding="utf-8")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                           "-fPIC", "-shared", str(c), "-o", str(so), "-lm"])
    return str(so)


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    so = _build_mutant(tmp_path, name, old, new)
    failed = []
    with O.use_library(so):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except (AssertionError, OverflowError, ValueError, IndexError):
                failed.append(pin.__name__)
    assert failed, "no pin caught the planted mistake %r" % name
