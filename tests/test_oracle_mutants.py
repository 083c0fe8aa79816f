"""The pins catch plausible slips in the oracle.

Each case copies the oracle's C source, plants one slip (a wrong rounding, a
dropped term, a flipped sign, an off-by-one index, a wrong tie-break),
builds it, and runs tests/test_oracle_pins.py against that copy in a child
process.  The pins must fail for every mutant.  Nothing here touches a GPU.
"""
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sq_oracle.c")

MUTANTS = {
    "round_floor_half_up": ("double r = round(t);", "double r = floor(t + 0.5);"),
    "scale_divides_by_128": ("return (float)(a / 127.0);", "return (float)(a / 128.0);"),
    "clip_to_minus_128": ("if (r < -127.0)\n        r = -127.0;", "if (r < -128.0)\n        r = -128.0;"),
    "sign_of_zero_negative": ("(uint8_t)(w[j] >= 0.0f)", "(uint8_t)(w[j] > 0.0f)"),
    "residual_adds_trunk": ("t = sign[row * K + j] ? (double)a : -(double)a;",
                            "t = sign[row * K + j] ? -(double)a : (double)a;"),
    "alpha_over_all_entries": ("            if (mask[row * K + j]) {\n                sum +=",
                               "            if (1) {\n                sum +="),
    "threshold_not_strict": ("(fabsf(w[j]) > tau)", "(fabsf(w[j]) >= tau)"),
    "percentile_rank_off_by_one": ("((int64_t)P * K + 99) / 100", "((int64_t)P * K) / 100 + 1"),
    "group_drops_last_channel": ("int64_t j1 = j0 + G < K ? j0 + G : K;",
                                 "int64_t j1 = j0 + G < K ? j0 + G - 1 : K;"),
    "act_absmax_includes_outliers": ("if (!is_out[j] && fabs((double)v[j]) > a)",
                                     "if (fabs((double)v[j]) > a)"),
    "outlier_term_dropped": ("out += dequant_weight(sign, mask, alpha, q, s, K, ng, G, r, idx[i]) *",
                             "out += 0.0 * dequant_weight(sign, mask, alpha, q, s, K, ng, G, r, idx[i]) *"),
    "outlier_weight_without_residual": ("return t + (double)s[r * ng + j / G] * (double)q[r * K + j];",
                                        "return t;"),
    "calibration_ties_to_higher_index": ("(best < 0 || mag[j] > mag[best])",
                                         "(best < 0 || mag[j] >= mag[best])"),
    "popcount_sign_plane_positive": ("int64_t c = p < 7 ? ((int64_t)1 << p) : -128;",
                                     "int64_t c = p < 7 ? ((int64_t)1 << p) : 128;"),
    "trunk_scale_missing": ("double inner = (double)alpha[r] * (double)T[t * N + r];",
                            "double inner = (double)T[t * N + r];"),
    "group_scale_index_shifted": ("inner += (double)s[r * ng + g] * (double)R[(t * N + r) * ng + g];",
                                  "inner += (double)s[r * ng + (g + 1) % ng] * (double)R[(t * N + r) * ng + g];"),
    "trunk_only_ignores_mask": ("                if (mask[r * K + j])\n                    T +=",
                                "                if (1)\n                    T +="),
    "trunk_only_sign_flipped": ("T += (sign[r * K + j] ? 1 : -1) * (int64_t)xq[t * K + j];",
                                "T += (sign[r * K + j] ? -1 : 1) * (int64_t)xq[t * K + j];"),
    "trunk_only_outliers_dropped": ("out += wt * (double)xout[t * n_out + i];",
                                    "out += 0.0 * wt * (double)xout[t * n_out + i];"),
    "trunk_only_outlier_weight_unmasked": ("double wt = mask[r * K + j] ? (sign[r * K + j]",
                                           "double wt = 1 ? (sign[r * K + j]"),
    "trunk_only_scale_missing": ("double out = (double)sx[t] * ((double)alpha[r] * (double)T);",
                                 "double out = (double)alpha[r] * (double)T;"),
    "sparse_keeps_ties": ("keep[j] = (uint8_t)(fabs(r[j]) > theta);",
                          "keep[j] = (uint8_t)(fabs(r[j]) >= theta);"),
    "sparse_rank_floor_plus_one": ("int64_t rank = ((int64_t)Ps * K + 99) / 100;",
                                   "int64_t rank = ((int64_t)Ps * K) / 100 + 1;"),
    "sparse_quantizes_dropped_entries": ("kept[j] = keep[j] ? r[j] : 0.0;", "kept[j] = r[j];"),
    "sparse_theta_next_rank": ("theta = a[rank - 1];", "theta = a[rank < K ? rank : K - 1];"),
    "asym_group_drops_last_channel": ("int64_t j1 = K < j0 + G ? K : j0 + G;",
                                      "int64_t j1 = K < j0 + G ? K : j0 + G - 1;"),
    "asym_zero_point_floor": ("z[g] = (int32_t)round(-lo / sd - 128.0);",
                              "z[g] = (int32_t)floor(-lo / sd - 128.0);"),
    "asym_zero_point_sign": ("z[g] = (int32_t)round(-lo / sd - 128.0);",
                             "z[g] = (int32_t)round(lo / sd - 128.0);"),
    "asym_range_254": ("s[g] = (float)((hi - lo) / 255.0);", "s[g] = (float)((hi - lo) / 254.0);"),
    "asym_clip_minus_127": ("            if (v < -128.0)\n                v = -128.0;",
                            "            if (v < -127.0)\n                v = -127.0;"),
    "asym_linear_drops_zero_point": ("(double)(R - (int64_t)z[r * ng + g] * S);", "(double)R;"),
    "asym_outlier_weight_drops_zero_point": ("(double)((int64_t)q[r * K + j] - z[r * ng + g]);",
                                             "(double)q[r * K + j];"),
    "abs_dot_drops_fabs": ("acc += fabs((double)W[r * K + j] * (double)x[t * K + j]);",
                           "acc += (double)W[r * K + j] * (double)x[t * K + j];"),
    "abs_dot_doubles_term": ("acc += fabs((double)W[r * K + j] * (double)x[t * K + j]);",
                             "acc += 2.0 * fabs((double)W[r * K + j] * (double)x[t * K + j]);"),
    "abs_dot_transposes_output": ("out[t * N + r] = acc;", "out[r * M + t] = acc;"),
    "layer_error_not_squared": ("            e += d * d;\n        }\n        total += e;\n    }\n    *err = total;\n    return SQO_OK;\n}\n\nint sqo_plain_sq_error",
                                "            e += fabs(d);\n        }\n        total += e;\n    }\n    *err = total;\n    return SQO_OK;\n}\n\nint sqo_plain_sq_error"),
    "layer_error_drops_zero_point": ("int64_t zz = z ? (int64_t)z[r * ng + g] : 0;", "int64_t zz = 0;"),
    "layer_error_trunk_sign_flipped": ("double t = mask[r * K + j] ? (sign[r * K + j] ? (double)alpha[r] : -(double)alpha[r]) : 0.0;\n            int64_t zz",
                                       "double t = mask[r * K + j] ? (sign[r * K + j] ? -(double)alpha[r] : (double)alpha[r]) : 0.0;\n            int64_t zz"),
    "plain_error_without_quantizer_clip": ("double d = w - (double)sg * (double)sqo_quantize(w, sg);",
                                           "double d = w - (double)sg * round(w / (double)sg * 1.001);"),
    "e2m1_ties_to_odd": ("if (dc < db || (dc == db && (c & 1) == 0))",
                         "if (dc < db || (dc == db && (c & 1) == 1))"),
    "e2m1_negative_zero": ("    if (best == 0)\n        return 0;\n    return v < 0.0",
                           "    return v < 0.0"),
    "ue4m3_bias_8": ("return ldexp(1.0 + (double)m / 8.0, e - 7);",
                     "return ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "ue4m3_ties_away": ("if (dc < db || (dc == db && c % 2 == 0))", "if (dc <= db)"),
    "nvfp4_scale_without_six": ("sqo_ue4m3_round(ab / (6.0 * gr))", "sqo_ue4m3_round(ab / gr)"),
    "nvfp4_tensor_scale_448": ("g[0] = (float)(amax_all / 2688.0);", "g[0] = (float)(amax_all / 448.0);"),
    "nvfp4_row_scale_448": ("g[r] = (float)(a / 2688.0);", "g[r] = (float)(a / 448.0);"),
    "nvfp4_block_drops_last": ("int64_t j0 = 16 * b, j1 = j0 + 16 < K ? j0 + 16 : K;",
                               "int64_t j0 = 16 * b, j1 = j0 + 15 < K ? j0 + 15 : K;"),
    "nvfp4_linear_drops_weight_scale": ("                           (double)gw;", "                           1.0;"),
    "nvfp4_linear_token_scale_of_row": ("                           (double)gx[t];",
                                        "                           (double)gx[0];"),
}


def _build_mutant(tmp, name, old, new):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"{name}: pattern must occur exactly once"
    d = os.path.join(tmp, name)
    os.makedirs(d)
    shutil.copy(os.path.join(ROOT, "oracle", "sq_oracle.h"), d)
    with open(os.path.join(d, "sq_oracle.c"), "w", encoding="utf-8") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(d, "libmutant.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", lib, os.path.join(d, "sq_oracle.c"), "-lm"])
    return lib


def test_every_mutant_is_caught():
    tmp = tempfile.mkdtemp(prefix="sq_mutants_")
    try:
        procs = {}
        for name, (old, new) in MUTANTS.items():
            lib = _build_mutant(tmp, name, old, new)
            env = dict(os.environ, SQ_ORACLE_LIB=lib)
            procs[name] = subprocess.Popen(
                [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                 os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                cwd=ROOT, env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
        survivors = []
        for name, p in procs.items():
            out, _ = p.communicate(timeout=600)
            if p.returncode == 0:
                survivors.append(name)
        assert not survivors, f"mutants not caught by the pins: {survivors}"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def test_unmutated_copy_passes():
    """Control: the same harness with no slip planted passes."""
    tmp = tempfile.mkdtemp(prefix="sq_control_")
    try:
        lib = _build_mutant(tmp, "control", "#include <math.h>", "#include <math.h>")
        env = dict(os.environ, SQ_ORACLE_LIB=lib)
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout[-2000:]
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
