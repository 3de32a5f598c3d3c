"""The oracle pins catch plausible mistakes.

Each case copies the oracle sources to a temporary folder, plants one mistake
(a dropped term, a wrong sign or index, a transposed operand, a wrong rounding
tie, a missing check), builds the copy and runs the pin tests against it in a
subprocess. The pins must fail for every planted mistake. The real oracle is
never modified.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle")

MUTATIONS = {
    "padding_digit_0": ("oref_format_a.c",
                        "(j < G) ? (t[j] + 1) : 1;", "(j < G) ? (t[j] + 1) : 0;"),
    "digit_order_msb_first": ("oref_format_a.c",
                              "int32_t j = 5 * m + i;\n      int digit",
                              "int32_t j = 5 * m + (4 - i);\n      int digit"),
    "ties_away_from_zero": ("oref_format_a.c",
                            "if (fabs(v[j]) > half)", "if (fabs(v[j]) >= half)"),
    "dropped_abs_in_mean": ("oref_format_a.c",
                            "sum += fabs(v[j]);", "sum += v[j];"),
    "mean_divides_by_g_minus_1": ("oref_format_a.c",
                                  "sum / (double)G;", "sum / (double)(G - 1);"),
    "no_zero_scale_rule": ("oref_format_a.c", "if (s != 0.0) {", "if (1) {"),
    "residual_sign": ("oref_format_a.c", "v[j] - s * (double)t[j]",
                      "v[j] + s * (double)t[j]"),
    "second_plane_reads_first": ("oref_format_a.c",
                                 "p * plane_groups + r * gpr + g;",
                                 "r * gpr + g;"),
    "x_index_transposed_A": ("oref_format_a.c",
                             "acc += w[j] * oref_bf16_to_f64(xb[j]);",
                             "acc += w[j] * oref_bf16_to_f64(xb[k - 1 - j]);"),
    "missing_243_check": ("oref_format_a.c", "if (b >= 243) status",
                          "if (b > 243) status"),
    "missing_padding_check": ("oref_format_a.c", "} else if (digit != 1) {",
                              "} else if (digit > 2) {"),
    "lut_ladder_reversed": ("oref_format_b.c", "(double)ladder[i];",
                            "(double)ladder[4 - i];"),
    "lut_digit_sign": ("oref_format_b.c", "int c = rest % 3 - 1;",
                       "int c = 1 - rest % 3;"),
    "rho_row_index": ("oref_format_b.c",
                      "double scale = (rps > 0) ? oref_f16_to_f64(rho[r / rps]) : 1.0;\n    const float *L = row_lut(lut, lut_rows, r);\n    for (int64_t j = 0; j < k; ++j) {\n      uint8_t c = codes[r * k + j];\n      if (c >= 243 && status == OREF_OK) status = OREF_ERR_BAD_CODE;\n      w_out",
                      "double scale = (rps > 0) ? oref_f16_to_f64(rho[r % rps]) : 1.0;\n    const float *L = row_lut(lut, lut_rows, r);\n    for (int64_t j = 0; j < k; ++j) {\n      uint8_t c = codes[r * k + j];\n      if (c >= 243 && status == OREF_OK) status = OREF_ERR_BAD_CODE;\n      w_out"),
    "dropped_rho_in_matmul": ("oref_format_b.c",
                              "w_out[i * k + j] = scale * (double)L[c];",
                              "w_out[i * k + j] = (double)L[c];"),
    "lut_block_index_off_by_one_row": ("oref_format_b.c",
                                       "lut + 256 * (r / lut_rows)",
                                       "lut + 256 * ((r + 1) / lut_rows)"),
    "lut_block_ignored": ("oref_format_b.c",
                          "return lut_rows > 0 ? lut + 256 * (r / lut_rows) : lut;",
                          "return lut;"),
    "encode_tie_to_nonzero": ("oref_format_b.c",
                              "if (fabsf(rn) < ar) {", "if (fabsf(rn) <= ar) {"),
    "encode_zero_bias_ignored": ("oref_format_b.c",
                                 "if (!(ar < zs[i])) {", "if (1) {"),
    "encode_residual_not_updated": ("oref_format_b.c",
                                    "          r = rn;\n", "\n"),
    "encode_digit_order_reversed": ("oref_format_b.c",
                                    "code += (c + 1) * p3;",
                                    "code += (c + 1) * (81 / p3);"),
    "encode_rho_inverted": ("oref_format_b.c",
                            "oref_f64_to_f16((double)a / (double)alpha)",
                            "oref_f64_to_f16((double)alpha / (double)a)"),
    "encode_global_scale_for_rows": ("oref_format_b.c",
                                     "      a = (float)gmax;",
                                     "      a = alpha;"),
    "experts_hot_prefix_off_by_one": ("oref_format_a.c",
                                      "const double wj = e < n_hot ?",
                                      "const double wj = e <= n_hot ?"),
    "experts_ignore_expert_id": ("oref_format_a.c",
                                 "int s = oref_weights_A(codes1 + e * cstride,",
                                 "int s = oref_weights_A(codes1,"),
    "experts_drop_second_plane": ("oref_format_a.c",
                                  "? w1[j] + w2[j] : w1[j];", "? w1[j] : w1[j];"),
    "pack7_bits_msb_first": ("oref_format_b.c",
                             "const int pos = 7 * j + bit;\n            out[pos / 8]",
                             "const int pos = 7 * j + (6 - bit);\n            out[pos / 8]"),
    "pack7_pad_word_zero": ("oref_format_b.c",
                            "for (int i = count; i < 128; ++i) used[i] = 121;",
                            "for (int i = count; i < 128; ++i) used[i] = 0;"),
    "unpack7_index_off_by_one": ("oref_format_b.c",
                                 "codes[r * k + 16 * ch + j] = used[idx];",
                                 "codes[r * k + 16 * ch + j] = used[(idx + 1) & 127];"),
    "round_ties_up": ("oref_fp.c",
                      "return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;",
                      "return f + 1.0;"),
    "subnormal_spacing": ("oref_fp.c", "const int emin = 1 - bias;",
                          "const int emin = -bias;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    fname, old, new = MUTATIONS[name]
    src = tmp_path / "src"
    shutil.copytree(ORACLE, src, ignore=shutil.ignore_patterns(
        "*.so", "__pycache__"))
    path = src / fname
    text = path.read_text()
    assert text.count(old) >= 1, f"mutation anchor not found: {name}"
    path.write_text(text.replace(old, new, 1))
    sys.path.insert(0, ORACLE)
    try:
        import build as oracle_build  # noqa: E402  (oracle/build.py)
    finally:
        sys.path.pop(0)
    lib = oracle_build.build(out=str(tmp_path / "liboref_mut.so"),
                             extra_flags=("-Wno-error",), src_dir=str(src))
    env = dict(os.environ, OREF_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q",
                        "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode != 0, f"pins did not catch mutation {name}"
