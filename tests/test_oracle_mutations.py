"""Shows the oracle pins are sharp: each plausible mistake, planted in a
temporary copy of the oracle (CPU only), makes tests/test_oracle_pins.py fail.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "scale_divisor_8": ("float s = amax / seven;", "float s = amax / 8.0f;"),
    "round_half_away": ("float r = nearbyintf(quot);", "float r = roundf(quot);"),
    "nibble_order_swapped": ("    int shift = ((i % ORACLE_GROUP) % 2) ? 4 : 0;\n    packed[b]",
                             "    int shift = ((i % ORACLE_GROUP) % 2) ? 0 : 4;\n    packed[b]"),
    "query_rotated_by_transpose": ("acc += Q[(int64_t)i * d + j] * qv[j];",
                                   "acc += Q[(int64_t)j * d + i] * qv[j];"),
    "output_not_inverse_rotated": ("acc += O[(int64_t)j * d + i] * orot[i];",
                                   "acc += O[(int64_t)i * d + j] * orot[i];"),
    "signs_applied_after_hadamard": ("* (double)signs[j];", "* (double)signs[i];"),
    "append_leaves_rotation_off": ("n_new, d, pos, R, R, k_packed", "n_new, d, pos, NULL, NULL, k_packed"),
    "value_scale_wrong_group": ("(double)sv[i / ORACLE_GROUP] * (double)codes[i]",
                                "(double)sv[0] * (double)codes[i]"),
    "gqa_map_modulo": ("hk = hq / G;\n    int64_t T = ctx_lens[b];\n    double qv[512], qr[512], orot[512];\n    int8_t codes",
                       "hk = hq % Hkv;\n    int64_t T = ctx_lens[b];\n    double qv[512], qr[512], orot[512];\n    int8_t codes"),
    "cb_gqa_map_modulo": ("hk = hq / G;\n    int64_t T = ctx_lens[b];\n    double qv[512], qr[512], orot[512];\n    uint8_t ci",
                          "hk = hq % Hkv;\n    int64_t T = ctx_lens[b];\n    double qv[512], qr[512], orot[512];\n    uint8_t ci"),
    "missing_softmax_normalizer": ("double p = S[t] / Z;\n      for (int i = 0; i < d; ++i) orot[i] += p * ((double)sv[i / ORACLE_GROUP] * (double)codes[i]);",
                                   "double p = S[t];\n      for (int i = 0; i < d; ++i) orot[i] += p * ((double)sv[i / ORACLE_GROUP] * (double)codes[i]);"),
    "byte_index_group_stride": ("+ 2 * g + (j % 4) / 2;", "+ g + (j % 4) / 2;"),
    "hartley_cos_minus_sin": ("return (cos(th) + sin(th)) / sqrt((double)d);",
                              "return (cos(th) - sin(th)) / sqrt((double)d);"),
    "hartley_unnormalized": ("return (cos(th) + sin(th)) / sqrt((double)d);",
                             "return (cos(th) + sin(th)) / (double)d;"),
    "srft_sign_on_output_index": ("if (signs) v *= (double)signs[j];",
                                  "if (signs) v *= (double)signs[k];"),
    "srft_lambda_on_input_index": ("if (lambda) v *= (double)lambda[k];",
                                   "if (lambda) v *= (double)lambda[j];"),
    "srft_query_times_lambda": ("f * sj / (lambda_k ? (double)lambda_k[k] : 1.0);",
                                "f * sj * (lambda_k ? (double)lambda_k[k] : 1.0);"),
    "srft_output_without_lambda": ("sj * f / (lambda_v ? (double)lambda_v[k] : 1.0);", "sj * f;"),
    "srft_output_sign_index": ("O[(int64_t)j * d + k] = sj", "O[(int64_t)j * d + k] = (signs ? (double)signs[k] : 1.0)"),
    "cb_tie_goes_up": ("if (u > t[i]) ++k;", "if (u >= t[i]) ++k;"),
    "cb_sample_std": ("float sigma = (float)sqrt(S / (double)ORACLE_GROUP);",
                      "float sigma = (float)sqrt(S / (double)(ORACLE_GROUP - 1));"),
    "cb_clip_at_two": ("if (u > 3.0f) u = 3.0f;", "if (u > 2.0f) u = 2.0f;"),
    "cb_bit_order_reversed": ("|= (uint8_t)(1u << (bit % 8));", "|= (uint8_t)(1u << (7 - bit % 8));"),
    "lloyd_cell_mean_sign": ("double m = (pa - pb) / (cb - ca);", "double m = (pb - pa) / (cb - ca);"),
    "cb_value_scale_wrong_group": ("(double)sv[i / ORACLE_GROUP] * (double)C[ci[i]]",
                                   "(double)sv[0] * (double)C[ci[i]]"),
    "uniform_divisor_m_plus_1": ("float s = amax / top;", "float s = amax / (top + 1.0f);"),
    "uniform_round_half_away": ("float rq = nearbyintf(uq);", "float rq = roundf(uq);"),
    "uniform_clamp_below_m": ("if (rq > (float)m) rq = (float)m;", "if (rq > (float)(m - 1)) rq = (float)(m - 1);"),
    "uniform_twos_complement_index": ("idx[g * ORACLE_GROUP + j] = (uint8_t)(c + m);",
                                      "idx[g * ORACLE_GROUP + j] = (uint8_t)(c & ((1 << bits) - 1));"),
    "uniform_levels_shifted": ("levels[u] = (float)(u - m);", "levels[u] = (float)(u - m - 1);"),
    # mistakes that only show with levels that are not symmetric about zero
    "cb_threshold_assumes_symmetric": ("volatile float sum = C[i] + C[i + 1];",
                                       "volatile float sum = C[i] - C[L - 2 - i];"),
    "cb_score_level_mirrored": ("(double)sk[i / ORACLE_GROUP] * (double)C[ci[i]]",
                                "(double)sk[i / ORACLE_GROUP] * -(double)C[(1 << bits) - 1 - ci[i]]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    (tmp_path / "oracle").mkdir()
    (tmp_path / "oracle" / "oracle.c").write_text(src.replace(old, new))
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), tmp_path / "oracle" / "__init__.py")
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), tmp_path / "tests" / "golden")
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), tmp_path / "tests" / f)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=tmp_path, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 1 and "failed" in r.stdout, r.stdout[-2000:]
