"""The oracle's pins must catch plausible mistakes.

Each case copies oracle/qknr_oracle.c, plants one mistake by a textual edit,
compiles the copy on the CPU, and runs the pins of test_oracle_pins.py against
it: at least one pin must fail. (The direction of the FP8 scale is a reading
the pages leave open, so no case flips it.)
"""
import os
import subprocess

import pytest

import oracle as O
from tests import test_oracle_pins as P

SRC = os.path.join(os.path.dirname(O.__file__), "qknr_oracle.c")

MUTATIONS = {
    "rotation_sign_a": ("out[pa[j]] = a * cos_t[j] - b * sin_t[j];",
                        "out[pa[j]] = a * cos_t[j] + b * sin_t[j];"),
    "rotation_sign_b": ("out[pb[j]] = b * cos_t[j] + a * sin_t[j];",
                        "out[pb[j]] = b * cos_t[j] - a * sin_t[j];"),
    "dropped_eps": ("sqrt(ssq / (double)n + eps)", "sqrt(ssq / (double)n)"),
    "mean_over_n_plus_1": ("sqrt(ssq / (double)n + eps)", "sqrt(ssq / (double)(n + 1) + eps)"),
    "per_head_norm_in_3d": (
        "qknr_oracle_rmsnorm(x, n, pass ? wk : wq, eps, y); /* across all H heads */",
        "for (int32_t hh = 0; hh < H; ++hh) qknr_oracle_rmsnorm(x + (int64_t)hh * D, D, "
        "(pass ? wk : wq) + (int64_t)hh * D, eps, y + (int64_t)hh * D);"),
    "weight_reversed": ("y[c] = x[c] * r * (weight ? weight[c] : 1.0);",
                        "y[c] = x[c] * r * (weight ? weight[n - 1 - c] : 1.0);"),
    "frequency_exponent_halved": ("pow(base, -2.0 * i / C[a])", "pow(base, -1.0 * i / C[a])"),
    "frequency_over_head_dim": ("pow(base, -2.0 * i / C[a])",
                                "pow(base, -2.0 * i / (C[0] + C[1] + C[2]))"),
    "axis_order_swapped": ("int64_t pos[3] = {f, h, w};", "int64_t pos[3] = {w, h, f};"),
    "position_height_index": ("*h = (s / ppw) % pph;", "*h = (s / pph) % ppw;"),
    "pos_offset_ignored": ("int64_t s = (t + pos_offset) % P;", "int64_t s = t % P;"),
    "per_axis_partner_mirrored": ("pb[off / 2 + i] = off + i + C[a] / 2;",
                                  "pb[off / 2 + i] = off + C[a] - 1 - i;"),
    "per_axis_flag_ignored": ("} else if (!neox_per_axis) {", "} else if (1) {"),
    "half_split_mirrored": ("pb[j] = interleaved ? 2 * j + 1 : j + rotary_dim / 2;",
                            "pb[j] = interleaved ? 2 * j + 1 : rotary_dim - 1 - j;"),
    "table_sin_column": ("s[j] = row[R / 2 + j];\n            } else {",
                         "s[j] = row[2 * j + 1];\n            } else {"),
    "bf16_ties_away": ("return fl + fmod(fl, 2.0);", "return fl + 1.0;"),
    "bf16_no_subnormal_floor": ("if (e < -126) e = -126;", ""),
    "e4m3_no_saturation": ("if (v > 448.0) v = 448.0;", ""),
    "e4m3_subnormal_floor": ("if (e < -6) e = -6;", "if (e < -7) e = -7;"),
    "v_uses_qk_scale": ("qknr_oracle_e4m3_from_double(ev[i] * v_scale)",
                        "qknr_oracle_e4m3_from_double(ev[i] * q_scale)"),
    "norm_flag_ignored": ("if (is_qk_norm)\n            qknr_oracle_rmsnorm",
                          "if (1)\n            qknr_oracle_rmsnorm"),
    "f16_exponent_bias": ("return s * ldexp(1.0 + m / 1024.0, e - 15);",
                          "return s * ldexp(1.0 + m / 1024.0, e - 16);"),
    "f16_no_subnormal_floor": ("if (e < -14) e = -14;", ""),
    "f16_overflow_early": ("if (v >= 65536.0) return (uint16_t)(sign | 0x7C00u);",
                           "if (v >= 65504.0) return (uint16_t)(sign | 0x7C00u);"),
    "act_type_ignored": ("return act_is_f16 ? qknr_oracle_f16_to_double(b) : qknr_oracle_bf16_to_double(b);",
                         "return qknr_oracle_bf16_to_double(b);"),
    "f16_nine_bit_significand": ("double quantum = ldexp(1.0, e - 10);",
                                 "double quantum = ldexp(1.0, e - 9);"),
    "f16_subnormal_unit": ("ldexp(1.0, -24)", "ldexp(1.0, -23)"),
    "f16_outputs_rounded_as_bf16": ("if (rc == 0 && act_is_f16) {", "if (rc == 0 && 0) {"),
    "f16_weights_read_as_bf16": ("wq[d] = act_to_double(q_weight[d], act_is_f16);",
                                 "wq[d] = act_to_double(q_weight[d], 0);"),
    "f16_table_read_as_bf16": ("c[j] = act_to_double(row[j], act_is_f16);",
                               "c[j] = act_to_double(row[j], 0);"),
    "ucpe_relu_dropped": ("y[i] = x[i] > 0.0 ? x[i] : 0.0;", "y[i] = x[i];"),
    "ucpe_relu_leaky": ("y[i] = x[i] > 0.0 ? x[i] : 0.0;", "y[i] = x[i] > 0.0 ? x[i] : 0.01 * x[i];"),
    "ucpe_projection_transposed": ("acc += m[4 * i + j] * x[b + j];",
                                   "acc += m[4 * j + i] * x[b + j];"),
    "ucpe_k_scale_dropped": ("for (int32_t d = 0; d < D; ++d) r[d] *= k_scale;", ""),
    "ucpe_v_through_relu": ("qknr_oracle_ray_project(mkv, x, D, y);",
                            "qknr_oracle_relu(x, D, r); qknr_oracle_ray_project(mkv, r, D, y);"),
    "ucpe_v_rotated": ("for (int32_t d = 0; d < D; ++d) v_out[out + (int64_t)d * N] = y[d];",
                       "qknr_oracle_rotate(y, D, D / 2, pa, pb, c, s, o); "
                       "for (int32_t d = 0; d < D; ++d) v_out[out + (int64_t)d * N] = o[d];"),
    "ucpe_q_takes_kv_matrix": ("qknr_oracle_ray_project(mq, r, D, y);",
                               "qknr_oracle_ray_project(mkv, r, D, y);"),
    "ucpe_half_split_pairs": ("qknr_oracle_pairs_table(D, 1, pa, pb); /* U4",
                              "qknr_oracle_pairs_table(D, 0, pa, pb); /* U4"),
    "ucpe_heads_batch_swapped": ("const int64_t out = (b * H + h) * D * N + n;",
                                 "const int64_t out = (h * B + b) * D * N + n;"),
    "ucpe_table_row_ignored": ("c[j] = rope_cos[n * (D / 2) + j];", "c[j] = rope_cos[j];"),
    "ucpe_matrix_of_first_token": ("mq[i] = proj_q[(b * N + n) * 16 + i];",
                                   "mq[i] = proj_q[(b * N) * 16 + i];"),
    "ucpe_inflation_inverted": ("before > 0.0 ? after / before : 1.0",
                                "before > 0.0 ? before / (after > 0.0 ? after : 1.0) : 1.0"),
    "ucpe_inflation_zero_key": ("before > 0.0 ? after / before : 1.0",
                                "before > 0.0 ? after / before : 0.0"),
    "ucpe_f16_outputs_as_bf16": ("act_is_f16 ? qknr_oracle_f16_from_double_array : "
                                 "qknr_oracle_bf16_from_double_array;",
                                 "qknr_oracle_bf16_from_double_array;"),
}

# cheap pins first, so a planted mistake is usually caught within a second
ORDER = sorted(P.ALL_PINS, key=lambda f: ("rounding_vs_torch" in f.__name__, f.__name__))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(so),
                    str(path), "-lm"], check=True)
    O.use_library(str(so))
    try:
        caught = []
        for pin in ORDER:
            try:
                pin()
            except (AssertionError, ValueError):
                caught.append(pin.__name__)
                break
        assert caught, f"no pin caught the planted mistake {name}"
    finally:
        O.use_library()
