"""Plant one plausible mistake at a time in a copy of the oracle (on the CPU)
and check that the pins in tests/test_oracle.py catch every one of them."""
from __future__ import annotations

import subprocess

import pytest

from oracle import oracle as orc
from tests import test_oracle as pins

# (name, exact text in oracle.c, replacement)
MUTATIONS = [
    ("relu_dropped", "double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    ("relu_wrong_side", "double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot < 0.0 ? dot : 0.0;"),
    ("weight_sign", "acc += wt[h] * relu;", "acc -= wt[h] * relu;"),
    ("sigma_dropped", "*I_out = sigma * acc;", "*I_out = acc;"),
    ("q_transposed", "double p = qd[h * ORC_DIM + d] * kd[d];",
     "double p = qd[d * heads + h] * kd[d];"),
    ("weight_index", "wt[h] = (double)weights[t * heads + h];",
     "wt[h] = (double)weights[t * heads + (h + 1) % heads];"),
    ("first_key_dropped", "for (int64_t s = ks[t]; s < ke[t]; ++s) {",
     "for (int64_t s = ks[t] + 1; s < ke[t]; ++s) {"),
    ("error_scale_signed", "err += fabs(wt[h]) * absdot;", "err += wt[h] * absdot;"),
    ("tie_to_larger_index", "return (x->i < y->i) ? -1 : (x->i > y->i) ? 1 : 0;",
     "return (x->i > y->i) ? -1 : (x->i < y->i) ? 1 : 0;"),
    ("ascending_order", "if (x->v > y->v)\n            return -1;", "if (x->v < y->v)\n            return -1;"),
    ("e4m3_bias", "mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);",
     "mag = ldexp(1.0 + (double)m / 8.0, (int)e - 8);"),
    ("e4m3_subnormal", "mag = ldexp((double)m / 8.0, -6);", "mag = ldexp((double)m / 8.0, -7);"),
    ("bf16_shift", "uint32_t w = (uint32_t)(bits & 0xFFFFu) << 16;",
     "uint32_t w = (uint32_t)(bits & 0xFFFFu) << 15;"),
    ("padding_index", "out_idx[j] = j < n ? buf[j].i : -1;", "out_idx[j] = j < n ? buf[j].i : 0;"),
    ("short_window_loses_one", "int64_t n = L < k ? L : k;", "int64_t n = L < k ? L - 1 : k;"),
    ("bound_negative_weight_uses_upper", "ub += wt[h] * (L > 0.0 ? L : 0.0);",
     "ub += wt[h] * (U > 0.0 ? U : 0.0);"),
    ("bound_upper_takes_min", "U += x > y ? x : y;", "U += x < y ? x : y;"),
    ("bound_sigma_dropped", "double v = sigma * element(dtype, kv, s * ORC_DIM + d);",
     "double v = element(dtype, kv, s * ORC_DIM + d);"),
    ("bound_last_key_dropped", "for (int64_t s = b * block; s < S && s < (b + 1) * block; ++s) {",
     "for (int64_t s = b * block; s < S && s < (b + 1) * block - 1; ++s) {"),
    ("last_head_dropped", "for (int h = 0; h < heads; ++h) {\n        double dot = 0.0, absdot = 0.0;",
     "for (int h = 0; h < heads - 1; ++h) {\n        double dot = 0.0, absdot = 0.0;"),
    ("q_row_stride_of_32_heads",
     "qd[i] = element(dtype, q, t * heads * ORC_DIM + i);\n        for (int h = 0; h < heads; ++h)\n"
     "            wt[h] = (double)weights",
     "qd[i] = element(dtype, q, t * 32 * ORC_DIM + i);\n        for (int h = 0; h < heads; ++h)\n"
     "            wt[h] = (double)weights"),
    ("weight_row_stride_of_32_heads", "wt[h] = (double)weights[t * heads + h];",
     "wt[h] = (double)weights[t * 32 + h];"),
    ("bound_scale_smaller_side",
     "(fabs(bh[d]) > fabs(bl[d]) ? fabs(bh[d]) : fabs(bl[d]))",
     "(fabs(bh[d]) < fabs(bl[d]) ? fabs(bh[d]) : fabs(bl[d]))"),
]

CHECKS = [
    pins.check_e4m3_table,
    pins.check_bf16_table,
    lambda: pins.check_score_equal_heads_matmul("fp8"),
    lambda: pins.check_score_equal_heads_matmul("bf16"),
    lambda: pins.check_score_one_hot_heads("fp8"),
    lambda: pins.check_score_one_hot_heads("bf16"),
    lambda: pins.check_score_linear_in_weights("fp8"),
    lambda: pins.check_score_single_head("fp8"),
    lambda: pins.check_score_heads_split("bf16"),
    pins.check_score_head_permutation,
    pins.check_score_homogeneity,
    pins.check_hand_example,
    pins.check_select_brute_force,
    pins.check_select_all_equal,
    pins.check_select_torch_topk_tie_free,
    pins.check_select_signed_zero,
    pins.check_topk_rows_brute_force,
    pins.check_topk_rows_torch_tie_free,
    pins.check_fused_all_equal,
    lambda: pins.check_bound_dominates_scores("fp8"),
    lambda: pins.check_bound_one_key_blocks("bf16"),
    pins.check_bound_hand_example,
]


def _build_mutant(tmp_path, old, new):
    src = open(orc.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    path = tmp_path / "oracle_mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(so), str(path), "-lm"])
    return str(so)


def test_pins_pass_on_the_real_oracle():
    for chk in CHECKS:
        chk()


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    so = _build_mutant(tmp_path, old, new)
    caught = []
    with orc.use_library(so):
        for chk in CHECKS:
            try:
                chk()
            except AssertionError:
                caught.append(chk)
                break
    assert caught, f"no pin catches the planted mistake {name}"
