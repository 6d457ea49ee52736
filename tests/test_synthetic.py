"""Seeded input generators: determinism, row-range regeneration, recipes."""

import numpy as np

import oracle as O
from hadamard_rotation_outlier_b200 import synthetic as S


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 lies halfway between bf16 1.0 and 1.0078125 -> even (1.0);
    # 1 + 3*2^-8 lies halfway between 1.0078125 and 1.015625 -> even (1.015625).
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -200.0, 0.0], dtype=np.float32)
    got = O.bf16_bits_to_f64(S.f32_to_bf16_bits(x))
    np.testing.assert_array_equal(got, [1.0, 1.015625, -200.0, 0.0])


def test_row_ranges_regenerate_identically():
    wl = S.WORKLOADS["c4_kv_h8_t131072_d128_int4_g128"].with_rows(8 * 1000)
    full = S.tensor(wl, 0)
    part = S.tensor_rows(wl, 0, 300, 2100)
    np.testing.assert_array_equal(full[300:2100], part)
    np.testing.assert_array_equal(S.tensor(wl, 0), full)


def test_outlier_recipe_c2_shared_by_q_and_k():
    wl = S.WORKLOADS["c2_qk_h32_s8192_d128_int8"]
    cq = S.outlier_columns(wl.tensors[0], wl.dim)
    ck = S.outlier_columns(wl.tensors[1], wl.dim)
    assert cq.shape == (32, 2)
    np.testing.assert_array_equal(cq, ck)
    x = O.bf16_bits_to_f64(S.tensor_rows(wl, 0, 0, 512))
    mean_abs = np.abs(x).mean(0)
    assert set(np.argsort(mean_abs)[-2:]) == set(cq[0])


def test_workload_byte_counts():
    wl = S.WORKLOADS
    assert wl["c1_tok256_h4096_b128_int4"].quant_bytes() == 2_622_464
    assert wl["c2_qk_h32_s8192_d128_int8"].quant_bytes() == 203_423_744
    assert wl["c3_tok16384_h4096_full_signs_int4"].quant_bytes() == 167_837_696
    assert wl["c4_kv_h8_t131072_d128_int4_g128"].quant_bytes() == 679_477_248
    assert wl["c4_kv_h8_t131072_d128_int4_g128"].dequant_bytes(2) == 679_477_248
    assert wl["c5_tok32768_w11008_b128_signs_int4_g128"].quant_bytes() == 913_047_552
    # the mixed-precision variant adds the int32 keep table and 196 kept bf16 rows per head (16 heads)
    k = wl["c4k_kv_h8_t131072_d128_int4_g128_keep196"]
    assert (k.heads, k.tokens, k.n_keep) == (16, 131072, 196)
    assert k.quant_bytes() == 679_477_248 + 4 * 131072 + 2 * 16 * 196 * 128
    assert k.dequant_bytes(2) == k.quant_bytes()


def test_vertical_tokens_seeded_and_in_range():
    a = S.vertical_tokens(1000, 20, 3, 4, 100)
    np.testing.assert_array_equal(a, S.vertical_tokens(1000, 20, 3, 4, 100))
    assert len(set(a)) == 20 and a.min() >= 4 and a.max() < 900 and np.all(np.diff(a) > 0)


def test_signs_are_pm1():
    s = S.signs(S.WORKLOADS["c3_tok16384_h4096_full_signs_int4"])
    assert s.dtype == np.int8 and set(np.unique(s)) == {-1, 1}
    assert S.signs(S.WORKLOADS["c1_tok256_h4096_b128_int4"]) is None
