"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks one oracle function against something the pages or the
mathematics fix: values the pages print, hand-worked cases, closed forms,
library routines (scipy's Sylvester construction) and brute force.  Every test
here runs on the CPU.
"""

import math

import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle as O
from hadamard_rotation_outlier_b200 import synthetic as S

POW2 = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024]


def _popcount_matrix(n):
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    bits = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(bits % 2 == 0, 1, -1).astype(np.int64)


# ---------------------------------------------------------------- H itself

@pytest.mark.parametrize("n", POW2)
def test_sylvester_equals_scipy_hadamard(n):
    # scipy.linalg.hadamard builds the same Sylvester matrix with +-1 entries.
    ref = scipy.linalg.hadamard(n).astype(np.float64) / math.sqrt(n)
    np.testing.assert_allclose(O.sylvester(n), ref, rtol=0, atol=1e-14)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 32, 128])
def test_sylvester_closed_form_popcount(n):
    # Textbook closed form: H[i, j] = (-1)^popcount(i & j) / sqrt(n).
    np.testing.assert_allclose(O.sylvester(n) * math.sqrt(n), _popcount_matrix(n),
                               rtol=0, atol=1e-12)


def test_h2_printed_and_h4_kronecker(golden_pages):
    h2 = np.array(golden_pages["h2_unnormalised"]).reshape(2, 2)
    np.testing.assert_allclose(O.sylvester(2) * math.sqrt(2), h2, atol=1e-15)
    # [Outlier nemesis] §2.1: H4 = H2 (x) H2
    np.testing.assert_allclose(O.sylvester(4), np.kron(O.sylvester(2), O.sylvester(2)),
                               atol=1e-15)


@pytest.mark.parametrize("n", [2, 4, 16, 64, 256])
def test_kronecker_recursion(n):
    np.testing.assert_allclose(O.sylvester(2 * n), np.kron(O.sylvester(2), O.sylvester(n)),
                               atol=1e-14)


@pytest.mark.parametrize("n", POW2 + [4096])
def test_orthogonal_symmetric_involution(n):
    H = O.sylvester(n)
    eye = np.eye(n)
    np.testing.assert_allclose(H @ H.T, eye, atol=1e-12)
    np.testing.assert_array_equal(H, H.T)
    np.testing.assert_allclose(H @ H, eye, atol=1e-12)
    np.testing.assert_allclose(np.abs(H), 1.0 / math.sqrt(n), rtol=1e-13)


def test_sylvester_rejects_non_power_of_two():
    for n in (0, 3, 6, 12, 11008):
        with pytest.raises(ValueError):
            O.sylvester(n)


# ------------------------------------------------------------------ FWHT

@pytest.mark.parametrize("n", POW2)
def test_fwht_brute_force_integers(n):
    # Brute force: y_j = sum_i x_i (-1)^popcount(i&j), exact in int64.
    rng = np.random.default_rng(n)
    x = rng.integers(-1000, 1000, size=(5, n))
    brute = x @ _popcount_matrix(n)
    got = O.fwht(x.astype(np.float64)) * math.sqrt(n)
    if round(math.sqrt(n)) ** 2 == n:
        # n = 4^k: sqrt(n) is a power of two, so every step is exact.
        np.testing.assert_array_equal(got, brute.astype(np.float64))
    else:
        np.testing.assert_allclose(got, brute, rtol=1e-13, atol=1e-9)


@pytest.mark.parametrize("n", [8, 128, 1024])
def test_fwht_matches_dense_product(n):
    x = np.random.default_rng(7).standard_normal((9, n))
    np.testing.assert_allclose(O.fwht(x), x @ O.sylvester(n), rtol=0, atol=1e-12)


def test_fwht_matches_dense_sampled_rows_4096():
    x = np.random.default_rng(8).standard_normal((3, 4096))
    np.testing.assert_allclose(O.fwht(x), x @ O.sylvester(4096), rtol=0, atol=1e-11)


# -------------------------------------------------------------- rotation

@pytest.mark.parametrize("method", ["dense", "fwht"])
def test_rotation_preserves_norm(method):
    x = np.random.default_rng(1).standard_normal((16, 512))
    for block in (-1, 128, 8):
        y = O.rotate(x, block=block, method=method)
        np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1),
                                   rtol=1e-13)


@pytest.mark.parametrize("method", ["dense", "fwht"])
def test_qk_scores_invariant(method):
    # [Hartmann rotation] §1: Q_rot K_rot^T == Q K^T because H is orthogonal.
    rng = np.random.default_rng(2)
    Q = rng.standard_normal((32, 128))
    K = rng.standard_normal((48, 128))
    Q[:, 7] *= 50.0
    K[:, 7] *= 50.0
    Qr = O.rotate(Q, method=method)
    Kr = O.rotate(K, method=method)
    np.testing.assert_allclose(Qr @ Kr.T, Q @ K.T, rtol=0, atol=1e-10 * np.abs(Q @ K.T).max())


def test_single_outlier_spreads_to_30_over_64(golden_pages):
    # [Outlier nemesis] §2.2: one 30 among 4096 -> ~0.47 everywhere; exactly 30/64.
    n = int(golden_pages["spread_example_dim"][0])
    x = np.zeros((1, n))
    x[0, 42] = golden_pages["spread_example_outlier"][0]
    for method in ("dense", "fwht"):
        y = O.rotate(x, method=method)
        np.testing.assert_allclose(np.abs(y), 30.0 / 64.0, rtol=1e-12)
        assert abs(30.0 / 64.0 - golden_pages["spread_example_magnitude_approx"][0]) < 0.005


@pytest.mark.parametrize("dim,B,p", [(512, 128, 300), (96, 32, 5), (4096, 128, 4095)])
def test_block_diagonal_one_hot_closed_form(dim, B, p):
    x = np.zeros((1, dim))
    x[0, p] = 1.0
    y = O.rotate(x, block=B)[0]
    b0 = (p // B) * B
    expect = np.zeros(dim)
    j = np.arange(B)
    bits = np.array([bin(int((p % B) & int(v))).count("1") for v in j])
    expect[b0:b0 + B] = np.where(bits % 2 == 0, 1.0, -1.0) / math.sqrt(B)
    np.testing.assert_allclose(y, expect, atol=1e-14)


def test_signs_apply_before_h_closed_form():
    # Randomised Hadamard = diag(s) then H: e_p -> s_p * H[p, :] (not s * H[p, :]).
    n = 64
    s = S.random_signs(n, 3)
    for p in (0, 5, 63):
        x = np.zeros((1, n))
        x[0, p] = 1.0
        y = O.rotate(x, signs=s)[0]
        np.testing.assert_allclose(y, s[p] * O.sylvester(n)[p], atol=1e-15)
    assert np.any(s < 0) and np.any(s > 0)


def test_hand_worked_rotations(golden_hand):
    g = golden_hand
    x = np.array([g["ex1_x"]])
    np.testing.assert_allclose(O.rotate(x)[0], g["ex1_y"], atol=1e-14)
    np.testing.assert_allclose(O.rotate(x, signs=np.array(g["ex2_signs"]))[0], g["ex2_y"],
                               atol=1e-14)
    x3 = np.array([g["ex3_x"]])
    np.testing.assert_allclose(O.rotate(x3, block=4)[0], g["ex3_block4_y"], atol=1e-14)
    np.testing.assert_allclose(O.rotate(x3)[0] * math.sqrt(8), g["ex3_full_y_times_sqrt8"],
                               atol=1e-13)


@pytest.mark.parametrize("method", ["dense", "fwht"])
def test_inverse_undoes_forward(method):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((6, 384))
    s = S.random_signs(384, 9)
    for block in (128, 64, 1):
        y = O.rotate(x, block=block, signs=s, method=method)
        np.testing.assert_allclose(O.inverse_rotate(y, block=block, signs=s, method=method), x,
                                   atol=1e-12)


# ------------------------------------------------------------- quantiser

def test_int8_scale_example_from_page(golden_pages):
    # [Hartmann rotation] §1: 200 among ~1 -> scale 200/127 ~ 1.57; small values -> +-1.
    y = np.array([[200.0, 1.0, -1.0, 0.9, -1.1, 1.05, -0.95, 1.0]])
    q, s64, s32, _ = O.quantize(y, 8, -1)
    assert s64[0, 0] == pytest.approx(golden_pages["int8_scale_example_absmax"][0] / 127.0,
                                      rel=1e-15)
    assert round(float(s64[0, 0]), 2) == golden_pages["int8_scale_example_scale_approx"][0]
    assert q[0, 0] == 127
    assert set(np.unique(q[0, 1:])) == set(int(v) for v in
                                           golden_pages["int8_scale_example_small_codes"])


def test_hand_worked_quantisation(golden_hand):
    g = golden_hand
    y = np.array([g["ex1_y"]])
    q, s64, s32, _ = O.quantize(y, 4, -1)
    np.testing.assert_array_equal(q[0], g["ex1_int4_q"])
    num, den = g["ex1_int4_scale_num_den"]
    assert s64[0, 0] == pytest.approx(num / den, rel=1e-15)
    assert s32[0, 0] == np.float32(num / den)
    q8, _, _, _ = O.quantize(y, 8, -1)
    np.testing.assert_array_equal(q8[0], g["ex1_int8_q"])
    np.testing.assert_array_equal(O.pack_int4(q)[0], g["ex1_int4_bytes"])
    q4, _, _, _ = O.quantize(np.array([g["ex4_y"]]), 4, -1)
    np.testing.assert_array_equal(q4[0], g["ex4_q"])


def test_hand_worked_end_to_end(golden_hand):
    """rotate_quantize on bf16 inputs against the hand-derived codes and bytes."""
    g = golden_hand

    def bits(vals):
        return S.f32_to_bf16_bits(np.array([vals], dtype=np.float32))

    r = O.rotate_quantize(bits(g["ex1_x"]), block=-1, bits=4)
    np.testing.assert_array_equal(r["codes"][0], g["ex1_int4_bytes"])
    r = O.rotate_quantize(bits(g["ex1_x"]), block=-1, signs=np.array(g["ex2_signs"], np.int8),
                          bits=4)
    np.testing.assert_array_equal(r["q"][0], g["ex2_int4_q"])
    np.testing.assert_array_equal(r["codes"][0], g["ex2_int4_bytes"])
    r = O.rotate_quantize(bits(g["ex1_x"]), block=-1, bits=8)
    np.testing.assert_array_equal(r["codes"][0], np.array(g["ex1_int8_q"], np.int8))
    r = O.rotate_quantize(bits(g["ex3_x"]), block=4, bits=4, group=4)
    np.testing.assert_array_equal(r["q"][0], g["ex3_block4_group4_q"])
    np.testing.assert_array_equal(r["codes"][0], g["ex3_block4_group4_bytes"])
    np.testing.assert_allclose(r["scales"][0], [5 / 7, 4 / 7], rtol=1e-7)
    r = O.rotate_quantize(bits(g["ex3_x"]), block=4, bits=4, group=-1)
    np.testing.assert_array_equal(r["q"][0], g["ex3_block4_rowgroup_q"])
    r = O.rotate_quantize(bits(g["ex3_x"]), block=-1, bits=8, group=-1)
    np.testing.assert_array_equal(r["q"][0], g["ex3_full_int8_q"])
    r = O.rotate_quantize(bits(g["ex4_y"]), block=1, bits=4)
    np.testing.assert_array_equal(r["q"][0], g["ex4_q"])


def test_hand_worked_dequant(golden_hand):
    g = golden_hand
    codes = np.array([g["ex1_int4_bytes"]], dtype=np.uint8)
    scales = np.array([[np.float32(5 / 7)]])
    xh = O.dequant_rotate_inv(codes, scales, 4, block=-1, bits=4)
    np.testing.assert_allclose(xh[0] * 14, g["ex1_int4_recon_times_14"], rtol=1e-7)
    codes = np.array([g["ex2_int4_bytes"]], dtype=np.uint8)
    xh = O.dequant_rotate_inv(codes, scales, 4, block=-1, bits=4,
                              signs=np.array(g["ex2_signs"], np.int8))
    # x*s had y = [-1,5,0,-2]; q = [-1,7,0,-3] -> yhat = [-5/7,5,0,-15/7]
    yh = np.array([-5 / 7, 5, 0, -15 / 7])
    expect = (yh @ (O.sylvester(4))) * np.array(g["ex2_signs"])
    np.testing.assert_allclose(xh[0], expect, rtol=1e-7)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("group", [-1, 16, 64])
def test_quantiser_bounds(bits, group):
    rng = np.random.default_rng(bits * 100 + group)
    y = rng.standard_normal((20, 128)) * rng.uniform(0.01, 100, size=(20, 1))
    q, s64, s32, v = O.quantize(y, bits, group)
    qmax = 2 ** (bits - 1) - 1
    G = 128 if group == -1 else group
    assert q.min() >= -qmax and q.max() <= qmax
    sg = np.repeat(s64, G, axis=1)
    # every value is within half a step of its reconstruction (no clipping ever happens)
    assert np.all(np.abs(y - q * sg) <= sg / 2 * (1 + 1e-12))
    # the largest |y| of each group maps to +-qmax
    yg = y.reshape(20, -1, G)
    qg = q.reshape(20, -1, G)
    idx = np.argmax(np.abs(yg), axis=-1)
    np.testing.assert_array_equal(np.abs(np.take_along_axis(qg, idx[..., None], -1)), qmax)
    # scales are per group, in column order
    np.testing.assert_allclose(s64, np.abs(yg).max(-1) / qmax, rtol=1e-15)


def test_group_order_and_zero_group():
    y = np.zeros((1, 24))
    y[0, 8:16] = np.linspace(-3, 2, 8)
    y[0, 16:24] = 70.0
    q, s64, s32, v = O.quantize(y, 8, 8)
    np.testing.assert_allclose(s64[0], [0.0, 3 / 127, 70 / 127])
    np.testing.assert_array_equal(q[0, :8], 0)
    np.testing.assert_array_equal(q[0, 16:], 127)
    assert q[0, 8] == -127 and np.all(v[0, :8] == 0)


def test_int4_pack_roundtrip_all_codes():
    q = np.array([np.arange(-7, 8), np.arange(7, -8, -1)]).T.reshape(1, -1)
    packed = O.pack_int4(q)
    assert packed.shape == (1, q.shape[1] // 2)
    np.testing.assert_array_equal(O.unpack_int4(packed), q)
    np.testing.assert_array_equal(O.pack_int4(np.array([[-1, 7, -7, 0]])), [[0x7F, 0x09]])


def test_reconstruction_error_bound():
    rng = np.random.default_rng(11)
    n = 256
    x_bits = S.random_bf16(8, n, 5, outlier_cols=[3, 200])
    for bits in (4, 8):
        r = O.rotate_quantize(x_bits, block=128, bits=bits, group=64)
        xh = O.dequant_rotate_inv(r["codes"], r["scales"], n, block=128, bits=bits, group=64)
        x = O.bf16_bits_to_f64(x_bits)
        smax = r["scales"].astype(np.float64).max(axis=1)
        err = np.linalg.norm(x - xh, axis=1)
        assert np.all(err <= math.sqrt(n) * smax / 2 * 1.0001)
    del rng


def test_rotated_error_far_below_unrotated(golden_pages):
    """[Outlier nemesis] §2.2 example, orthonormal H (the page's numbers are garbled)."""
    g = golden_pages
    rng = np.random.default_rng(int(g["error_example_seed"][0]))
    w = rng.standard_normal((1, 4096)).astype(np.float32)
    w[0, int(g["error_example_outlier_index"][0])] = g["error_example_outlier_value"][0]
    e0 = O.quant_error(w, 4)
    e1 = O.quant_error(O.rotate(w.astype(np.float64)), 4)
    assert e1 < e0 / 4
    e0_8 = O.quant_error(w, 8)
    e1_8 = O.quant_error(O.rotate(w.astype(np.float64)), 8)
    assert e1_8 < e0_8 / 4


def test_quant_error_definition_small():
    # hand: x = [2, -1, 0.5], INT4: scale = 2/7; x/scale = [7, -3.5, 1.75]
    # q = [7, -4, 2] (tie -3.5 -> -4, even); deq = [2, -8/7, 4/7]
    # |err| = [0, 1/7, 1/14] -> mean = (3/14)/3 = 1/14
    assert O.quant_error(np.array([2.0, -1.0, 0.5]), 4) == pytest.approx(1 / 14, rel=1e-12)


def test_bf16_decode(golden_hand):
    bits = np.array(golden_hand["bf16_bits"], dtype=np.uint16)
    np.testing.assert_array_equal(O.bf16_bits_to_f64(bits), golden_hand["bf16_values"])


def test_half_boundary_distance():
    v = np.array([0.5, 2.5001, -3.4999, 7.0, -0.0])
    np.testing.assert_allclose(O.half_boundary_distance(v), [0, 1e-4, 1e-4, 0.5, 0.5], atol=1e-9)


def test_planted_mistakes_are_caught(golden_hand):
    """A wrong sign, index or operand in a copy of the oracle fails the pins above."""
    g = golden_hand
    x = np.array([g["ex3_x"]])

    def rotate_sign_after(x, signs):  # signs after H instead of before
        return O.rotate(x) * signs

    s = np.array([1, -1, 1, -1, 1, -1, 1, -1])
    assert not np.allclose(rotate_sign_after(x, s), O.rotate(x, signs=s))

    def rotate_wrong_block_axis(x, B):  # blocks taken as strided columns
        n = x.shape[-1]
        xb = x.reshape(-1, B, n // B).transpose(0, 2, 1)
        return (xb @ O.sylvester(B)).transpose(0, 2, 1).reshape(x.shape)

    assert not np.allclose(rotate_wrong_block_axis(x, 4)[0], g["ex3_block4_y"])

    def unnormalised(x):
        return x @ (O.sylvester(4) * 2)

    assert not np.allclose(unnormalised(np.array([g["ex1_x"]]))[0], g["ex1_y"])


# ------------------------------------------------- decode attention over the KV cache

def _random_kv_codes(rng, nb, nkh, T, dim, bits, G):
    qmax = 2 ** (bits - 1) - 1
    q = rng.integers(-qmax, qmax + 1, size=(nb, nkh, T, dim))
    codes = q.astype(np.int8) if bits == 8 else O.pack_int4(q)
    scales = rng.uniform(0.01, 0.2, size=(nb, nkh, T, dim // G)).astype(np.float32)
    return q, codes, scales


def _scipy_unrotate(yrot, dim, B, signs):
    # x = (y @ H_B) * s with H_B from scipy's Sylvester construction.
    H = scipy.linalg.hadamard(B).astype(np.float64) / math.sqrt(B)
    x = (yrot.reshape(yrot.shape[:-1] + (dim // B, B)) @ H).reshape(yrot.shape)
    if signs is not None:
        x = x * np.where(np.asarray(signs) < 0, -1.0, 1.0)
    return x


@pytest.mark.parametrize("bits,G,B,with_signs", [(4, 128, 128, False), (8, 64, 128, True),
                                                 (4, 32, 64, True), (4, 128, -1, False)])
def test_decode_attention_matches_unrotated_attention(bits, G, B, with_signs):
    # Q_rot K_rot^T = Q K^T: the oracle's rotated-basis attention must equal
    # textbook attention on the un-rotated K, V (undone with scipy's H) and the
    # raw query, with scipy's softmax.  Consecutive query heads share a KV head.
    rng = np.random.default_rng(11 + bits + G)
    nb, nqh, nkh, T, dim = 2, 4, 2, 37, 128
    Bn = dim if B == -1 else B
    signs = S.random_signs(dim, 5) if with_signs else None
    qk, kc, ks = _random_kv_codes(rng, nb, nkh, T, dim, bits, G)
    qv, vc, vs = _random_kv_codes(rng, nb, nkh, T, dim, bits, G)
    qbits = S.f32_to_bf16_bits(rng.normal(size=(nb, nqh, dim)).astype(np.float32))
    got = O.kv_decode_attention(qbits, kc, ks, vc, vs, dim, B, signs, bits, G)

    def deq(qcodes, sc):
        return (qcodes.reshape(nb, nkh, T, dim // G, G) * sc.astype(np.float64)[..., None]
                ).reshape(nb, nkh, T, dim)

    K = _scipy_unrotate(deq(qk, ks), dim, Bn, signs)
    V = _scipy_unrotate(deq(qv, vs), dim, Bn, signs)
    x = O.bf16_bits_to_f64(qbits)
    want = np.empty((nb, nqh, dim))
    for b in range(nb):
        for h in range(nqh):
            kvh = h // (nqh // nkh)
            p = scipy.special.softmax(K[b, kvh] @ x[b, h] / math.sqrt(dim))
            want[b, h] = p @ V[b, kvh]
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_decode_attention_single_token_returns_its_value_row():
    # One cached token: softmax weight 1, output = that V row un-rotated.
    rng = np.random.default_rng(3)
    dim = 128
    qv, vc, vs = _random_kv_codes(rng, 1, 1, 1, dim, 4, 128)
    _, kc, ks = _random_kv_codes(rng, 1, 1, 1, dim, 4, 128)
    qbits = S.f32_to_bf16_bits(rng.normal(size=(1, 3, dim)).astype(np.float32))
    got = O.kv_decode_attention(qbits, kc, ks, vc, vs, dim, 128, None, 4, 128)
    row = _scipy_unrotate(qv[0, 0, 0] * np.float64(vs[0, 0, 0, 0]), dim, 128, None)
    for h in range(3):
        np.testing.assert_allclose(got[0, h], row, rtol=0, atol=1e-13)


def test_decode_attention_zero_query_averages_values():
    # q = 0: every score is 0, the weights are uniform, output = mean of V.
    rng = np.random.default_rng(4)
    dim, T = 64, 9
    qv, vc, vs = _random_kv_codes(rng, 1, 1, T, dim, 8, 32)
    _, kc, ks = _random_kv_codes(rng, 1, 1, T, dim, 8, 32)
    qbits = np.zeros((1, 1, dim), np.uint16)
    got = O.kv_decode_attention(qbits, kc, ks, vc, vs, dim, -1, None, 8, 32)
    deq = (qv.reshape(T, 2, 32) * vs.reshape(T, 2, 1).astype(np.float64)).reshape(T, dim)
    want = _scipy_unrotate(deq.mean(axis=0), dim, dim, None)
    np.testing.assert_allclose(got[0, 0], want, rtol=0, atol=1e-13)


def test_decode_attention_dominant_key_selects_its_value():
    # One key aligned with the (rotated) query and far larger than the rest:
    # its weight is 1 to within exp(-huge), so the output is its V row.
    dim, T, hot = 128, 16, 11
    H = scipy.linalg.hadamard(dim).astype(np.float64) / math.sqrt(dim)
    x = np.zeros(dim)
    x[0] = 1.0                              # rotated query = H[0] = all +1/sqrt(128)
    qk = np.zeros((1, 1, T, dim), np.int64)
    qk[0, 0, hot] = 7
    ks = np.full((1, 1, T, 1), 1.0, np.float32)
    qv = np.tile(np.arange(T)[:, None] % 15 - 7, (1, dim))[None, None]
    vs = np.full((1, 1, T, 1), 0.5, np.float32)
    qbits = S.f32_to_bf16_bits(x.astype(np.float32)[None, None])
    got = O.kv_decode_attention(qbits, O.pack_int4(qk), ks, O.pack_int4(qv), vs, dim, -1, None, 4,
                                -1, softmax_scale=1.0)
    want = (H @ (qv[0, 0, hot] * 0.5))       # inverse rotation of the hot V row
    np.testing.assert_allclose(got[0, 0], want, rtol=0, atol=1e-12)
    assert abs(got[0, 0].sum() - want.sum()) < 1e-12


def test_decode_attention_rejects_bad_head_ratio():
    rng = np.random.default_rng(5)
    _, kc, ks = _random_kv_codes(rng, 1, 2, 3, 64, 8, 64)
    qbits = np.zeros((1, 3, 64), np.uint16)
    with pytest.raises(ValueError):
        O.kv_decode_attention(qbits, kc, ks, kc, ks, 64, -1, None, 8, 64)


def test_decode_scores_equal_unrotated_dot_products():
    # The scores alone: rotated query against rotated keys = q . k / sqrt(d)
    # with the keys un-rotated through scipy's H.
    rng = np.random.default_rng(12)
    nb, nqh, nkv, T, dim = 1, 6, 3, 11, 64
    signs = S.random_signs(dim, 12)
    qk, kc, ks = _random_kv_codes(rng, nb, nkv, T, dim, 4, 32)
    qbits = S.f32_to_bf16_bits(rng.normal(size=(nb, nqh, dim)).astype(np.float32))
    got = O.kv_decode_scores(qbits, kc, ks, dim, 32, signs, 4, 32, softmax_scale=0.3)
    deq = (qk.reshape(nb, nkv, T, 2, 32) * ks.astype(np.float64)[..., None]).reshape(nb, nkv, T, dim)
    K = _scipy_unrotate(deq, dim, 32, signs)
    x = O.bf16_bits_to_f64(qbits)
    for h in range(nqh):
        np.testing.assert_allclose(got[0, h], 0.3 * K[0, h // 2] @ x[0, h], rtol=1e-12, atol=1e-12)


# ------------------------------------------------ mixed-precision (kept tokens) KV

def _keep_case(heads=3, tokens=11, dim=64, seed=21):
    x = S.random_bf16(heads * tokens, dim, seed, outlier_cols=[5], outlier_scale=30.0)
    slots = np.full(tokens, -1, np.int32)
    for rank, t in enumerate((0, 4, 9, 10)):        # a sink, a vertical line, a 2-token window
        slots[t] = rank
    return x, slots, 4


def test_keep_nothing_equals_plain_quantisation():
    x, _, _ = _keep_case()
    slots = np.full(11, -1, np.int32)
    r = O.rotate_quantize_keep(x, 3, 11, slots, 0, block=32, bits=4, group=16)
    p = O.rotate_quantize(x, block=32, bits=4, group=16)
    np.testing.assert_array_equal(r["codes"], p["codes"])
    np.testing.assert_array_equal(r["scales"], p["scales"])
    assert r["kept"].shape == (3, 0, 64)


def test_kept_rows_are_copied_bit_exactly_and_zeroed():
    x, slots, n_keep = _keep_case()
    r = O.rotate_quantize_keep(x, 3, 11, slots, n_keep, block=-1, bits=4, group=-1)
    p = O.rotate_quantize(x, block=-1, bits=4, group=-1)
    for h in range(3):
        for t in range(11):
            row = h * 11 + t
            if slots[t] >= 0:
                np.testing.assert_array_equal(r["kept"][h, slots[t]], x[row])
                assert not r["codes"][row].any() and r["scales"][row].item() == 0.0
            else:
                np.testing.assert_array_equal(r["codes"][row], p["codes"][row])
                assert r["scales"][row].item() == p["scales"][row].item()
    assert r["keep_row"].sum() == 3 * n_keep


def test_slots_outside_the_range_mean_quantise():
    x, slots, _ = _keep_case()
    bad = slots.copy()
    bad[4] = 4                       # n_keep = 4: out of range
    bad[9] = -7
    r = O.rotate_quantize_keep(x, 3, 11, bad, 4, bits=8)
    p = O.rotate_quantize(x, bits=8)
    for h in range(3):
        for t in (4, 9):
            np.testing.assert_array_equal(r["codes"][h * 11 + t], p["codes"][h * 11 + t])
    assert not r["kept"][:, 1].any() and not r["kept"][:, 2].any()   # slots 1, 2 unused


def test_mixed_cache_reads_back_kept_rows_exactly():
    x, slots, n_keep = _keep_case()
    signs = S.random_signs(64, 3)
    r = O.rotate_quantize_keep(x, 3, 11, slots, n_keep, block=64, signs=signs, bits=4, group=32)
    back = O.dequant_rotate_inv_keep(r["codes"], r["scales"], r["kept"], slots, n_keep, 3, 11, 64, block=64,
                                     signs=signs, bits=4, group=32)
    plain = O.dequant_rotate_inv(r["codes"], r["scales"], 64, block=64, signs=signs, bits=4, group=32)
    xf = O.bf16_bits_to_f64(x)
    for h in range(3):
        for t in range(11):
            row = h * 11 + t
            want = xf[row] if slots[t] >= 0 else plain[row]
            np.testing.assert_array_equal(back[row], want)
    # the quantised rows still reconstruct within the INT4 error bound
    q = ~r["keep_row"]
    assert np.max(np.abs(back[q] - xf[q])) < 0.5 * np.max(r["scales"]) * 8


# ------------------------------------------------------ asymmetric (zero-point) quantiser

def test_asym_hand_worked_group():
    # y = [-1, 0, 2, 3], 4 bits: lo = -1, hi = 3, scale = 4/15, zero point
    # round(3.75) = 4; codes round([-3.75, 0, 7.5, 11.25]) + 4 = [0, 4, 12, 15]
    # (7.5 rounds to the even 8).
    q, s64, _, zp, _, _ = O.quantize_asym(np.array([[-1.0, 0.0, 2.0, 3.0]]), 4, -1)
    assert s64[0] == 4 / 15 and zp[0] == 4
    np.testing.assert_array_equal(q[0], [0, 4, 12, 15])


@pytest.mark.parametrize("bits", [4, 8])
def test_asym_closed_forms(bits):
    qmax = 2 ** bits - 1
    rng = np.random.default_rng(bits)
    pos = np.abs(rng.normal(size=(3, 16))) + 0.1
    q, s64, _, zp, _, _ = O.quantize_asym(pos, bits, -1)
    assert np.all(zp == 0)                                    # all positive: lo = 0
    np.testing.assert_array_equal(q.max(axis=1), qmax)        # the maximum maps to the top code
    q, s64, _, zp, _, _ = O.quantize_asym(-pos, bits, -1)
    assert np.all(zp == qmax)                                 # all negative: hi = 0
    np.testing.assert_array_equal(q.min(axis=1), 0)
    # zeros are exact, and a zero group gets scale 0, codes 0
    y = np.concatenate([rng.normal(size=(2, 8)), np.zeros((2, 8))], axis=1)
    y[:, 3] = 0.0
    q, s64, s32, zp, _, _ = O.quantize_asym(y, bits, 8)
    assert np.all(q[:, 3] == zp[:, 0]) and np.all(s64[:, 1] == 0) and np.all(q[:, 8:] == 0)


@pytest.mark.parametrize("bits,G", [(4, 8), (4, 16), (8, 32)])
def test_asym_codes_are_the_nearest_grid_points(bits, G):
    # Brute force: the code is an argmin over all 2^b codes of |(k - zp) scale - y|.
    rng = np.random.default_rng(40 + bits + G)
    y = rng.standard_t(3, size=(6, 64))
    q, s64, _, zp, _, _ = O.quantize_asym(y, bits, G)
    k = np.arange(2 ** bits)
    yg, qg = y.reshape(6, -1, G), q.reshape(6, -1, G)
    for r in range(6):
        for g in range(64 // G):
            grid = (k - zp[r, g]) * s64[r, g]
            d = np.abs(grid[None, :] - yg[r, g][:, None])
            best = d.min(axis=1)
            np.testing.assert_allclose(d[np.arange(G), qg[r, g]], best, rtol=0, atol=1e-12)
            assert np.all(np.abs((qg[r, g] - zp[r, g]) * s64[r, g] - yg[r, g]) <= s64[r, g] / 2 + 1e-12)


def test_asym_uint4_pack_roundtrip():
    q = np.stack([np.arange(16), np.arange(16)[::-1]])
    b = O.pack_uint4(q)
    np.testing.assert_array_equal(O.unpack_uint4(b), q)
    assert b[0, 0] == 0x10 and b[0, 7] == 0xFE and b[1, 0] == 0xEF


def test_asym_rotate_quantize_and_back():
    x = S.random_bf16(5, 256, 8, outlier_cols=[3, 200], outlier_scale=50.0)
    signs = S.random_signs(256, 8)
    r = O.rotate_quantize_asym(x, block=128, signs=signs, bits=4, group=64)
    back = O.dequant_rotate_inv_asym(r["codes"], r["scales"], r["zero_points"], 256, block=128, signs=signs,
                                     bits=4, group=64)
    # error bound: each rotated value is off by at most scale/2, H orthonormal
    yerr = (r["q"].reshape(5, 4, 64) - r["zero_points"][..., None].astype(np.int64)) * \
        r["scales"][..., None].astype(np.float64) - r["rotated"].reshape(5, 4, 64)
    assert np.all(np.abs(yerr) <= r["scales"][..., None] / 2 * (1 + 1e-6))
    xf = O.bf16_bits_to_f64(x)
    assert np.linalg.norm(back - xf, axis=1).max() <= np.linalg.norm(yerr.reshape(5, 256), axis=1).max() + 1e-9


# -------------------------------------------------------------- Kronecker rotation

def _paley_hadamard(q):
    """Paley construction I (textbook): a Hadamard matrix of order q + 1 for a
    prime q = 3 (mod 4), from the quadratic-residue character of GF(q)."""
    res = {(i * i) % q for i in range(1, q)}
    chi = lambda v: 0 if v % q == 0 else (1 if v % q in res else -1)
    Q = np.array([[chi(j - i) for j in range(q)] for i in range(q)])
    S = np.zeros((q + 1, q + 1), dtype=np.int64)
    S[0, 1:] = 1
    S[1:, 0] = -1
    S[1:, 1:] = Q
    return S + np.eye(q + 1, dtype=np.int64)


@pytest.mark.parametrize("q", [3, 7, 11, 19])
def test_paley_matrix_is_hadamard(q):
    S = _paley_hadamard(q)
    n = q + 1
    assert set(np.unique(S)) == {-1, 1}
    np.testing.assert_array_equal(S @ S.T, n * np.eye(n, dtype=np.int64))


@pytest.mark.parametrize("a,b", [(1, 64), (2, 64), (4, 32), (8, 16)])
def test_kron_of_sylvester_factors_is_the_sylvester_block(a, b):
    # Sylvester H_a (x) H_b = H_ab (the Kronecker recursion): the Kronecker
    # rotation with a Sylvester factor is the block rotation of size a * b.
    x = S.random_bf16(3, a * b, a + b)
    xf = O.bf16_bits_to_f64(x)
    Fa = scipy.linalg.hadamard(a) / math.sqrt(a)
    got = O.kron_rotate(xf, Fa, b)
    want = xf @ (scipy.linalg.hadamard(a * b) / math.sqrt(a * b)).T
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_kron_matches_the_explicit_kronecker_matrix():
    # vec(F X H^T) = (F (x) H) vec(X), checked against numpy's kron.
    Fa = _paley_hadamard(11) / math.sqrt(12)
    b = 16
    x = S.random_bf16(4, 12 * b, 9, outlier_cols=[5], outlier_scale=40.0)
    signs = S.random_signs(12 * b, 9)
    xf = O.bf16_bits_to_f64(x)
    M = np.kron(Fa, scipy.linalg.hadamard(b) / math.sqrt(b))
    np.testing.assert_allclose(O.kron_rotate(xf, Fa, b, signs), (xf * np.where(signs < 0, -1, 1)) @ M.T,
                               rtol=0, atol=1e-12)
    y = O.kron_rotate(xf, Fa, b, signs)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(xf, axis=1), rtol=1e-13)
    np.testing.assert_allclose(O.kron_inverse_rotate(y, Fa, b, signs), xf, rtol=0, atol=1e-12)


def test_kron_quantise_and_back():
    Fa = _paley_hadamard(19) / math.sqrt(20)
    x = S.random_bf16(5, 20 * 32, 3, outlier_cols=[7, 300], outlier_scale=80.0)
    r = O.rotate_quantize_kron(x, Fa, 32, bits=4, group=32)
    p = O.quantize(r["rotated"], 4, 32)
    np.testing.assert_array_equal(r["q"], p[0])
    back = O.dequant_rotate_inv_kron(r["codes"], r["scales"], Fa, 32, bits=4, group=32)
    xf = O.bf16_bits_to_f64(x)
    err = np.linalg.norm(back - xf, axis=1)
    bound = np.sqrt(20 * 32) * 0.5 * r["scale64"].max(axis=1)
    assert np.all(err <= bound)
