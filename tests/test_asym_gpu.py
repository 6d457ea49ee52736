"""Parity of the asymmetric (zero-point) quantiser and its inverse with the
float64 oracle (rules in tests/parity.py: scales within 1e-5, zero points and
codes exact up to .5-boundary cases, reconstructions within 1e-5 of
max(|o|, row RMS), one bf16 ulp more for bf16 output)."""

import numpy as np
import pytest
import torch

import oracle as O
from hadamard_rotation_outlier_b200 import binding as B
from hadamard_rotation_outlier_b200 import synthetic as S
from hadamard_rotation_outlier_b200.steps import bf16_tensor_to_bits, bits_to_bf16_tensor

from parity import check_asym, check_bf16, check_values

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CASES = [
    # rows, dim, block, group, bits, signs, dist
    (300, 128, 128, 128, 4, False, "normal"),
    (77, 128, -1, -1, 8, True, "normal"),
    (40, 4096, 128, -1, 4, True, "normal"),
    (50, 512, 64, 256, 4, False, "student_t3"),
    (33, 256, 16, 128, 8, True, "student_t3"),
    (20, 1024, 32, 1024, 4, False, "normal"),
    (1, 128, 8, 128, 4, False, "normal"),
]


def _check_case(x_bits, dim, block, group, bits, signs, max_mismatches=None):
    dev = "cuda"
    rows = x_bits.shape[0]
    sg = None if signs is None else torch.from_numpy(signs).to(dev)
    x = bits_to_bf16_tensor(x_bits, dev)
    codes, scales, zp = B.hadq_rotate_quantize_asym(x, block=block, signs=sg, bits=bits, group=group)
    torch.cuda.synchronize()
    ref = O.rotate_quantize_asym(x_bits, block=block, signs=signs, bits=bits, group=group, method="fwht")
    c = codes.cpu().numpy()
    gq = c.astype(np.int64).reshape(rows, dim) if bits == 8 else O.unpack_uint4(c.reshape(rows, dim // 2))
    assert gq.min() >= 0 and gq.max() <= 2 ** bits - 1
    check_asym(gq, scales.cpu().numpy(), zp.cpu().numpy(), ref, bits, max_mismatches)
    want = O.dequant_rotate_inv_asym(c, scales.cpu().numpy(), zp.cpu().numpy(), dim, block=block, signs=signs,
                                     bits=bits, group=group, method="fwht")
    out = B.hadq_dequant_rotate_inv_asym(codes, scales, zp, dim, block=block, signs=sg, bits=bits, group=group,
                                         out_dtype=torch.float32)
    outb = B.hadq_dequant_rotate_inv_asym(codes, scales, zp, dim, block=block, signs=sg, bits=bits, group=group)
    torch.cuda.synchronize()
    check_values(out.cpu().numpy().reshape(rows, dim), want, "asym dequant f32")
    check_bf16(bf16_tensor_to_bits(outb).reshape(rows, dim), want, "asym dequant bf16")
    return ref, gq


@pytest.mark.parametrize("rows,dim,block,group,bits,with_signs,dist", CASES)
def test_asym_matches_oracle(rows, dim, block, group, bits, with_signs, dist):
    seed = rows + dim + bits
    x = S.random_bf16(rows, dim, seed, dist=dist, outlier_cols=[dim // 4], outlier_scale=60.0)
    signs = S.random_signs(dim, seed) if with_signs else None
    _check_case(x, dim, block, group, bits, signs)


def test_asym_edge_rows():
    # zero rows, one-signed rows, one-hot rows, tiny and subnormal magnitudes.
    # A one-hot row rotates to +-v: its zero point is exactly 15/2 and its
    # extreme codes sit exactly on ties, which float rounding breaks either
    # way, so its mismatches are not counted (each must still be a tie).
    dim = 128
    rng = np.random.default_rng(4)
    rows = [np.zeros(dim, np.float32),
            np.abs(rng.normal(size=dim)).astype(np.float32) + 0.5,
            -np.abs(rng.normal(size=dim)).astype(np.float32) - 0.5,
            np.eye(dim, dtype=np.float32)[5] * 3.0,
            (rng.normal(size=dim) * 1e-30).astype(np.float32),
            (rng.normal(size=dim) * 1e-40).astype(np.float32)]
    x = S.f32_to_bf16_bits(np.stack(rows))
    for block, bits in ((8, 4), (32, 8), (128, 4)):
        ref, gq = _check_case(x, dim, block, 128, bits, None, max_mismatches=dim)
        assert not gq[0].any()   # a zero row: scale 0, zero point 0, codes 0


def test_exact_ties_round_half_even():
    # 8-point blocks where the unnormalised transform is exact and the
    # multiplier 15 / range is exact in float32, so the ties are exact (the
    # float64 oracle, which divides by sqrt(8), lands a rounding error off
    # them, hence the hand-derived expectations):
    #  x = [2, 1, 1, 0, ...] -> v = [4, 2, 2, 0] x 2: lo 0, hi 4, codes 4 * 3.75 = 15
    #    and 2 * 3.75 = 7.5 -> 8 (half to even);
    #  x = [0, 5, 0, ...] -> v = [5, -5] x 4: zero point 5 * 1.5 = 7.5 -> 8, codes
    #    7.5 -> 8, + 8 -> 16 clamped to 15, and -7.5 -> -8, + 8 = 0.
    dim = 128
    a = np.zeros((2, dim), np.float32)
    a[0].reshape(16, 8)[:, :3] = [2, 1, 1]
    a[1].reshape(16, 8)[:, 1] = 5
    x = bits_to_bf16_tensor(S.f32_to_bf16_bits(a), "cuda")
    codes, scales, zp = B.hadq_rotate_quantize_asym(x, block=8, bits=4, group=128)
    torch.cuda.synchronize()
    gq = O.unpack_uint4(codes.cpu().numpy())
    np.testing.assert_array_equal(gq[0], np.tile([15, 8, 8, 0], 32))
    np.testing.assert_array_equal(gq[1], np.tile([15, 0], 64))
    np.testing.assert_array_equal(zp.cpu().numpy().ravel(), [0, 8])
    np.testing.assert_allclose(scales.cpu().numpy().ravel(), [4 / np.sqrt(8) / 15, 10 / np.sqrt(8) / 15],
                               rtol=1e-6)


def test_full_size_kv_cache_asym_sampled():
    wl = S.WORKLOADS["c4_kv_h8_t131072_d128_int4_g128"]
    x = S.tensor(wl, 0)
    dev = "cuda"
    codes, scales, zp = B.hadq_rotate_quantize_asym(bits_to_bf16_tensor(x, dev), block=128, bits=4, group=128)
    torch.cuda.synchronize()
    rng = np.random.default_rng(8)
    rows = np.unique(np.concatenate([[0, len(x) - 1], rng.integers(0, len(x), size=60)]))
    idx = torch.from_numpy(rows).to(dev)
    ref = O.rotate_quantize_asym(x[rows], block=128, bits=4, group=128, method="fwht")
    gq = O.unpack_uint4(codes.index_select(0, idx).cpu().numpy())
    check_asym(gq, scales.index_select(0, idx).cpu().numpy(), zp.index_select(0, idx).cpu().numpy(), ref, 4)
    assert torch.all(scales > 0)
