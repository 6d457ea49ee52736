"""Parity of the Kronecker rotation + quantiser (F (x) H_b) and its inverse
with the float64 oracle (rules of tests/parity.py)."""

import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as O
from hadamard_rotation_outlier_b200 import binding as B
from hadamard_rotation_outlier_b200 import synthetic as S
from hadamard_rotation_outlier_b200.steps import bf16_tensor_to_bits, bits_to_bf16_tensor

from parity import check_bf16, check_codes, check_scales, check_values, gpu_codes_to_int

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def factor(kind, a, seed=0):
    if kind == "sylvester":
        return scipy.linalg.hadamard(a) / math.sqrt(a)
    if kind == "paley":
        return S.paley_hadamard(a - 1).astype(np.float64) / math.sqrt(a)
    q, _ = np.linalg.qr(np.random.default_rng(seed).normal(size=(a, a)))   # any orthogonal factor
    return q


CASES = [
    # rows, factor kind, a, b, bits, group, signs
    (40, "sylvester", 4, 64, 4, 128, False),
    (33, "paley", 12, 32, 8, 64, True),
    (64, "paley", 20, 256, 4, 128, True),
    (17, "sylvester", 1, 128, 8, -1, False),
    (20, "paley", 24, 16, 4, 32, False),
    (9, "orthogonal", 7, 32, 8, 56, True),
    (6, "paley", 108, 64, 4, 64, True),
    # tensor-core variant (a <= 32, a * b a multiple of 512): every K / N
    # padding (ceil(a / 8) = 1 .. 4), both code widths, one-lane and
    # whole-warp sub-blocks
    (50, "sylvester", 8, 64, 4, 64, False),
    (40, "orthogonal", 16, 32, 8, 32, True),
    (30, "orthogonal", 28, 256, 4, 128, True),
    (20, "orthogonal", 32, 128, 8, 256, False),
    (33, "orthogonal", 3, 512, 4, 512, True),
    (17, "sylvester", 1, 512, 8, -1, False),
    (9, "paley", 12, 128, 4, 16, True),
]

# the kernel variant each case runs (hadq_kron_plan), asserted below so the
# cases keep covering all three
VARIANTS = ["reg16", "reg16", "mma", "reg16", "reg16", "smem", "reg16",
            "mma", "mma", "mma", "mma", "mma", "mma", "mma"]


def test_cases_cover_every_variant():
    got = [B.hadq_kron_plan(0, rows, a, b, bits, group) for rows, _, a, b, bits, group, _ in CASES]
    assert got == VARIANTS


@pytest.mark.parametrize("rows,kind,a,b,bits,group,with_signs", CASES)
def test_kron_matches_oracle(rows, kind, a, b, bits, group, with_signs):
    dim = a * b
    seed = rows + a + b
    x = S.random_bf16(rows, dim, seed, outlier_cols=[dim // 3, 5], outlier_scale=80.0)
    signs = S.random_signs(dim, seed) if with_signs else None
    F = factor(kind, a, seed)
    dev = "cuda"
    fa = torch.from_numpy(F.astype(np.float32)).to(dev)
    sg = None if signs is None else torch.from_numpy(signs).to(dev)
    rot = torch.empty((rows, dim), dtype=torch.float32, device=dev)
    codes, scales = B.hadq_rotate_quantize_kron(bits_to_bf16_tensor(x, dev), fa, b, signs=sg, bits=bits,
                                                group=group, rotated_out=rot)
    torch.cuda.synchronize()
    F32 = F.astype(np.float32).astype(np.float64)           # the factor the kernel used
    ref = O.rotate_quantize_kron(x, F32, b, signs, bits, group)
    check_values(rot.cpu().numpy(), ref["rotated"], "rotated")
    check_scales(scales.cpu().numpy(), ref["scales"])
    check_codes(gpu_codes_to_int(codes.cpu().numpy(), bits, dim), ref["q"], ref["pre_round"])
    want = O.dequant_rotate_inv_kron(codes.cpu().numpy(), scales.cpu().numpy(), F32, b, signs, bits, group)
    out = B.hadq_dequant_rotate_inv_kron(codes, scales, fa, b, signs=sg, bits=bits, group=group,
                                         out_dtype=torch.float32)
    outb = B.hadq_dequant_rotate_inv_kron(codes, scales, fa, b, signs=sg, bits=bits, group=group)
    torch.cuda.synchronize()
    check_values(out.cpu().numpy(), want, "inverse f32")
    check_bf16(bf16_tensor_to_bits(outb), want, "inverse bf16")


def test_sylvester_factor_equals_the_block_rotation():
    # H_4 (x) H_64 = H_256: the Kronecker kernel and the block kernel agree.
    x = S.random_bf16(50, 256, 2, outlier_cols=[9], outlier_scale=50.0)
    xt = bits_to_bf16_tensor(x, "cuda")
    fa = torch.from_numpy((scipy.linalg.hadamard(4) / 2.0).astype(np.float32)).cuda()
    ya = torch.empty((50, 256), dtype=torch.float32, device="cuda")
    yb = torch.empty_like(ya)
    B.hadq_rotate_quantize_kron(xt, fa, 64, bits=8, rotated_out=ya)
    B.hadq_rotate_quantize(xt, block=256, bits=8, rotated_out=yb)
    torch.cuda.synchronize()
    ref = O.rotate(O.bf16_bits_to_f64(x), block=256)
    check_values(ya.cpu().numpy(), ref, "kron")
    check_values(yb.cpu().numpy(), ref, "block")


def test_kron_rejections():
    fa = torch.eye(4, device="cuda")
    x = torch.zeros((2, 5 * 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):                    # 320 columns != 4 * 64
        B.hadq_rotate_quantize_kron(x, fa, 64)
    big = torch.eye(256, device="cuda")
    xb = torch.zeros((1, 256 * 128), dtype=torch.bfloat16, device="cuda")
    n0 = B.hadq_launch_count()
    with pytest.raises(B.HadqError) as e:              # 256 KB of coefficients alone
        B.hadq_rotate_quantize_kron(xb, big, 128)
    assert e.value.status == B.HADQ_ERR_UNSUPPORTED and "shared memory" in str(e.value)
    assert B.hadq_launch_count() == n0


def _edge_rows(dim, rng):
    rows = [np.zeros(dim, np.float32),
            np.eye(dim, dtype=np.float32)[dim // 3] * 3.0,
            (rng.normal(size=dim) * 1e-30).astype(np.float32),
            (rng.normal(size=dim) * 1e30).astype(np.float32),
            np.where(rng.random(dim) < 0.01, 1e4, rng.normal(size=dim)).astype(np.float32)]
    return S.f32_to_bf16_bits(np.stack(rows))


def _run_and_check(x, F, b, bits, group, what):
    dev = "cuda"
    fa = torch.from_numpy(F.astype(np.float32)).to(dev)
    rows, dim = x.shape
    rot = torch.empty((rows, dim), dtype=torch.float32, device=dev)
    codes, scales = B.hadq_rotate_quantize_kron(bits_to_bf16_tensor(x, dev), fa, b, bits=bits, group=group,
                                                rotated_out=rot)
    torch.cuda.synchronize()
    ref = O.rotate_quantize_kron(x, F.astype(np.float32).astype(np.float64), b, None, bits, group)
    check_values(rot.cpu().numpy(), ref["rotated"], what + " rotated")
    check_scales(scales.cpu().numpy(), ref["scales"])
    check_codes(gpu_codes_to_int(codes.cpu().numpy(), bits, dim), ref["q"], ref["pre_round"], max_mismatches=dim)
    return ref


@pytest.mark.parametrize("a,b", [(20, 256), (8, 64), (32, 16)])
def test_edge_rows(a, b):
    # zero, one-hot, tiny (1e-30), huge (1e30) and spiky rows
    x = _edge_rows(a * b, np.random.default_rng(a + b))
    _run_and_check(x, factor("orthogonal", a, 3), b, 4, 128 if b >= 128 else 64, f"edge a={a} b={b}")


def test_subnormal_rows():
    # rows made only of bf16 subnormals (|x| < 2^-126)
    a, b = 20, 256
    rng = np.random.default_rng(11)
    v = (rng.normal(size=(3, a * b)) * 1e-39).astype(np.float32)
    x = S.f32_to_bf16_bits(v)
    _run_and_check(x, factor("orthogonal", a, 4), b, 4, 128, "subnormal")


@pytest.mark.parametrize("a,b", [(20, 256), (12, 128)])
def test_constant_row_closed_form(a, b):
    # x = c everywhere: F X = c s 1^T with s_r = sum_i F[r][i], and the
    # normalised H_b maps a constant row to sqrt(b) c s_r at column 0 and to
    # exact zeros elsewhere.  (A float64 matrix product leaves rounding noise
    # in those zeros, so this row is checked against the closed form.)
    F = factor("orthogonal", a, 5).astype(np.float32)
    c = -2.5
    x = S.f32_to_bf16_bits(np.full((2, a * b), c, np.float32))
    dev = "cuda"
    rot = torch.empty((2, a * b), dtype=torch.float32, device=dev)
    codes, scales = B.hadq_rotate_quantize_kron(bits_to_bf16_tensor(x, dev), torch.from_numpy(F).to(dev), b,
                                                bits=4, group=128, rotated_out=rot)
    torch.cuda.synchronize()
    y0 = math.sqrt(b) * c * F.astype(np.float64).sum(axis=1)            # [a]
    got = rot.cpu().numpy().reshape(2, a, b).astype(np.float64)
    np.testing.assert_allclose(got[:, :, 0], np.broadcast_to(y0, (2, a)), rtol=1e-5)
    rest = np.abs(got[:, :, 1:]).max(axis=-1)
    assert np.all(rest <= 1e-6 * np.abs(y0)), rest.max()
    sc = scales.cpu().numpy().reshape(2, a, b // 128).astype(np.float64)
    np.testing.assert_allclose(sc[:, :, 0], np.broadcast_to(np.abs(y0) / 7, (2, a)), rtol=1e-5)
    q = gpu_codes_to_int(codes.cpu().numpy(), 4, a * b).reshape(2, a, b)
    np.testing.assert_array_equal(q[:, :, 0], np.broadcast_to(np.sign(y0) * 7, (2, a)))
    assert not q[:, :, 1:128].any()


def pm1_matrix(a):
    """A +-1 Hadamard matrix of order a: Paley when a - 1 is a prime = 3 mod 4,
    else Sylvester."""
    q = a - 1
    if q >= 3 and q % 4 == 3 and all(q % d for d in range(2, int(q ** 0.5) + 1)):
        return S.paley_hadamard(q)
    return scipy.linalg.hadamard(a).astype(np.int8)


PM1_CASES = [
    # rows, a, b, bits, group, signs, variant
    (64, 20, 256, 4, 128, True, "mma"),
    (50, 8, 64, 8, 64, True, "mma"),
    (30, 12, 128, 4, 128, False, "mma"),
    (21, 32, 16, 4, 64, True, "mma"),
    (40, 4, 64, 4, 128, False, "reg16"),
    (20, 24, 16, 4, 32, False, "reg16"),
    (6, 108, 64, 4, 64, True, "reg16"),
    (9, 20, 32, 8, 40, True, "smem"),
]


@pytest.mark.parametrize("rows,a,b,bits,group,with_signs,variant", PM1_CASES)
def test_pm1_factor_matches_oracle(rows, a, b, bits, group, with_signs, variant):
    # the factor given as the stored +-1 matrix: F = S_a / sqrt(a), exactly
    assert B.hadq_kron_plan(0, rows, a, b, bits, group) == variant
    dim = a * b
    seed = 3 * rows + a + b
    x = S.random_bf16(rows, dim, seed, outlier_cols=[dim // 5, 1], outlier_scale=70.0)
    signs = S.random_signs(dim, seed) if with_signs else None
    Sa = pm1_matrix(a)
    assert np.array_equal(Sa.astype(np.int64) @ Sa.T.astype(np.int64), a * np.eye(a, dtype=np.int64))
    F = Sa.astype(np.float64) / math.sqrt(a)
    dev = "cuda"
    sa = torch.from_numpy(np.ascontiguousarray(Sa)).to(dev)
    sg = None if signs is None else torch.from_numpy(signs).to(dev)
    rot = torch.empty((rows, dim), dtype=torch.float32, device=dev)
    codes, scales = B.hadq_rotate_quantize_kron_pm1(bits_to_bf16_tensor(x, dev), sa, b, signs=sg, bits=bits,
                                                    group=group, rotated_out=rot)
    torch.cuda.synchronize()
    ref = O.rotate_quantize_kron(x, F, b, signs, bits, group)
    check_values(rot.cpu().numpy(), ref["rotated"], "rotated")
    check_scales(scales.cpu().numpy(), ref["scales"])
    check_codes(gpu_codes_to_int(codes.cpu().numpy(), bits, dim), ref["q"], ref["pre_round"])
    want = O.dequant_rotate_inv_kron(codes.cpu().numpy(), scales.cpu().numpy(), F, b, signs, bits, group)
    out = B.hadq_dequant_rotate_inv_kron_pm1(codes, scales, sa, b, signs=sg, bits=bits, group=group,
                                             out_dtype=torch.float32)
    outb = B.hadq_dequant_rotate_inv_kron_pm1(codes, scales, sa, b, signs=sg, bits=bits, group=group)
    torch.cuda.synchronize()
    check_values(out.cpu().numpy(), want, "inverse f32")
    check_bf16(bf16_tensor_to_bits(outb), want, "inverse bf16")


def test_full_size_pm1_workload_sampled():
    # the 8192 x 5120 workload (Paley S_20, b = 256, INT4 group 128, signs)
    # in the launch configuration the benchmark times; sampled rows
    wl = S.WORKLOADS["c6_tok8192_d5120_kron20x256_int4_g128"]
    x = S.tensor(wl, 0)
    Sa = S.paley_hadamard(wl.kron_a - 1)
    signs = S.signs(wl)
    dev = "cuda"
    codes, scales = B.hadq_rotate_quantize_kron_pm1(
        bits_to_bf16_tensor(x, dev), torch.from_numpy(Sa).to(dev), wl.dim // wl.kron_a,
        signs=None if signs is None else torch.from_numpy(signs).to(dev), bits=wl.bits, group=wl.group)
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    rows = np.unique(np.concatenate([[0, wl.rows - 1], rng.integers(0, wl.rows, size=40)]))
    ref = O.rotate_quantize_kron(x[rows], Sa.astype(np.float64) / math.sqrt(wl.kron_a), wl.dim // wl.kron_a,
                                 signs, wl.bits, wl.group)
    idx = torch.from_numpy(rows).to(dev)
    check_scales(scales.index_select(0, idx).cpu().numpy(), ref["scales"])
    check_codes(gpu_codes_to_int(codes.index_select(0, idx).cpu().numpy(), wl.bits, wl.dim), ref["q"],
                ref["pre_round"])
    assert torch.all(scales > 0)
