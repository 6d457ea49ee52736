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
]


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
