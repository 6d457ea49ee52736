"""Parity of the mixed-precision (kept-token) quantiser and its read-back with
the float64 oracle.

Kept rows must be copied bit for bit (and read back bit for bit); every other
row follows the rules of tests/parity.py: codes bit-exact up to .5-boundary
cases, scales within 1e-5, reconstructions within 1e-5 of max(|o|, row RMS)
(one bf16 ulp more for bf16 output).  The full-size case is the KV-cache
workload with a HyQuant-style keep set, in the launch configuration the
benchmark times.
"""

import numpy as np
import pytest
import torch

import oracle as O
from hadamard_rotation_outlier_b200 import binding as B
from hadamard_rotation_outlier_b200 import synthetic as S
from hadamard_rotation_outlier_b200.steps import bf16_tensor_to_bits, bits_to_bf16_tensor

from parity import check_bf16, check_codes, check_scales, check_values, gpu_codes_to_int

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CASES = [
    # heads, tokens, dim, block, group, bits, signs, (n_sink, window, vertical)
    (2, 300, 128, 128, 128, 4, False, (4, 16, (50, 51, 200))),
    (3, 129, 256, 64, 256, 8, True, (1, 8, (3,))),
    (1, 70, 4096, 128, -1, 4, True, (2, 5, (30,))),
    (4, 77, 128, 32, 128, 4, True, (0, 0, ())),          # nothing kept
    (2, 40, 128, 128, -1, 8, False, (40, 0, ())),        # everything kept
    (2, 33, 512, 16, 256, 4, False, (3, 3, (17,))),
    # block = group = 128: the tensor-core quantiser's kept-token instances
    (2, 300, 128, 128, 128, 4, True, (4, 16, (50, 51, 200))),
    (3, 97, 256, 128, 128, 8, False, (1, 8, (3,))),    # two blocks per row, ragged last slab
    (2, 40, 128, 128, 128, 4, True, (40, 0, ())),       # everything kept
    (5, 61, 384, 128, 128, 4, False, (0, 0, ())),       # nothing kept, three blocks per row
    (1, 1, 128, 128, 128, 8, True, (1, 0, ())),         # one token, kept
]


def _run(heads, tokens, dim, block, group, bits, with_signs, keep, seed):
    x = S.random_bf16(heads * tokens, dim, seed, outlier_cols=[dim // 3], outlier_scale=40.0)
    signs = S.random_signs(dim, seed) if with_signs else None
    slots, n_keep = B.hyquant_keep_slots(tokens, *keep[:2], vertical=keep[2])
    dev = "cuda"
    xt = bits_to_bf16_tensor(x, dev).view(heads, tokens, dim)
    st = torch.from_numpy(slots).to(dev)
    sg = None if signs is None else torch.from_numpy(signs).to(dev)
    codes, scales, kept = B.hadq_rotate_quantize_keep(xt, st, n_keep, block=block, signs=sg, bits=bits,
                                                      group=group)
    torch.cuda.synchronize()
    ref = O.rotate_quantize_keep(x, heads, tokens, slots, n_keep, block=block, signs=signs, bits=bits,
                                 group=group, method="fwht")
    return x, signs, slots, n_keep, (st, sg), (codes, scales, kept), ref


@pytest.mark.parametrize("heads,tokens,dim,block,group,bits,with_signs,keep", CASES)
def test_keep_quantise_and_read_back(heads, tokens, dim, block, group, bits, with_signs, keep):
    x, signs, slots, n_keep, (st, sg), (codes, scales, kept), ref = _run(
        heads, tokens, dim, block, group, bits, with_signs, keep, seed=tokens + dim)
    rows = heads * tokens
    # kept rows: exact copies, codes 0, scale 0
    if n_keep:
        np.testing.assert_array_equal(bf16_tensor_to_bits(kept).reshape(heads, n_keep, dim), ref["kept"])
    q = gpu_codes_to_int(codes.cpu().numpy(), bits, dim)
    sc = scales.cpu().numpy().reshape(ref["scales"].shape)
    kr = ref["keep_row"]
    assert not q[kr].any() and not sc[kr].any()
    # quantised rows: the usual parity rules
    check_codes(q[~kr], ref["q"].reshape(rows, dim)[~kr], ref["pre_round"].reshape(rows, dim)[~kr])
    check_scales(sc[~kr], ref["scales"][~kr])
    # read-back, both output types
    G = dim if group == -1 else group
    for out_dtype in (torch.float32, torch.bfloat16):
        out = B.hadq_dequant_rotate_inv_keep(codes, scales, kept, st, n_keep, dim, block=block, signs=sg,
                                             bits=bits, group=group, out_dtype=out_dtype)
        torch.cuda.synchronize()
        want = O.dequant_rotate_inv_keep(codes.cpu().numpy().reshape(rows, -1), sc.reshape(rows, dim // G),
                                         bf16_tensor_to_bits(kept).reshape(heads, n_keep, dim), slots, n_keep,
                                         heads, tokens, dim, block=block, signs=signs, bits=bits, group=group,
                                         method="fwht")
        if out_dtype == torch.float32:
            got = out.cpu().numpy().reshape(rows, dim).astype(np.float64)
            np.testing.assert_array_equal(got[kr], O.bf16_bits_to_f64(x)[kr])
            check_values(got[~kr], want[~kr], "read-back f32")
        else:
            gb = bf16_tensor_to_bits(out).reshape(rows, dim)
            np.testing.assert_array_equal(gb[kr], x[kr])
            check_bf16(gb[~kr], want[~kr], "read-back bf16")


def test_out_of_range_slots_are_quantised():
    heads, tokens, dim = 2, 50, 128
    x = S.random_bf16(heads * tokens, dim, 5)
    slots = np.full(tokens, -1, np.int32)
    slots[[0, 10, 20, 30]] = [0, 1, 7, -3]        # n_keep = 2: tokens 20 and 30 are quantised
    dev = "cuda"
    codes, scales, kept = B.hadq_rotate_quantize_keep(bits_to_bf16_tensor(x, dev).view(heads, tokens, dim),
                                                      torch.from_numpy(slots).to(dev), 2, block=128, bits=4,
                                                      group=128)
    torch.cuda.synchronize()
    ref = O.rotate_quantize_keep(x, heads, tokens, slots, 2, block=128, bits=4, group=128)
    assert ref["keep_row"].sum() == 2 * heads
    np.testing.assert_array_equal(bf16_tensor_to_bits(kept).reshape(heads, 2, dim), ref["kept"])
    q = gpu_codes_to_int(codes.cpu().numpy(), 4, dim)
    check_codes(q, ref["q"].reshape(-1, dim), ref["pre_round"].reshape(-1, dim))


def test_full_size_kv_cache_with_kept_tokens():
    # K of the KV-cache workload, [8, 131072, 128], INT4 group 128, with 4 sink
    # tokens, 64 seeded vertical-line tokens and a 128-token window kept.
    wl = S.WORKLOADS["c4_kv_h8_t131072_d128_int4_g128"]
    heads, tokens, dim = 8, 131072, 128
    x = S.tensor(wl, 0)
    rng = np.random.default_rng(77)
    vertical = rng.choice(np.arange(4, tokens - 128), size=64, replace=False)
    slots, n_keep = B.hyquant_keep_slots(tokens, 4, 128, vertical)
    dev = "cuda"
    xt = bits_to_bf16_tensor(x, dev).view(heads, tokens, dim)
    st = torch.from_numpy(slots).to(dev)
    codes, scales, kept = B.hadq_rotate_quantize_keep(xt, st, n_keep, block=128, bits=4, group=128)
    torch.cuda.synchronize()
    kept_tokens = np.flatnonzero(slots >= 0)
    kb = bf16_tensor_to_bits(kept).reshape(heads, n_keep, dim)
    for h in range(heads):
        np.testing.assert_array_equal(kb[h, slots[kept_tokens]], x[h * tokens + kept_tokens])
    sc = scales.view(heads, tokens).cpu().numpy()
    assert not sc[:, kept_tokens].any()
    assert (sc[:, slots < 0] > 0).all()
    # sampled quantised rows against the oracle
    sample = np.concatenate([[5, tokens - 129], rng.integers(0, tokens, size=40)])
    sample = np.array([t for t in sample if slots[t] < 0])
    rows = np.array([h * tokens + t for h in (0, 3, 7) for t in sample])
    ref = O.rotate_quantize(x[rows], block=128, bits=4, group=128, method="fwht")
    c = codes.view(heads * tokens, dim // 2)[torch.from_numpy(rows).to(dev)].cpu().numpy()
    check_codes(O.unpack_int4(c), ref["q"], ref["pre_round"])
    check_scales(scales.view(-1)[torch.from_numpy(rows).to(dev)].cpu().numpy(), ref["scales"].reshape(-1))
