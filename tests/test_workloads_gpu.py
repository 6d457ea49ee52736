"""Full-size parity on the five synthetic workloads, in the launch configuration
the benchmark times (one quantise launch over all rows, no float output; the
KV-cache workload adds one dequantise launch to bf16).

The oracle recomputes a sample of rows one by one (first, last and random
rows, regenerated from the same seeded chunks); properties that hold at any
size are checked on every row.
"""

import zlib

import numpy as np
import pytest
import torch

import oracle as O
from hadamard_rotation_outlier_b200 import synthetic as S
from hadamard_rotation_outlier_b200.steps import WorkloadStep, bf16_tensor_to_bits

from parity import check_asym, check_bf16, check_codes, check_scales, gpu_codes_to_int

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

N_SAMPLE = 48


def sample_rows(wl, rng):
    """(tensor index, row in tensor, row in the stacked buffer) samples."""
    out = []
    base = 0
    for ti, t in enumerate(wl.tensors):
        rows = [0, t.rows - 1] + list(rng.integers(0, t.rows, size=N_SAMPLE // len(wl.tensors)))
        out += [(ti, int(r), base + int(r)) for r in sorted(set(rows))]
        base += t.rows
    return out


@pytest.mark.parametrize("name", S.WORKLOAD_ORDER)
def test_full_workload_sampled_parity(name):
    wl = S.WORKLOADS[name]
    st = WorkloadStep(wl, "cuda")
    st.step()
    torch.cuda.synchronize()

    bits, dim = wl.bits, wl.dim
    qmax = 2 ** (bits - 1) - 1
    codes = st.codes
    # properties over every row: code range (INT8 is stored directly; INT4 nibbles)
    if wl.asym:
        pass  # unsigned codes: every value is in range
    elif bits == 8:
        assert int(codes.min()) >= -qmax and int(codes.max()) <= qmax
    else:
        lo = (codes & 0xF).to(torch.int16)
        hi = (codes >> 4).to(torch.int16)
        assert not torch.any(lo == 8) and not torch.any(hi == 8), "INT4 code -8 never produced"
    if wl.keep:  # rows of kept tokens have scale 0; every other row has none all-zero
        quantised = torch.from_numpy(st.keep_slot_host < 0).to("cuda").repeat(wl.heads)
        assert torch.all(st.scales[quantised] > 0) and not st.scales[~quantised].any()
    else:
        assert torch.all(st.scales > 0), "these workloads have no all-zero group"
    assert torch.isfinite(st.scales).all()

    rng = np.random.default_rng(zlib.crc32(name.encode()))
    samples = sample_rows(wl, rng)
    idx = torch.tensor([s[2] for s in samples], device="cuda")
    g_codes = codes.index_select(0, idx).cpu().numpy()
    g_scales = st.scales.index_select(0, idx).cpu().numpy()
    x = np.stack([S.tensor_rows(wl, ti, r, r + 1)[0] for ti, r, _ in samples])
    np.testing.assert_array_equal(bf16_tensor_to_bits(st.x.index_select(0, idx)), x)
    signs = S.signs(wl)
    if wl.keep:
        # rows of kept tokens: codes 0, scale 0, the bf16 row in `kept` and in
        # the read-back; the sampled rows of the other tokens follow below
        rows = np.array([s[2] for s in samples])
        heads_of, tok_of = rows // wl.tokens, rows % wl.tokens
        slot = st.keep_slot_host[tok_of]
        kept_s = slot >= 0
        for extra in (0, wl.tokens - 1):     # a sink and a window token of every head
            assert st.keep_slot_host[extra] >= 0
        kept_rows = np.array([h * wl.tokens + t for h in range(wl.heads) for t in (0, wl.tokens - 1)])
        kidx = torch.from_numpy(kept_rows).to("cuda")
        kx = bf16_tensor_to_bits(st.x.index_select(0, kidx))
        assert not codes.index_select(0, kidx).any() and not st.scales.index_select(0, kidx).any()
        kb = bf16_tensor_to_bits(st.kept).reshape(wl.heads, wl.n_keep, dim)
        np.testing.assert_array_equal(kb[kept_rows // wl.tokens, st.keep_slot_host[kept_rows % wl.tokens]], kx)
        np.testing.assert_array_equal(bf16_tensor_to_bits(st.out.index_select(0, kidx)), kx)
        keep_q = ~kept_s
        x, g_codes, g_scales, idx = x[keep_q], g_codes[keep_q], g_scales[keep_q], idx[torch.from_numpy(keep_q).to("cuda")]
        assert len(x) > 20
    if wl.kron_a:
        F = S.paley_hadamard(wl.kron_a - 1).astype(np.float64) / np.sqrt(wl.kron_a)   # the exact factor
        ref = O.rotate_quantize_kron(x, F, dim // wl.kron_a, signs, bits, wl.group)
        check_scales(g_scales, ref["scales"])
        check_codes(gpu_codes_to_int(g_codes, bits, dim), ref["q"], ref["pre_round"])
        del st
        torch.cuda.empty_cache()
        return
    if wl.asym:
        ref = O.rotate_quantize_asym(x, block=wl.block, signs=signs, bits=bits, group=wl.group)
        g_zp = st.zero_points.index_select(0, idx).cpu().numpy()
        gq = g_codes.astype(np.int64) if bits == 8 else O.unpack_uint4(g_codes)
        check_asym(gq, g_scales, g_zp, ref, bits)
        rec = O.dequant_rotate_inv_asym(g_codes, g_scales, g_zp, dim, block=wl.block, signs=signs, bits=bits,
                                        group=wl.group)
        check_bf16(bf16_tensor_to_bits(st.out.index_select(0, idx)), rec, "asym dequant bf16")
        del st
        torch.cuda.empty_cache()
        return
    ref = O.rotate_quantize(x, block=wl.block, signs=signs, bits=bits, group=wl.group)
    check_scales(g_scales, ref["scales"])
    check_codes(gpu_codes_to_int(g_codes, bits, dim), ref["q"], ref["pre_round"])

    if wl.dequant:
        rec = O.dequant_rotate_inv(g_codes, g_scales, dim, block=wl.block, signs=signs, bits=bits,
                                   group=wl.group)
        check_bf16(bf16_tensor_to_bits(st.out.index_select(0, idx)), rec, "dequant bf16")
    del st
    torch.cuda.empty_cache()
