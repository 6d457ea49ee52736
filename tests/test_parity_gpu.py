"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Oracle-sized cases: every kernel family, block and group sizes inside and
across blocks, signs, INT4 and INT8, ragged row counts, odd shapes on the
generic kernel, unaligned pointers, degenerate groups.  Each case compares
rotated values, scales and codes, then feeds the GPU codes and scales to both
dequantisers and compares the reconstructions (float32 and bf16).
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

DEV = "cuda"


def oracle_method(dim, block):
    B_ = dim if block == -1 else block
    return "dense" if B_ <= 4096 else "fwht"


def run_case(rows, dim, block, group, bits, with_signs, seed=1, dist="normal", outliers=(),
             x_bits=None, offset=0, check_dequant=True, max_mismatches=None):
    if x_bits is None:
        x_bits = S.random_bf16(rows, dim, seed, dist=dist, outlier_cols=outliers)
    s = S.random_signs(dim, seed) if with_signs else None
    meth = oracle_method(dim, block)
    ref = O.rotate_quantize(x_bits, block=block, signs=s, bits=bits, group=group, method=meth)

    if offset:  # a view starting `offset` elements into a larger buffer: unaligned pointers
        xb = bits_to_bf16_tensor(np.concatenate([np.zeros(offset, np.uint16), x_bits.ravel()]), DEV)
        x = xb[offset:].view(rows, dim)
    else:
        x = bits_to_bf16_tensor(x_bits, DEV)
    sg = None if s is None else torch.from_numpy(s).to(DEV)
    rot = torch.empty((rows, dim), dtype=torch.float32, device=DEV)
    codes, scales = B.hadq_rotate_quantize(x, block=block, signs=sg, bits=bits, group=group,
                                           rotated_out=rot)
    torch.cuda.synchronize()
    check_values(rot.cpu().numpy(), ref["rotated"], "rotated")
    check_scales(scales.cpu().numpy(), ref["scales"])
    check_codes(gpu_codes_to_int(codes.cpu().numpy(), bits, dim), ref["q"], ref["pre_round"], max_mismatches)

    # the same codes without the optional float output (the timed configuration)
    codes2, scales2 = B.hadq_rotate_quantize(x, block=block, signs=sg, bits=bits, group=group)
    torch.cuda.synchronize()
    if B.hadq_plan(0, rows, dim, block, bits, group, with_signs, True) == "h4096_tc" and offset == 0:
        # without rotated_out these blocks take the tcgen05 kernel, whose float32
        # accumulation order differs from the kernel above: checked against the
        # oracle on its own
        B.hadq_device_status()
        check_scales(scales2.cpu().numpy(), ref["scales"])
        check_codes(gpu_codes_to_int(codes2.cpu().numpy(), bits, dim), ref["q"], ref["pre_round"], max_mismatches)
    else:
        assert torch.equal(codes2, codes) and torch.equal(scales2, scales)

    if check_dequant:
        g_codes = codes.cpu().numpy()
        g_scales = scales.cpu().numpy()
        o_rec = O.dequant_rotate_inv(g_codes, g_scales, dim, block=block, signs=s, bits=bits,
                                     group=group, method=meth)
        f32 = B.hadq_dequant_rotate_inv(codes, scales, dim, block=block, signs=sg, bits=bits,
                                        group=group, out_dtype=torch.float32)
        b16 = B.hadq_dequant_rotate_inv(codes, scales, dim, block=block, signs=sg, bits=bits,
                                        group=group, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        check_values(f32.cpu().numpy(), o_rec, "dequant fp32")
        check_bf16(bf16_tensor_to_bits(b16), o_rec, "dequant bf16")
    return codes, scales


# (rows, dim, block, group, bits, signs, expected forward path)
CASES = [
    (300, 128, -1, -1, 8, False, "chunk_mma"),        # Q/K heads, INT8, per row
    (301, 128, 128, 128, 4, False, "chunk_mma"),    # KV rows, INT4, group 128
    (33, 384, 128, 128, 8, False, "chunk_mma"),     # three blocks per row, a short last slab
    (7, 11008, 128, 128, 4, False, "chunk_mma"),    # 86 blocks per row
    (1, 128, 128, 128, 4, False, "chunk_mma"),      # one block
    (65, 1024, 128, 128, 8, False, "chunk_mma"),
    (1000, 11008, 128, 128, 4, True, "chunk_mma"),  # 86000 blocks: every warp takes several slabs
    (640, 2560, 128, 128, 8, True, "chunk_mma"),    # INT8 with signs, 12800 blocks
    (2049, 128, -1, -1, 4, False, "chunk_mma"),     # one block per row, a ragged last slab
    (37, 4096, 128, -1, 4, False, "chunk"),         # per-token scale over 32 blocks
    (9, 11008, 128, 128, 4, True, "chunk_mma"),     # 86 blocks, signs
    (45, 1152, 128, 128, 8, True, "chunk_mma"),     # signs, 9 blocks per row, a short last slab
    (300, 128, 128, 128, 8, True, "chunk_mma"),     # signs, one block per row (every block at column 0)
    (77, 384, 128, 128, 4, True, "chunk_mma"),      # signs, 3 blocks per row: slabs start at every column
    (41, 4096, 128, 128, 4, True, "chunk_mma"),     # signs, exactly one slab per row
    (23, 2560, 128, 128, 8, True, "chunk_mma"),     # signs, 20 blocks per row (< one slab)
    (13, 5248, 128, 128, 4, True, "chunk_mma"),     # signs, 41 blocks per row (> one slab, < two)
    (5, 11008, 128, -1, 8, True, "chunk"),          # 86 blocks, one scale per row
    (300, 256, 32, 8, 4, False, "chunk"),           # groups smaller than a block
    (70, 512, 64, 16, 8, True, "chunk"),
    (140, 384, 16, 32, 4, True, "chunk"),           # groups wider than blocks, inside a chunk
    (40, 2048, 32, 256, 8, False, "chunk"),         # groups of two chunks (warp shuffle)
    (20, 6144, 64, 2048, 8, True, "chunk"),         # groups of 16 chunks (warp shuffle)
    (30, 768, 128, 384, 4, False, "chunk"),         # groups of 3 chunks (CTA shared-memory max)
    (3, 16384, 128, -1, 4, True, "chunk"),          # one row per slab
    (33, 1152, 8, 64, 8, False, "chunk"),           # 8-point blocks, 9 chunks per row
    (5, 32768, 128, 128, 4, True, "chunk_mma"),     # widest row, signs (largest sign-word table)
    (5, 32768, 128, 64, 4, True, "chunk"),          # widest row, groups inside chunks
    (33, 1024, 256, 64, 4, True, "blocked"),        # 256-point blocks
    (17, 768, 256, -1, 8, False, "blocked"),        # row of three 256-blocks
    (6, 8192, 256, 1024, 8, True, "blocked"),
    (129, 64, 64, 32, 4, False, "blocked"),         # dim not a multiple of 128
    (61, 96, 32, 8, 8, True, "blocked"),
    (21, 4096, -1, -1, 4, True, "h4096_tc"),        # full 4096 + signs, per token (ragged last tile)
    (22, 4096, -1, -1, 8, False, "h4096_tc"),
    (37, 4096, -1, -1, 8, True, "h4096_tc"),        # INT8 with signs
    (1, 4096, -1, -1, 4, False, "h4096_tc"),        # a single row
    (1201, 4096, -1, -1, 4, True, "h4096_tc"),      # 301 tiles: every CTA loops, stages and accumulators wrap
    (613, 4096, 4096, 4096, 8, True, "h4096_tc"),
    (5, 8192, 4096, 4096, 8, True, "wide4096"),     # two 4096-blocks per row, scale per block
    (4, 8192, 4096, 4096, 4, True, "wide4096"),
    (3, 12288, 4096, 4096, 4, False, "h4096_tc"),   # three blocks per row, no signs
    (203, 8192, 4096, 4096, 8, False, "h4096_tc"),  # 406 blocks, two per row
    (19, 4096, -1, 128, 8, False, "full4096"),
    (7, 4096, 4096, 64, 4, True, "full4096"),
    (11, 4096, -1, 1024, 8, True, "full4096"),
    (8, 4096, -1, 2048, 4, False, "full4096"),
    (13, 4096, -1, 512, 4, False, "full4096"),
    (10, 4096, -1, 256, 8, True, "full4096"),
    (5, 12, 4, 3, 8, False, "generic"),             # odd group, tiny block
    (9, 4096, -1, 32, 4, True, "generic"),          # groups too small for the 4096 path
    (4, 8192, -1, -1, 4, True, "generic"),          # 8192-point block
    (6, 100, 4, 10, 4, False, "generic"),
    (3, 2048, -1, -1, 8, True, "generic"),
    (12, 24, 8, 8, 4, False, "generic"),
    (2, 32768, 128, -1, 4, False, "generic"),       # widest row, one scale per row
    (1, 1, 1, 1, 8, False, "generic"),
    (50, 64, 16, 16, 8, True, "generic"),
    (3, 6, 2, 6, 4, False, "generic"),
]


@pytest.mark.parametrize("rows,dim,block,group,bits,signs,path", CASES)
def test_parity_shapes(rows, dim, block, group, bits, signs, path):
    assert B.hadq_plan(0, rows, dim, block, bits, group, signs, True) == path
    run_case(rows, dim, block, group, bits, signs, seed=rows * 7 + dim, outliers=[dim // 3])


@pytest.mark.parametrize("dist", ["normal", "student_t3"])
def test_parity_distributions(dist):
    run_case(64, 1024, 128, 128, 4, True, seed=5, dist=dist)


def test_unaligned_pointer_takes_generic_path_and_matches():
    run_case(31, 128, -1, -1, 8, False, seed=3, offset=1, check_dequant=False)
    run_case(9, 4096, -1, -1, 4, True, seed=4, offset=3, check_dequant=False)


def test_zero_rows_and_zero_groups():
    for dim, block, group, bits in [(128, -1, -1, 8), (256, 128, 64, 4), (4096, -1, -1, 4),
                                    (4096, 128, -1, 4), (12, 4, 3, 8)]:
        x = np.zeros((4, dim), np.uint16)
        x[1] = S.random_bf16(1, dim, 9)[0]
        codes, scales = run_case(4, dim, block, group, bits, False, x_bits=x)
        sc = scales.cpu().numpy().reshape(4, -1)
        assert np.all(sc[0] == 0) and np.all(sc[2:] == 0)
        assert not torch.any(codes[0].to(torch.int32)) and not torch.any(codes[2:].to(torch.int32))
    x = torch.empty((0, 128), dtype=torch.bfloat16, device=DEV)
    codes, scales = B.hadq_rotate_quantize(x, block=-1, bits=8)
    assert codes.shape == (0, 128) and scales.shape == (0, 1)


def test_tiny_and_subnormal_groups():
    """Groups whose maximum is subnormal-sized: qmax/max would overflow float32."""
    for dim, block, group in [(128, 128, 128), (4096, -1, -1), (12, 4, 3)]:
        rng = np.random.default_rng(dim)
        x = rng.integers(1, 0x7F, size=(3, dim)).astype(np.uint16)       # subnormal bf16
        x |= (rng.integers(0, 2, size=(3, dim)) << 15).astype(np.uint16)  # random signs
        x[2] = S.random_bf16(1, dim, 3)[0]
        run_case(3, dim, block, group, 4, False, x_bits=x)
        run_case(3, dim, block, group, 8, False, x_bits=x)


def test_exact_ties_round_half_even():
    # block 1 (no rotation): scale = 7/7 = 1, values on .5 exactly.
    y = np.array([[7, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5]], dtype=np.float32)
    x = S.f32_to_bf16_bits(np.repeat(y, 40, axis=0).reshape(40, 8))
    for group in (8, -1):
        codes, _ = B.hadq_rotate_quantize(bits_to_bf16_tensor(x, DEV), block=1, bits=4, group=group)
        q = gpu_codes_to_int(codes.cpu().numpy(), 4, 8)
        np.testing.assert_array_equal(q, np.tile([7, 0, 2, 2, 0, -2, -2, 4], (40, 1)))
    # through 32-wide blocks: y = H x with x = 2*e_0 gives +-2/sqrt(32); add a
    # block where the quantiser sees exact halves after an exact transform.
    x = np.zeros((2, 32), np.float32)
    x[0, 0] = 14.0           # y = 14/sqrt(32) everywhere -> all codes 7
    x[1, :2] = [3.0, 1.0]    # y in {4, 2}/sqrt(32): INT4 codes 7 and 3.5 -> 4 (even)
    codes, _ = B.hadq_rotate_quantize(bits_to_bf16_tensor(S.f32_to_bf16_bits(x), DEV), block=32,
                                      bits=4, group=32)
    q = gpu_codes_to_int(codes.cpu().numpy(), 4, 32)
    assert np.all(q[0] == 7)
    assert set(np.abs(q[1]).tolist()) == {7, 4}


def test_hand_worked_examples_on_gpu(golden_hand):
    g = golden_hand
    x = bits_to_bf16_tensor(S.f32_to_bf16_bits(np.array([g["ex1_x"]], np.float32)), DEV)
    codes, scales = B.hadq_rotate_quantize(x, block=-1, bits=4)
    assert codes.cpu().numpy().ravel().tolist() == [int(v) for v in g["ex1_int4_bytes"]]
    assert scales.item() == pytest.approx(5 / 7, rel=1e-6)
    codes, _ = B.hadq_rotate_quantize(x, block=-1, bits=8)
    assert codes.cpu().numpy().ravel().tolist() == [int(v) for v in g["ex1_int8_q"]]
    sg = torch.tensor(g["ex2_signs"], dtype=torch.int8, device=DEV)
    codes, _ = B.hadq_rotate_quantize(x, block=-1, signs=sg, bits=4)
    assert codes.cpu().numpy().ravel().tolist() == [int(v) for v in g["ex2_int4_bytes"]]


def test_non_default_stream_and_launch_count():
    x_bits = S.random_bf16(64, 128, 2)
    x = bits_to_bf16_tensor(x_bits, DEV)
    st = torch.cuda.Stream()
    n0 = B.hadq_launch_count()
    with torch.cuda.stream(st):
        codes, scales = B.hadq_rotate_quantize(x, block=-1, bits=8, stream=st)
    st.synchronize()
    assert B.hadq_launch_count() == n0 + 1
    ref = O.rotate_quantize(x_bits, block=-1, bits=8)
    check_codes(gpu_codes_to_int(codes.cpu().numpy(), 8, 128), ref["q"], ref["pre_round"])


def test_binding_rejects_bad_tensors():
    x = torch.zeros((4, 128), dtype=torch.float32, device=DEV)
    with pytest.raises(TypeError):
        B.hadq_rotate_quantize(x)
    x = torch.zeros((4, 100), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(B.HadqError) as e:
        B.hadq_rotate_quantize(x, block=64, bits=4)
    assert e.value.status == B.HADQ_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        B.hadq_rotate_quantize(torch.zeros((128, 4), dtype=torch.bfloat16, device=DEV).t(), bits=8)


@pytest.mark.parametrize("bits,with_signs", [(4, True), (8, False)])
def test_h4096_edge_rows(bits, with_signs):
    # both tensor-core 4096 kernels (the rotated_out call takes the mma.sync
    # one, the codes-only call the tcgen05 one): zero, one-hot, tiny (1e-30,
    # bf16 subnormal 1e-39), huge (1e30) and spiky rows, and a row count that
    # leaves the last tile short
    rng = np.random.default_rng(31)
    dim = 4096
    rows = [np.zeros(dim, np.float32),
            np.eye(dim, dtype=np.float32)[1234] * 3.0,
            (rng.normal(size=dim) * 1e-30).astype(np.float32),
            (rng.normal(size=dim) * 1e-39).astype(np.float32),
            (rng.normal(size=dim) * 1e30).astype(np.float32),
            np.where(rng.random(dim) < 0.001, 5e3, rng.normal(size=dim)).astype(np.float32),
            rng.normal(size=dim).astype(np.float32)]
    x = S.f32_to_bf16_bits(np.stack(rows))
    assert B.hadq_plan(0, len(rows), dim, -1, bits, -1, with_signs, True) == "h4096_tc"
    run_case(len(rows), dim, -1, -1, bits, with_signs, seed=12, x_bits=x)


@pytest.mark.parametrize("dim,bits,with_signs", [(128, 8, False), (384, 4, False), (384, 8, True),
                                                (11008, 4, True)])
def test_chunk_mma_edge_rows(dim, bits, with_signs):
    # the tensor-core 128 path: zero, one-hot, tiny (1e-30, bf16 subnormal
    # 1e-39), huge (1e30) and spiky rows; 40 rows = one full slab of 32
    # blocks plus a short one.  A block with K spikes of 5e3 puts pre-round
    # values next to the ties 7 k / K, so boundary mismatches (each still
    # within 1e-4 of a .5 boundary) are not capped at one here.
    rng = np.random.default_rng(dim + bits)
    base = [np.zeros(dim, np.float32),
            np.eye(dim, dtype=np.float32)[dim // 3] * 3.0,
            (rng.normal(size=dim) * 1e-30).astype(np.float32),
            (rng.normal(size=dim) * 1e-39).astype(np.float32),
            (rng.normal(size=dim) * 1e30).astype(np.float32),
            np.where(rng.random(dim) < 0.02, 5e3, rng.normal(size=dim)).astype(np.float32)]
    rows = base + [rng.normal(size=dim).astype(np.float32) for _ in range(40 - len(base))]
    x = S.f32_to_bf16_bits(np.stack(rows))
    assert B.hadq_plan(0, len(rows), dim, 128, bits, 128, with_signs, True) == "chunk_mma"
    run_case(len(rows), dim, 128, 128, bits, with_signs, seed=13, x_bits=x, max_mismatches=16)
