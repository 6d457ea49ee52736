"""Parity of the decode-attention kernel with the float64 oracle.

Small cases take their KV cache from the oracle's own rotate+quantise of
seeded bf16 rows (with outlier columns), so the cache holds what the
production path stores.  The full-size case (32 query heads, 8 KV heads,
131072 cached tokens) uses seeded random INT4 codes and row scales, runs in
the launch configuration the benchmark times, and compares sampled heads.

Rule (tests/parity.py): float32 output within 1e-5 of max(|o|, row RMS of o)
plus the float32 conditioning of softmax on the scores; bf16 output within one
bf16 ulp more.
"""

import numpy as np
import pytest
import torch

import oracle as O
from hadamard_rotation_outlier_b200 import binding as B
from hadamard_rotation_outlier_b200 import synthetic as S

from parity import attention_allowance, check_attention

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DIM = 128


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _q_tensor(bits):
    return _dev(bits.view(np.int16)).view(torch.bfloat16)


def oracle_cache(batch, nkv, stride, seed, with_outliers=True, signs=None, group=128, bits=4):
    """K and V caches quantised by the oracle from seeded bf16 rows; codes
    [batch, nkv, stride, dim * bits / 8], scales [batch, nkv, stride] for
    group 128, else [batch, nkv, stride, 128/group]."""
    rows = batch * nkv * stride
    cols = (3, 77, 101) if with_outliers else ()
    kx = S.random_bf16(rows, DIM, seed, outlier_cols=cols, outlier_scale=30.0)
    vx = S.random_bf16(rows, DIM, seed + 1)
    k = O.rotate_quantize(kx, block=128, signs=signs, bits=bits, group=group, method="fwht")
    v = O.rotate_quantize(vx, block=128, signs=signs, bits=bits, group=group, method="fwht")
    shape = (batch, nkv, stride)
    sshape = shape if group == 128 else shape + (DIM // group,)
    per_row = DIM * bits // 8
    return (k["codes"].reshape(shape + (per_row,)), k["scales"].reshape(sshape),
            v["codes"].reshape(shape + (per_row,)), v["scales"].reshape(sshape))


def run_gpu(qbits, kc, ks, vc, vs, tokens, signs, out_dtype, softmax_scale=None, workspace=None, group=128,
            bits=4):
    sg = None if signs is None else _dev(signs)
    out = B.hadq_kv_decode_attention(_q_tensor(qbits), _dev(kc), _dev(ks), _dev(vc), _dev(vs),
                                     tokens=tokens, block=128, signs=sg, bits=bits, group=group,
                                     softmax_scale=softmax_scale, out_dtype=out_dtype,
                                     workspace=workspace)
    torch.cuda.synchronize()
    return out


def oracle_attention(qbits, kc, ks, vc, vs, signs=None, softmax_scale=None, group=128, bits=4):
    """Oracle output and its allowance for the cache rows given."""
    want = O.kv_decode_attention(qbits, kc, ks, vc, vs, DIM, 128, signs, bits, group, softmax_scale)
    scores = O.kv_decode_scores(qbits, kc, ks, DIM, 128, signs, bits, group, softmax_scale)
    nb, nkv, T = ks.shape[:3]
    values = O.dequant_rotate_inv(vc.reshape(-1, DIM * bits // 8), vs.reshape(-1), DIM, 128, signs, bits, group,
                                  method="fwht").reshape(nb, nkv, T, DIM)
    return want, attention_allowance(want, scores, values, qbits.shape[1] // nkv)


def compare(out, want, out_dtype, what):
    want, allow = want
    if out_dtype == torch.float32:
        return check_attention(out.cpu().numpy(), want, allow, what)
    bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    return check_attention(bits, want, allow, what, bf16=True)


CASES = [
    # batch, n_q_heads, n_kv_heads, tokens, stride, signs
    (1, 4, 1, 1, 1, False),          # one cached token
    (1, 4, 1, 16, 16, False),        # one tile
    (2, 8, 2, 37, 40, False),        # ragged tail, stride > tokens
    (1, 32, 8, 1000, 1000, True),    # GQA 4 with signs
    (2, 6, 2, 300, 300, False),      # 3 query heads per KV head
    (1, 16, 2, 513, 520, True),      # 8 per KV head: two head groups
    (1, 2, 2, 129, 129, False),      # MHA
    (3, 12, 12, 77, 80, True),
    (1, 8, 1, 5000, 5000, False),    # many splits
]


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("batch,nqh,nkv,tokens,stride,with_signs", CASES)
def test_decode_attention_matches_oracle(batch, nqh, nkv, tokens, stride, with_signs, out_dtype):
    seed = 1000 + batch * 7 + nqh * 13 + tokens
    signs = S.random_signs(DIM, seed) if with_signs else None
    kc, ks, vc, vs = oracle_cache(batch, nkv, stride, seed, signs=signs)
    qbits = S.decode_query(batch, nqh, DIM, seed)
    want = oracle_attention(qbits, kc[:, :, :tokens], ks[:, :, :tokens], vc[:, :, :tokens],
                            vs[:, :, :tokens], signs)
    out = run_gpu(qbits, kc, ks, vc, vs, tokens, signs, out_dtype)
    compare(out, want, out_dtype, f"attention {batch}x{nqh}/{nkv} T={tokens}")


def test_peaked_and_flat_softmax():
    # A large softmax scale makes the weights nearly one-hot (scores span
    # hundreds of log2 units); a zero query makes them uniform.
    kc, ks, vc, vs = oracle_cache(1, 2, 700, 5)
    qbits = S.decode_query(1, 8, DIM, 5)
    for scale in (4.0, 0.001):
        want = oracle_attention(qbits, kc, ks, vc, vs, softmax_scale=scale)
        out = run_gpu(qbits, kc, ks, vc, vs, 700, None, torch.float32, softmax_scale=scale)
        compare(out, want, torch.float32, f"softmax scale {scale}")
    zq = np.zeros_like(qbits)
    want = oracle_attention(zq, kc, ks, vc, vs)
    out = run_gpu(zq, kc, ks, vc, vs, 700, None, torch.float32)
    compare(out, want, torch.float32, "zero query")


def test_increasing_scores_force_rescales():
    # Keys ordered so every later tile holds a larger score: the running max
    # is raised again and again.
    rng = np.random.default_rng(9)
    T = 640
    q = np.zeros(DIM)
    q[0] = 1.0
    qbits = S.f32_to_bf16_bits(q.astype(np.float32))[None, None].repeat(4, axis=1)
    qk = np.zeros((1, 1, T, DIM), np.int64)
    qk[..., :] = rng.integers(-7, 8, size=(1, 1, T, DIM))
    qk[..., :] = np.sign(qk.sum(-1, keepdims=True) + 0.5) * qk   # positive row sums
    ks = np.linspace(0.01, 30.0, T, dtype=np.float32).reshape(1, 1, T)
    vq = rng.integers(-7, 8, size=(1, 1, T, DIM))
    vs = rng.uniform(0.1, 1.0, size=(1, 1, T)).astype(np.float32)
    kc, vc = O.pack_int4(qk), O.pack_int4(vq)
    want = oracle_attention(qbits, kc, ks, vc, vs, softmax_scale=1.0)
    out = run_gpu(qbits, kc, ks, vc, vs, T, None, torch.float32, softmax_scale=1.0)
    compare(out, want, torch.float32, "increasing scores")


def test_workspace_is_reusable_and_results_repeat():
    kc, ks, vc, vs = oracle_cache(2, 4, 333, 21)
    qbits = S.decode_query(2, 16, DIM, 21)
    need = B.hadq_kv_decode_workspace_size(2, 16, 4, 333)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    a = run_gpu(qbits, kc, ks, vc, vs, 333, None, torch.float32, workspace=ws)
    b = run_gpu(qbits, kc, ks, vc, vs, 333, None, torch.float32, workspace=ws)
    assert torch.equal(a, b)
    head = ws[:2 * 4 * 4].view(torch.int32)   # counters are back at zero
    assert int(head.abs().sum()) == 0
    want = oracle_attention(qbits, kc, ks, vc, vs)
    compare(a, want, torch.float32, "reused workspace")


def test_one_launch_per_call_on_the_given_stream():
    kc, ks, vc, vs = oracle_cache(1, 1, 64, 3)
    qbits = S.decode_query(1, 4, DIM, 3)
    args = [_q_tensor(qbits), _dev(kc), _dev(ks), _dev(vc), _dev(vs)]
    ws = torch.zeros(B.hadq_kv_decode_workspace_size(1, 4, 1, 64), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    n0 = B.hadq_launch_count()
    with torch.cuda.stream(s):
        out = B.hadq_kv_decode_attention(*args, workspace=ws, out_dtype=torch.float32, stream=s)
    s.synchronize()
    assert B.hadq_launch_count() == n0 + 1
    want = oracle_attention(qbits, kc, ks, vc, vs)
    compare(out, want, torch.float32, "side stream")


def test_rejections_leave_output_untouched():
    kc, ks, vc, vs = oracle_cache(1, 1, 32, 4)
    qbits = S.decode_query(1, 4, DIM, 4)
    args = [_q_tensor(qbits), _dev(kc), _dev(ks), _dev(vc), _dev(vs)]
    out = torch.full((1, 4, DIM), 7.0, device="cuda")
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.HadqError) as e:
        B.hadq_kv_decode_attention(*args, out=out, out_dtype=torch.float32, workspace=small)
    assert e.value.status == B.HADQ_ERR_INVALID_ARG and "workspace" in str(e.value)
    with pytest.raises(B.HadqError) as e:
        B.hadq_kv_decode_attention(*args, out=out, out_dtype=torch.float32, block=64)
    assert e.value.status == B.HADQ_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_full_size_decode_sampled_heads():
    dw = S.DECODE_WORKLOADS["d1_decode_q32_kv8_t131072_d128_int4"]
    kc, ks = S.random_int4_cache(dw.batch, dw.n_kv_heads, dw.tokens, DIM, 71)
    vc, vs = S.random_int4_cache(dw.batch, dw.n_kv_heads, dw.tokens, DIM, 72)
    qbits = S.decode_query(dw.batch, dw.n_q_heads, DIM, 73)
    out = run_gpu(qbits, kc, ks, vc, vs, dw.tokens, None, torch.bfloat16)
    g = dw.n_q_heads // dw.n_kv_heads
    for kvh in (0, 5, 7):
        sl = slice(kvh * g, (kvh + 1) * g)
        want = oracle_attention(qbits[:, sl], kc[:, kvh:kvh + 1], ks[:, kvh:kvh + 1],
                                vc[:, kvh:kvh + 1], vs[:, kvh:kvh + 1])
        compare(out[:, sl].contiguous(), want, torch.bfloat16, f"full size, KV head {kvh}")
    assert torch.isfinite(out.float()).all()


GROUP_CASES = [
    # batch, n_q_heads, n_kv_heads, tokens, stride, signs, group (the cache's scale group)
    (1, 4, 1, 1, 4, False, 64),        # one cached token
    (1, 8, 2, 300, 300, False, 64),    # GQA 4
    (1, 8, 2, 45, 46, True, 64),       # ragged tail, stride > tokens
    (2, 8, 2, 37, 40, True, 32),       # ragged tail, groups of 32
    (1, 32, 8, 1000, 1000, True, 32),  # GQA 4 with signs
    (1, 16, 2, 513, 520, False, 32),   # two head groups per KV head
    (1, 8, 1, 5000, 5000, False, 64),  # many splits
]


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("batch,nqh,nkv,tokens,stride,with_signs,group", GROUP_CASES)
def test_decode_attention_grouped_cache(batch, nqh, nkv, tokens, stride, with_signs, group, out_dtype):
    # caches quantised with 2 or 4 scales per row (groups of 64 or 32 columns)
    seed = 2000 + batch * 7 + nqh * 13 + tokens + group
    signs = S.random_signs(DIM, seed) if with_signs else None
    kc, ks, vc, vs = oracle_cache(batch, nkv, stride, seed, signs=signs, group=group)
    qbits = S.decode_query(batch, nqh, DIM, seed)
    want = oracle_attention(qbits, kc[:, :, :tokens], ks[:, :, :tokens], vc[:, :, :tokens],
                            vs[:, :, :tokens], signs, group=group)
    out = run_gpu(qbits, kc, ks, vc, vs, tokens, signs, out_dtype, group=group)
    compare(out, want, out_dtype, f"attention G={group} {batch}x{nqh}/{nkv} T={tokens}")


def test_grouped_cache_with_one_group_matches_row_scales():
    # scales given as [.., 4] with all four equal must give the same output as
    # the one-scale-per-row cache (the grouped path reduces to the row path)
    kc, ks, vc, vs = oracle_cache(1, 2, 700, 9)
    qbits = S.decode_query(1, 8, DIM, 9)
    a = run_gpu(qbits, kc, ks, vc, vs, 700, None, torch.float32)
    ks4 = np.repeat(ks[..., None], 4, axis=-1)
    vs4 = np.repeat(vs[..., None], 4, axis=-1)
    b = run_gpu(qbits, kc, ks4, vc, vs4, 700, None, torch.float32, group=32)
    want = oracle_attention(qbits, kc, ks, vc, vs)
    compare(b, want, torch.float32, "G=32 with equal group scales")
    # the grouped path sums its four group partials (each weighted by its
    # scale) where the row path scales one sum: equal up to float32 rounding
    np.testing.assert_allclose(b.cpu().numpy(), a.cpu().numpy(), rtol=1e-5, atol=1e-5)


def test_grouped_cache_rejections():
    q = torch.zeros((1, 4, DIM), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 1, 7, DIM // 2), dtype=torch.uint8, device="cuda")
    ks2 = torch.ones((1, 1, 7, 2), dtype=torch.float32, device="cuda")
    n0 = B.hadq_launch_count()
    with pytest.raises(B.HadqError) as e:   # groups of 64 need token_stride * 2 to be a multiple of 4
        B.hadq_kv_decode_attention(q, kc, ks2, kc, ks2, block=128, bits=4, group=64)
    assert e.value.status == B.HADQ_ERR_MISALIGNED
    ks8 = torch.ones((1, 1, 7, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(B.HadqError) as e:   # groups of 16 are not supported
        B.hadq_kv_decode_attention(q, kc, ks8, kc, ks8, block=128, bits=4, group=16)
    assert e.value.status == B.HADQ_ERR_UNSUPPORTED
    assert B.hadq_launch_count() == n0


INT8_CASES = [
    # batch, n_q_heads, n_kv_heads, tokens, stride, signs, group
    (1, 4, 1, 1, 1, False, 128),       # one cached token
    (1, 4, 1, 16, 16, False, 128),     # one tile
    (2, 8, 2, 37, 40, False, 128),     # ragged tail, stride > tokens
    (1, 32, 8, 1000, 1000, True, 128), # GQA 4 with signs
    (1, 16, 2, 513, 520, True, 128),   # two head groups per KV head
    (1, 8, 1, 5000, 5000, False, 128), # many splits
    (1, 8, 2, 300, 300, True, 64),     # groups of 64
    (2, 8, 2, 37, 40, False, 32),      # groups of 32, ragged
]


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("batch,nqh,nkv,tokens,stride,with_signs,group", INT8_CASES)
def test_decode_attention_int8_cache(batch, nqh, nkv, tokens, stride, with_signs, group, out_dtype):
    # caches quantised to INT8 (one scale per row, or per group of 64 or 32)
    seed = 3000 + batch * 7 + nqh * 13 + tokens + group
    signs = S.random_signs(DIM, seed) if with_signs else None
    kc, ks, vc, vs = oracle_cache(batch, nkv, stride, seed, signs=signs, group=group, bits=8)
    qbits = S.decode_query(batch, nqh, DIM, seed)
    want = oracle_attention(qbits, kc[:, :, :tokens], ks[:, :, :tokens], vc[:, :, :tokens],
                            vs[:, :, :tokens], signs, group=group, bits=8)
    out = run_gpu(qbits, kc, ks, vc, vs, tokens, signs, out_dtype, group=group, bits=8)
    compare(out, want, out_dtype, f"attention INT8 G={group} {batch}x{nqh}/{nkv} T={tokens}")


def test_int8_cache_extreme_codes():
    # every code at -128, -127 or +127 (the ends of the exact bf16 conversion)
    rng = np.random.default_rng(17)
    T = 200
    kc = rng.choice(np.array([-128, -127, 127], np.int8), size=(1, 1, T, DIM))
    vc = rng.choice(np.array([-128, -127, 127, 0, 1, -1], np.int8), size=(1, 1, T, DIM))
    ks = rng.uniform(0.001, 0.01, size=(1, 1, T)).astype(np.float32)
    vs = rng.uniform(0.001, 0.01, size=(1, 1, T)).astype(np.float32)
    qbits = S.decode_query(1, 4, DIM, 17)
    want = oracle_attention(qbits, kc, ks, vc, vs, bits=8)
    out = run_gpu(qbits, kc, ks, vc, vs, T, None, torch.float32, bits=8)
    compare(out, want, torch.float32, "INT8 extreme codes")


def test_full_size_int8_decode_sampled_heads():
    # the 131072-token decode shape with an INT8 cache, in the launch the
    # benchmark times for it
    dw = S.DECODE_WORKLOADS["d1_decode_q32_kv8_t131072_d128_int4"]
    kc, ks = S.random_int8_cache(dw.batch, dw.n_kv_heads, dw.tokens, DIM, 81)
    vc, vs = S.random_int8_cache(dw.batch, dw.n_kv_heads, dw.tokens, DIM, 82)
    qbits = S.decode_query(dw.batch, dw.n_q_heads, DIM, 83)
    out = run_gpu(qbits, kc, ks, vc, vs, dw.tokens, None, torch.bfloat16, bits=8)
    g = dw.n_q_heads // dw.n_kv_heads
    for kvh in (0, 3, 7):
        sl = slice(kvh * g, (kvh + 1) * g)
        want = oracle_attention(qbits[:, sl], kc[:, kvh:kvh + 1], ks[:, kvh:kvh + 1],
                                vc[:, kvh:kvh + 1], vs[:, kvh:kvh + 1], bits=8)
        compare(out[:, sl].contiguous(), want, torch.bfloat16, f"full size INT8, KV head {kvh}")
    assert torch.isfinite(out.float()).all()
