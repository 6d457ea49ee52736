"""Host-side checks of the C ABI: the library loads, exports every function
that include/hadq.h declares, and rejects bad arguments before any launch.

No call here reaches a kernel: every call either fails validation or is an
empty (rows == 0) call, both of which return before touching CUDA.
"""

import ctypes
import os
import re
import subprocess

import pytest

from hadamard_rotation_outlier_b200 import binding as B
from hadamard_rotation_outlier_b200.build import LIB, ROOT, build

HEADER = os.path.join(ROOT, "include", "hadq.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return B.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hadq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert names == sorted(B.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (hadq_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_version_and_status_strings(lib):
    assert B.hadq_version() == 1
    assert B.hadq_status_str(B.HADQ_OK) == "ok"
    assert "invalid" in B.hadq_status_str(B.HADQ_ERR_INVALID_ARG)
    assert "misaligned" in B.hadq_status_str(B.HADQ_ERR_MISALIGNED)
    assert "bounded wait" in B.hadq_status_str(B.HADQ_ERR_DEVICE)
    assert B.hadq_status_str(99) == "unknown status"


def test_bounded_wait_selftest_validates_before_launch(lib):
    assert lib.hadq_selftest_bounded_wait(None, None) == B.HADQ_ERR_INVALID_ARG
    assert "scratch" in B.hadq_last_error()
    assert lib.hadq_selftest_bounded_wait(ctypes.c_void_p(0x1008), None) == B.HADQ_ERR_MISALIGNED


@pytest.mark.parametrize("args,msg", [
    ((0, -1, 128, -1, 8, -1), "rows"),
    ((0, 4, 0, -1, 8, -1), "dim"),
    ((0, 4, 32769, 128, 8, -1), "dim"),
    ((0, 4, 128, -1, 5, -1), "bits"),
    ((0, 4, 127, 1, 4, -1), "even"),
    ((0, 4, 96, -1, 8, -1), "power-of-two dim"),
    ((0, 4, 128, 48, 8, -1), "power of two"),
    ((0, 4, 96, 64, 8, -1), "does not divide"),
    ((0, 4, 128, 128, 8, 0), "group"),
    ((0, 4, 128, 128, 8, 48), "does not divide"),
    ((2, 4, 128, 128, 8, -1), "direction"),
])
def test_plan_rejects(lib, args, msg):
    with pytest.raises(B.HadqError) as e:
        B.hadq_plan(*args)
    assert e.value.status == B.HADQ_ERR_INVALID_ARG
    assert msg in str(e.value)


@pytest.mark.parametrize("direction,rows,dim,block,bits,group,signs,a16,path", [
    (0, 0, 128, -1, 8, -1, False, True, "none"),
    (0, 524288, 128, -1, 8, -1, False, True, "chunk_mma"),        # Q/K heads, INT8
    (0, 256, 4096, 128, 4, -1, False, True, "chunk"),             # per-token over 32 blocks
    (0, 16384, 4096, -1, 4, -1, True, True, "h4096_tc"),          # full 4096 + signs
    (0, 16, 8192, 4096, 4, 4096, True, True, "wide4096"),         # two 4096 blocks + signs
    (0, 16, 8192, 4096, 4, 4096, False, True, "h4096_tc"),        # two 4096 blocks, no signs
    (0, 16384, 4096, -1, 4, 128, True, True, "full4096"),         # 4096 block, group 128
    (0, 2097152, 128, 128, 4, 128, False, True, "chunk_mma"),     # KV cache
    (1, 2097152, 128, 128, 4, 128, False, True, "chunk_mma"),     # KV dequant
    (1, 32768, 11008, 128, 4, 128, True, True, "chunk_mma"),      # dequant of 86 signed blocks
    (1, 100, 4096, 128, 8, -1, False, True, "chunk_mma"),         # dequant, one scale over 32 blocks
    (1, 100, 768, 128, 4, 384, True, True, "chunk_mma"),          # dequant, groups of 3 blocks
    (1, 100, 256, 128, 4, 64, False, True, "chunk"),              # dequant, groups inside a block
    (1, 100, 1024, 64, 4, 128, False, True, "chunk"),             # dequant, 64-point blocks
    (1, 10, 1024, 256, 4, 64, False, True, "blocked"),            # 256-point dequant
    (0, 32768, 11008, 128, 4, 128, True, True, "chunk_mma"),      # 86 blocks of 128, signs
    (0, 1 << 27, 1024, 128, 4, 128, False, True, "chunk"),        # 2^30 chunks: past 32-bit chunk indices
    (0, (1 << 27) - 1, 1024, 128, 4, 128, False, True, "chunk_mma"),  # the largest count that stays
    (1, 1 << 27, 1024, 128, 4, 128, False, True, "chunk"),        # the same limit for the dequantiser
    (0, 10, 1024, 256, 4, 64, True, True, "blocked"),             # 256-point blocks
    (0, 10, 96, 32, 8, -1, False, True, "blocked"),               # dim not a multiple of 128
    (0, 10, 32768, 128, 4, -1, False, True, "generic"),           # whole-row groups past 16384
    (0, 10, 128, -1, 8, -1, False, False, "generic"),             # unaligned pointers
    (0, 10, 4096, -1, 4, 32, False, True, "generic"),             # small groups on 4096
    (0, 10, 8192, -1, 4, -1, False, True, "generic"),             # 8192-point block
    (0, 10, 32768, 128, 4, 128, False, True, "chunk_mma"),        # widest row, group 128
    (0, 10, 32768, 128, 4, 128, True, True, "chunk_mma"),         # the same with signs
    (0, 10, 256, 128, 4, 64, False, True, "chunk"),               # groups smaller than the block
    (0, 10, 12, 4, 8, 3, False, True, "generic"),
    (1, 10, 4096, -1, 4, -1, True, True, "generic"),              # 4096 dequant
])
def test_plan_paths(lib, direction, rows, dim, block, bits, group, signs, a16, path):
    assert B.hadq_plan(direction, rows, dim, block, bits, group, signs, a16) == path


def test_invalid_calls_return_before_launch(lib):
    n0 = B.hadq_launch_count()
    vp = ctypes.c_void_p
    fake = vp(0x10000)
    # NULL outputs
    st = lib.hadq_rotate_quantize(fake, 4, 128, -1, None, 8, -1, None, fake, None, None)
    assert st == B.HADQ_ERR_INVALID_ARG and "NULL" in B.hadq_last_error()
    # misaligned bf16 input / scales / outputs
    st = lib.hadq_rotate_quantize(vp(0x10001), 4, 128, -1, None, 8, -1, fake, fake, None, None)
    assert st == B.HADQ_ERR_MISALIGNED
    st = lib.hadq_rotate_quantize(fake, 4, 128, -1, None, 8, -1, fake, vp(0x10002), None, None)
    assert st == B.HADQ_ERR_MISALIGNED
    st = lib.hadq_rotate_quantize(fake, 4, 128, -1, None, 8, -1, fake, fake, vp(0x10002), None)
    assert st == B.HADQ_ERR_MISALIGNED
    st = lib.hadq_dequant_rotate_inv(fake, fake, 4, 128, -1, None, 8, -1, vp(0x10002), B.HADQ_OUT_F32,
                                     None)
    assert st == B.HADQ_ERR_MISALIGNED
    st = lib.hadq_dequant_rotate_inv(fake, fake, 4, 128, -1, None, 8, -1, fake, 7, None)
    assert st == B.HADQ_ERR_INVALID_ARG
    st = lib.hadq_dequant_rotate_inv(None, fake, 4, 128, -1, None, 8, -1, fake, B.HADQ_OUT_BF16, None)
    assert st == B.HADQ_ERR_INVALID_ARG
    # bad sizes with otherwise valid pointers
    st = lib.hadq_rotate_quantize(fake, 4, 100, 64, None, 8, -1, fake, fake, None, None)
    assert st == B.HADQ_ERR_INVALID_ARG and "does not divide" in B.hadq_last_error()
    assert B.hadq_launch_count() == n0


def test_empty_call_is_a_noop(lib):
    n0 = B.hadq_launch_count()
    assert lib.hadq_rotate_quantize(None, 0, 128, -1, None, 8, -1, None, None, None, None) == B.HADQ_OK
    assert lib.hadq_dequant_rotate_inv(None, None, 0, 4096, -1, None, 4, -1, None, B.HADQ_OUT_BF16,
                                       None) == B.HADQ_OK
    assert B.hadq_launch_count() == n0
    # sizes are still validated for empty calls
    assert lib.hadq_rotate_quantize(None, 0, 100, 64, None, 8, -1, None, None, None, None) == \
        B.HADQ_ERR_INVALID_ARG


def test_last_error_is_cleared_by_a_good_call(lib):
    lib.hadq_rotate_quantize(None, 0, 100, 64, None, 8, -1, None, None, None, None)
    assert B.hadq_last_error()
    lib.hadq_rotate_quantize(None, 0, 128, 64, None, 8, -1, None, None, None, None)
    assert B.hadq_last_error() == ""


# ------------------------------------------------------ decode attention

def test_decode_workspace_size(lib):
    # counters (256-byte block), (m, l) per split and head, O per split and head
    n = B.hadq_kv_decode_workspace_size(1, 32, 8, 131072)
    groups, splits = 8, 256
    assert n == 256 + groups * splits * 4 * 2 * 4 + groups * splits * 4 * 128 * 4
    small = B.hadq_kv_decode_workspace_size(2, 8, 8, 10)   # one split per group
    assert small == 256 + 16 * 4 * 2 * 4 + 16 * 4 * 128 * 4
    assert B.hadq_kv_decode_workspace_size(0, 8, 8, 10) == 0


@pytest.mark.parametrize("args,msg", [
    ((-1, 8, 8, 10), "batch"),
    ((1, 0, 8, 10), "n_q_heads"),
    ((1, 6, 4, 10), "multiple"),
    ((1, 8, 8, 0), "tokens"),
])
def test_decode_workspace_size_rejects(lib, args, msg):
    with pytest.raises(B.HadqError) as e:
        B.hadq_kv_decode_workspace_size(*args)
    assert e.value.status == B.HADQ_ERR_INVALID_ARG and msg in str(e.value)


def _attn(lib, q=0x10000, kc=0x10000, ks=0x10000, vc=0x10000, vs=0x10000, batch=1, nqh=4, nkv=1,
          tokens=16, stride=16, dim=128, block=128, signs=None, bits=4, group=128, scale=0.1,
          out=0x10000, dtype=B.HADQ_OUT_BF16, ws=0x10000, ws_bytes=1 << 20):
    vp = ctypes.c_void_p
    p = lambda v: None if v is None else vp(v)
    return lib.hadq_kv_decode_attention(p(q), p(kc), p(ks), p(vc), p(vs), batch, nqh, nkv, tokens, stride,
                                        dim, block, p(signs), bits, group, scale, p(out), dtype, p(ws),
                                        ws_bytes, None)


@pytest.mark.parametrize("kw,status,msg", [
    (dict(stride=8), B.HADQ_ERR_INVALID_ARG, "token_stride"),
    (dict(tokens=0), B.HADQ_ERR_INVALID_ARG, "tokens"),
    (dict(nqh=6, nkv=4), B.HADQ_ERR_INVALID_ARG, "multiple"),
    (dict(scale=0.0), B.HADQ_ERR_INVALID_ARG, "softmax_scale"),
    (dict(scale=float("inf")), B.HADQ_ERR_INVALID_ARG, "softmax_scale"),
    (dict(dtype=5), B.HADQ_ERR_INVALID_ARG, "out_dtype"),
    (dict(dim=64, block=64, group=64), B.HADQ_ERR_UNSUPPORTED, "dim 128"),
    (dict(bits=5), B.HADQ_ERR_INVALID_ARG, "bits"),
    (dict(group=16), B.HADQ_ERR_UNSUPPORTED, "group 128, 64 or 32"),
    (dict(group=64, ks=0x10004), B.HADQ_ERR_MISALIGNED, "16-byte aligned"),
    (dict(group=64, stride=17, tokens=17), B.HADQ_ERR_MISALIGNED, "token_stride"),
    (dict(block=64), B.HADQ_ERR_UNSUPPORTED, "block 128"),
    (dict(block=48), B.HADQ_ERR_INVALID_ARG, "power of two"),
    (dict(ws=None), B.HADQ_ERR_INVALID_ARG, "NULL"),
    (dict(q=0x10004), B.HADQ_ERR_MISALIGNED, "q must"),
    (dict(kc=0x10008), B.HADQ_ERR_MISALIGNED, "codes"),
    (dict(vs=0x10002), B.HADQ_ERR_MISALIGNED, "scales"),
    (dict(signs=0x10002), B.HADQ_ERR_MISALIGNED, "signs"),
    (dict(out=0x10008, dtype=B.HADQ_OUT_F32), B.HADQ_ERR_MISALIGNED, "out"),
    (dict(ws=0x10010), B.HADQ_ERR_MISALIGNED, "workspace"),
    (dict(ws_bytes=100), B.HADQ_ERR_INVALID_ARG, "workspace of 100 bytes"),
])
def test_decode_attention_rejects_before_launch(lib, kw, status, msg):
    n0 = B.hadq_launch_count()
    st = _attn(lib, **kw)
    assert st == status, (st, B.hadq_last_error())
    assert msg in B.hadq_last_error()
    assert B.hadq_launch_count() == n0


def test_decode_attention_empty_batch_is_a_noop(lib):
    n0 = B.hadq_launch_count()
    assert _attn(lib, batch=0, q=None, kc=None, ks=None, vc=None, vs=None, out=None, ws=None) == B.HADQ_OK
    assert B.hadq_launch_count() == n0


def test_noalloc_entry_validates_before_launch(lib):
    vp = ctypes.c_void_p
    f = vp(0x10000)
    n0 = B.hadq_launch_count()
    call = lambda q, tokens, dim, block, group, bits: lib.hadq_kv_decode_attention_noalloc(
        q, f, f, f, f, 1, 4, 1, tokens, 16, dim, block, None, bits, group, 0.1, f, B.HADQ_OUT_BF16, None)
    assert call(f, 0, 128, 128, 128, 4) == B.HADQ_ERR_INVALID_ARG
    assert call(f, 16, 64, 64, 64, 4) == B.HADQ_ERR_UNSUPPORTED
    assert call(None, 16, 128, 128, 128, 4) == B.HADQ_ERR_INVALID_ARG
    assert call(vp(0x10002), 16, 128, 128, 128, 4) == B.HADQ_ERR_MISALIGNED
    assert B.hadq_launch_count() == n0
    # batch 0 is an empty call with no pointers at all
    assert lib.hadq_kv_decode_attention_noalloc(None, None, None, None, None, 0, 4, 1, 16, 16, 128, 128, None,
                                                4, 128, 0.1, None, B.HADQ_OUT_BF16, None) == B.HADQ_OK


# ------------------------------------------------------------ kept tokens

def _keep(lib, x=0x10000, heads=2, tokens=16, dim=128, block=128, signs=None, bits=4, group=128, slot=0x10000,
          n_keep=2, codes=0x10000, scales=0x10000, kept=0x10000):
    vp = ctypes.c_void_p
    p = lambda v: None if v is None else vp(v)
    return lib.hadq_rotate_quantize_keep(p(x), heads, tokens, dim, block, p(signs), bits, group, p(slot), n_keep,
                                         p(codes), p(scales), p(kept), None)


@pytest.mark.parametrize("kw,status,msg", [
    (dict(slot=None), B.HADQ_ERR_INVALID_ARG, "keep_slot"),
    (dict(kept=None), B.HADQ_ERR_INVALID_ARG, "kept"),
    (dict(n_keep=-1), B.HADQ_ERR_INVALID_ARG, "n_keep"),
    (dict(heads=-1), B.HADQ_ERR_INVALID_ARG, "heads"),
    (dict(slot=0x10002), B.HADQ_ERR_MISALIGNED, "keep_slot"),
    (dict(kept=0x10008), B.HADQ_ERR_MISALIGNED, "kept"),
    (dict(group=32), B.HADQ_ERR_UNSUPPORTED, "wide groups"),
    (dict(dim=96, block=32, group=96), B.HADQ_ERR_UNSUPPORTED, "wide groups"),
    (dict(dim=128 * 48, block=128, group=128 * 48), B.HADQ_ERR_UNSUPPORTED, "wide groups"),
    (dict(block=256, dim=256, group=256), B.HADQ_ERR_UNSUPPORTED, "wide groups"),
    (dict(x=0x10008), B.HADQ_ERR_UNSUPPORTED, "16-byte"),
    (dict(bits=5), B.HADQ_ERR_INVALID_ARG, "bits"),
])
def test_keep_entry_rejects_before_launch(lib, kw, status, msg):
    n0 = B.hadq_launch_count()
    assert _keep(lib, **kw) == status, B.hadq_last_error()
    assert msg in B.hadq_last_error()
    assert B.hadq_launch_count() == n0


def test_keep_entries_empty_calls(lib):
    n0 = B.hadq_launch_count()
    assert _keep(lib, heads=0, x=None, slot=None, codes=None, scales=None, kept=None) == B.HADQ_OK
    assert lib.hadq_dequant_rotate_inv_keep(None, None, None, None, 0, 3, 0, 128, 128, None, 4, 128, None,
                                            B.HADQ_OUT_BF16, None) == B.HADQ_OK
    assert B.hadq_launch_count() == n0


def test_hyquant_keep_slots():
    slots, n = B.hyquant_keep_slots(12, n_sink=2, window=3, vertical=[7, 1])
    assert n == 6
    assert slots.tolist() == [0, 1, -1, -1, -1, -1, -1, 2, -1, 3, 4, 5]
    slots, n = B.hyquant_keep_slots(5, n_sink=9, window=9)
    assert n == 5 and slots.tolist() == [0, 1, 2, 3, 4]
    with pytest.raises(ValueError):
        B.hyquant_keep_slots(5, vertical=[5])


# ------------------------------------------------------------ asymmetric quantiser

@pytest.mark.parametrize("kw,status,msg", [
    (dict(zp=None), B.HADQ_ERR_INVALID_ARG, "NULL"),
    (dict(group=64), B.HADQ_ERR_UNSUPPORTED, "asymmetric"),
    (dict(dim=96, block=32, group=96), B.HADQ_ERR_UNSUPPORTED, "asymmetric"),
    (dict(block=256, dim=256, group=256), B.HADQ_ERR_UNSUPPORTED, "asymmetric"),
    (dict(x=0x10008), B.HADQ_ERR_UNSUPPORTED, "16-byte"),
    (dict(scales=0x10002), B.HADQ_ERR_MISALIGNED, "scales"),
    (dict(bits=3), B.HADQ_ERR_INVALID_ARG, "bits"),
])
def test_asym_entry_rejects_before_launch(lib, kw, status, msg):
    vp = ctypes.c_void_p
    a = dict(x=0x10000, rows=4, dim=128, block=128, bits=4, group=128, codes=0x10000, scales=0x10000, zp=0x10000)
    a.update(kw)
    p = lambda v: None if v is None else vp(v)
    n0 = B.hadq_launch_count()
    st = lib.hadq_rotate_quantize_asym(p(a["x"]), a["rows"], a["dim"], a["block"], None, a["bits"], a["group"],
                                       p(a["codes"]), p(a["scales"]), p(a["zp"]), None)
    assert st == status, B.hadq_last_error()
    assert msg in B.hadq_last_error()
    assert B.hadq_launch_count() == n0


def test_asym_empty_calls(lib):
    assert lib.hadq_rotate_quantize_asym(None, 0, 128, 128, None, 4, 128, None, None, None, None) == B.HADQ_OK
    assert lib.hadq_dequant_rotate_inv_asym(None, None, None, 0, 128, 128, None, 4, 128, None, B.HADQ_OUT_F32,
                                            None) == B.HADQ_OK


# ------------------------------------------------------------ Kronecker rotation

@pytest.mark.parametrize("a,b,bits,group,status,msg", [
    (0, 64, 4, -1, B.HADQ_ERR_INVALID_ARG, "a must be"),
    (300, 64, 4, -1, B.HADQ_ERR_INVALID_ARG, "a must be"),
    (12, 48, 4, -1, B.HADQ_ERR_INVALID_ARG, "power of two"),
    (12, 1, 8, -1, B.HADQ_ERR_INVALID_ARG, "power of two"),
    (200, 256, 4, -1, B.HADQ_ERR_INVALID_ARG, "at most"),
    (12, 64, 4, 7, B.HADQ_ERR_INVALID_ARG, "does not divide"),
    (255, 128, 4, -1, B.HADQ_ERR_UNSUPPORTED, "shared memory"),
])
def test_kron_entry_validates(lib, a, b, bits, group, status, msg):
    vp = ctypes.c_void_p
    f = vp(0x10000)
    n0 = B.hadq_launch_count()
    st = lib.hadq_rotate_quantize_kron(f, 4, a, f, b, None, bits, group, f, f, None, None)
    assert st == status, B.hadq_last_error()
    assert msg in B.hadq_last_error()
    assert B.hadq_launch_count() == n0


@pytest.mark.parametrize("direction,a,b,group,a16,variant", [
    (0, 20, 256, 128, True, "mma"),     # the 5120-column workload
    (0, 8, 64, 64, True, "mma"),
    (0, 32, 128, 128, True, "mma"),
    (0, 1, 512, 512, True, "mma"),
    (0, 20, 256, 128, False, "smem"),   # pointers not 16-byte aligned
    (0, 12, 32, 64, True, "reg16"),     # 384 columns: not a multiple of 512
    (0, 40, 128, 128, True, "reg16"),   # a > 32
    (0, 28, 512, 128, True, "reg16"),   # 14336 columns: above 8192
    (0, 7, 32, 56, True, "smem"),       # group of 56 columns
    (0, 16, 8, 64, True, "smem"),       # b < 16
    (1, 20, 256, 128, True, "smem"),    # every inverse
])
def test_kron_plan_variants(lib, direction, a, b, group, a16, variant):
    assert B.hadq_kron_plan(direction, 100, a, b, 4, group, a16) == variant


def test_kron_plan_rejects_like_the_call(lib):
    with pytest.raises(B.HadqError) as e:
        B.hadq_kron_plan(0, 4, 12, 48)
    assert e.value.status == B.HADQ_ERR_INVALID_ARG and "power of two" in str(e.value)
    with pytest.raises(B.HadqError) as e:
        B.hadq_kron_plan(2, 4, 12, 64)
    assert e.value.status == B.HADQ_ERR_INVALID_ARG
    with pytest.raises(B.HadqError) as e:
        B.hadq_kron_plan(0, 4, 255, 128)
    assert e.value.status == B.HADQ_ERR_UNSUPPORTED
