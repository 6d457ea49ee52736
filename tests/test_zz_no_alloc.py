"""The allocation-free decode-attention entry point (static library scratch).

Runs last: it checks that the scratch counters are left at zero by every call,
so that later calls in the same process see a clean scratch.  Each call is
compared with the float64 oracle, and memory is checked to be unchanged across
calls (nothing allocated per call): torch's allocator always, the device-wide
free memory when no other process is on the device.
"""

import gc

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


def _alone_on_device() -> bool:
    """True when NVML lists at most one compute process on device 0 (this one),
    so that the device-wide free-memory figure reflects only this process."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())
        return len(pynvml.nvmlDeviceGetComputeRunningProcesses(h)) <= 1
    except Exception:
        return False


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _case(batch, nqh, nkv, tokens, seed, with_signs):
    signs = S.random_signs(DIM, seed) if with_signs else None
    kc, ks = S.random_int4_cache(batch, nkv, tokens, DIM, seed)
    vc, vs = S.random_int4_cache(batch, nkv, tokens, DIM, seed + 1)
    qbits = S.decode_query(batch, nqh, DIM, seed)
    want = O.kv_decode_attention(qbits, kc, ks, vc, vs, DIM, 128, signs, 4, 128)
    scores = O.kv_decode_scores(qbits, kc, ks, DIM, 128, signs, 4, 128)
    values = O.dequant_rotate_inv(vc.reshape(-1, DIM // 2), vs.reshape(-1), DIM, 128, signs, 4, 128,
                                  method="fwht").reshape(batch, nkv, tokens, DIM)
    allow = attention_allowance(want, scores, values, nqh // nkv)
    args = [_dev(qbits.view(np.int16)).view(torch.bfloat16), _dev(kc), _dev(ks), _dev(vc), _dev(vs)]
    return args, None if signs is None else _dev(signs), want, allow


@pytest.mark.parametrize("batch,nqh,nkv,tokens,with_signs", [
    (1, 32, 8, 4096, False),
    (2, 8, 2, 1001, True),
    (1, 16, 2, 37, False),
])
def test_noalloc_matches_oracle_and_allocates_nothing(batch, nqh, nkv, tokens, with_signs):
    args, sg, want, allow = _case(batch, nqh, nkv, tokens, 300 + tokens, with_signs)
    out = torch.empty((batch, nqh, DIM), dtype=torch.float32, device="cuda")
    B.hadq_kv_decode_attention_noalloc(*args, out=out, block=128, signs=sg, bits=4, group=128)
    torch.cuda.synchronize()
    gc.collect()  # tensors of earlier tests freed now, not during the calls below
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    n0 = B.hadq_launch_count()
    for _ in range(3):
        B.hadq_kv_decode_attention_noalloc(*args, out=out, block=128, signs=sg, bits=4, group=128)
    torch.cuda.synchronize()
    assert B.hadq_launch_count() == n0 + 3
    # nothing allocated through torch (a collection of an earlier test's
    # garbage could still lower the figure, never raise it)
    assert torch.cuda.memory_allocated() <= alloc0
    if _alone_on_device():
        # a device allocation takes at least one 2 MiB page; other processes
        # on the device would move this figure, so it is read only when alone
        assert torch.cuda.mem_get_info()[0] > free0 - (2 << 20)
    check_attention(out.cpu().numpy(), want, allow, "no-alloc entry")


def test_noalloc_equals_workspace_entry():
    args, sg, _, _ = _case(1, 8, 2, 2500, 77, False)
    a = torch.empty((1, 8, DIM), dtype=torch.bfloat16, device="cuda")
    b = B.hadq_kv_decode_attention(*args, block=128, bits=4, group=128)
    B.hadq_kv_decode_attention_noalloc(*args, out=a, block=128, bits=4, group=128)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 60000 head groups of one split each need about 125 MB of partials.
    q = torch.zeros((2000, 30, DIM), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((2000, 30, 16, DIM // 2), dtype=torch.uint8, device="cuda")
    ks = torch.ones((2000, 30, 16), dtype=torch.float32, device="cuda")
    out = torch.full((2000, 30, DIM), 3.0, dtype=torch.float32, device="cuda")
    n0 = B.hadq_launch_count()
    with pytest.raises(B.HadqError) as e:
        B.hadq_kv_decode_attention_noalloc(q, kc, ks, kc, ks, out=out, block=128, bits=4, group=128)
    assert e.value.status == B.HADQ_ERR_UNSUPPORTED and "scratch" in str(e.value)
    assert B.hadq_launch_count() == n0
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
