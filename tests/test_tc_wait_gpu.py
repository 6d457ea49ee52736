"""Bounded waits of the tcgen05 4096-block kernel.

The self-test entry withholds the load of the kernel's only tile, so the
waits for it run out after about a second: the kernel must record the fault,
leave without writing, free its tensor memory and leave the context usable.
The failure is made on the host (a load that is never issued); nothing
faults or hangs the GPU.
"""

import numpy as np
import pytest
import torch

import oracle as O
from hadamard_rotation_outlier_b200 import binding as B
from hadamard_rotation_outlier_b200 import synthetic as S
from hadamard_rotation_outlier_b200.steps import bits_to_bf16_tensor

from parity import check_codes, check_scales, gpu_codes_to_int

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_withheld_load_is_reported_and_the_context_stays_usable():
    scratch = torch.full((65536,), 0x5A, dtype=torch.uint8, device="cuda")
    assert B.hadq_selftest_bounded_wait(scratch) == B.HADQ_ERR_DEVICE
    B.hadq_device_status()  # the record was cleared by the report
    torch.cuda.synchronize()
    # the codes and scales areas were not written
    assert bool((scratch[32768:40976] == 0x5A).all())

    # the next call runs normally on the same context
    rows, dim = 9, 4096
    x_bits = S.random_bf16(rows, dim, 5)
    s = S.random_signs(dim, 5)
    assert B.hadq_plan(0, rows, dim, -1, 4, -1, True, True) == "h4096_tc"
    ref = O.rotate_quantize(x_bits, block=-1, signs=s, bits=4, group=-1, method="dense")
    codes, scales = B.hadq_rotate_quantize(bits_to_bf16_tensor(x_bits, "cuda"), block=-1,
                                           signs=torch.from_numpy(s).cuda(), bits=4, group=-1)
    B.hadq_device_status()
    check_scales(scales.cpu().numpy(), ref["scales"])
    check_codes(gpu_codes_to_int(codes.cpu().numpy(), 4, dim), ref["q"], ref["pre_round"], None)
