"""Code mismatches over every element of the five synthetic workloads.

The parity rule for codes is bit-exact agreement with the float64 oracle,
except at elements whose pre-round value lies within 1e-4 of a .5 boundary;
the number of such mismatches over a workload is reported and must stay at
or below 1e-5 of its elements.  The sampled tests compare rotated values and
reconstructions element by element; this one runs the launch configuration
the benchmark times (one quantise launch over all rows, plus the bf16
dequantise launch of the KV-cache workload) and streams every row through the
oracle in a process pool started with ``spawn``:

* every code: mismatch count, and no mismatch away from a boundary or by more
  than one;
* every scale within 1e-5 relative;
* the KV-cache workload: every bf16 reconstruction within one bf16 ulp plus
  the float32 allowance of the oracle's dequantisation of the GPU's codes.

The per-workload counts are printed at the end of the session.  With
``HADQ_PARITY_RECORD=<file>`` each count is also appended to that file as a
record line keyed by the kernel sources it was taken with.
"""

import datetime
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

from hadamard_rotation_outlier_b200 import records as R
from hadamard_rotation_outlier_b200 import synthetic as S
from hadamard_rotation_outlier_b200.steps import WorkloadStep, bf16_tensor_to_bits

import full_parity as FP
from parity import MISMATCH_RATE

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

FIVE = ["c1_tok256_h4096_b128_int4", "c2_qk_h32_s8192_d128_int8", "c3_tok16384_h4096_full_signs_int4",
        "c4_kv_h8_t131072_d128_int4_g128", "c5_tok32768_w11008_b128_signs_int4_g128"]
TASK_ELEMENTS = 1 << 22

# workload -> totals, printed by the session summary in conftest.py
RESULTS = FP.SUMMARY


@pytest.fixture(scope="module")
def pool():
    n = max(1, min(32, len(os.sched_getaffinity(0))))
    with mp.get_context("spawn").Pool(n, initializer=FP.init_worker) as p:
        yield p


def _row_tasks(wl):
    per = max(S.CHUNK_ROWS, (TASK_ELEMENTS // wl.dim) // S.CHUNK_ROWS * S.CHUNK_ROWS)
    base = 0
    for ti, t in enumerate(wl.tensors):
        for r0 in range(0, t.rows, per):
            r1 = min(t.rows, r0 + per)
            yield ti, r0, r1, base + r0, base + r1
        base += t.rows


@pytest.mark.parametrize("name", FIVE)
def test_every_code_of_the_workload(name, pool):
    wl = S.WORKLOADS[name]
    st = WorkloadStep(wl, "cuda")
    st.step()
    torch.cuda.synchronize()
    codes = st.codes.cpu().numpy()
    scales = st.scales.cpu().numpy()
    out_bits = bf16_tensor_to_bits(st.out) if wl.dequant else None
    del st
    torch.cuda.empty_cache()

    jobs = [pool.apply_async(FP.compare_rows, (name, ti, r0, r1, codes[a:b], scales[a:b],
                                               None if out_bits is None else out_bits[a:b]))
            for ti, r0, r1, a, b in _row_tasks(wl)]
    tot = {}
    for j in jobs:
        for k, v in j.get().items():
            tot[k] = max(tot.get(k, 0.0), v) if k == "max_scale_rel" else tot.get(k, 0) + v
    assert tot["elements"] == wl.elements
    RESULTS[name] = tot

    path = os.environ.get("HADQ_PARITY_RECORD")
    if path:
        when = datetime.datetime.now(datetime.timezone.utc).strftime("%Y-%m-%dT%H:%MZ")
        with open(path, "a") as f:
            f.write(R.parity_line(name, R.workload_family(wl), tot, when) + "\n")

    assert tot["far"] == 0, f"{name}: {tot['far']} code mismatches away from a .5 boundary or by more than one"
    assert tot["scale_bad"] == 0, f"{name}: {tot['scale_bad']} scales off by more than 1e-5 relative"
    assert tot["mismatches"] <= MISMATCH_RATE * tot["elements"], (
        f"{name}: {tot['mismatches']} boundary mismatches in {tot['elements']} elements "
        f"(rate {tot['mismatches'] / tot['elements']:.2e} > {MISMATCH_RATE:g})")
    if wl.dequant:
        assert tot["bf16_bad"] == 0, f"{name}: {tot['bf16_bad']} bf16 reconstructions off"
