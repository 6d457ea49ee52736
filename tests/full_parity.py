"""Worker side of the full-size parity count (tests/test_full_parity_gpu.py).

A worker regenerates a range of input rows from the seeded generator, runs the
float64 oracle on them and compares every code, every scale and (for the
KV-cache workload) every bf16 reconstruction with the GPU's.  It returns
counts, never raises on a mismatch, so that the parent can report the totals
of a whole workload.  Workers run in processes started with ``spawn``, each
with one BLAS thread.
"""

from __future__ import annotations

import numpy as np

import oracle as O
from hadamard_rotation_outlier_b200 import synthetic as S

from parity import BOUNDARY, REL_TOL, bf16_bits_rne, bf16_ulp, decode_bf16, gpu_codes_to_int

_limits = None

# workload -> totals of the current session (filled by the test, printed by the
# session summary in conftest.py)
SUMMARY = {}


def init_worker():
    """Keep each worker on one BLAS thread (the pool supplies the parallelism)."""
    global _limits
    from threadpoolctl import threadpool_limits
    _limits = threadpool_limits(1)


def oracle_method(wl) -> str:
    """Dense Sylvester products for blocks up to 512 (one small matrix), the
    FWHT oracle (pinned to the dense product) for wider blocks."""
    B = wl.dim if wl.block == -1 else wl.block
    return "dense" if B <= 512 else "fwht"


def compare_rows(name: str, ti: int, r0: int, r1: int, g_codes: np.ndarray, g_scales: np.ndarray,
                 g_out_bits: np.ndarray | None = None) -> dict:
    """Counts over rows [r0, r1) of tensor ``ti`` of workload ``name``.

    * ``mismatches``: codes that differ from the oracle's;
    * ``far``: of those, the ones whose oracle pre-round value is more than
      1e-4 from a .5 boundary, or that differ by more than one;
    * ``scale_bad``: scales off by more than 1e-5 relative;
    * ``bf16_bad``: reconstructed bf16 values outside one bf16 ulp plus the
      float32 allowance of the rounded oracle (dequantised from the GPU's own
      codes and scales).
    """
    wl = S.WORKLOADS[name]
    x = S.tensor_rows(wl, ti, r0, r1, threads=1)
    signs = S.signs(wl)
    method = oracle_method(wl)
    ref = O.rotate_quantize(x, block=wl.block, signs=signs, bits=wl.bits, group=wl.group, method=method)
    g_q = gpu_codes_to_int(g_codes, wl.bits, wl.dim)
    o_q = ref["q"]
    mism = g_q != o_q
    n = int(mism.sum())
    far = 0
    if n:
        d = O.half_boundary_distance(ref["pre_round"][mism])
        far = int(np.sum((d > BOUNDARY) | (np.abs(g_q[mism] - o_q[mism]) != 1)))
    gs = np.asarray(g_scales, dtype=np.float64).reshape(ref["scales"].shape)
    os_ = ref["scales"].astype(np.float64)
    err = np.abs(gs - os_)
    scale_bad = int(np.sum(err > np.maximum(REL_TOL * np.abs(os_), 2.0 ** -149)))
    with np.errstate(invalid="ignore", divide="ignore"):
        rel = np.where(os_ == 0, 0.0, err / np.abs(os_))
    out = {"mismatches": n, "elements": int(o_q.size), "far": far, "scale_bad": scale_bad,
           "max_scale_rel": float(rel.max()) if rel.size else 0.0}
    if g_out_bits is not None:
        rec = O.dequant_rotate_inv(g_codes, g_scales, wl.dim, block=wl.block, signs=signs, bits=wl.bits,
                                   group=wl.group, method=method)
        g = decode_bf16(np.asarray(g_out_bits, dtype=np.uint16).reshape(rec.shape))
        rms = np.sqrt(np.mean(rec * rec, axis=-1, keepdims=True))
        allowed = bf16_ulp(rec) + REL_TOL * np.maximum(np.abs(rec), rms)
        out["bf16_bad"] = int(np.sum(np.abs(g - rec) > allowed))
        out["bf16_exact"] = int(np.sum(np.asarray(g_out_bits, dtype=np.uint16).reshape(rec.shape)
                                       == bf16_bits_rne(rec)))
    return out
