"""Comparison rules between the CUDA path and the float64 oracle.

* Rotated values y (float32 from the GPU) and dequantised reconstructions in
  float32: |g - o| <= 1e-5 * max(|o|, rms of o over the row).  The row-RMS floor
  keeps entries near zero from failing on absolute rounding noise.
* Scales: |g - o| <= max(1e-5 * |o|, 2^-149) (exact 0 for an all-zero group);
  the floor is one float32 subnormal step, the storage resolution of a scale
  below 2^-126.
* Codes: bit-exact, except where the oracle's pre-round value y/scale lies
  within 1e-4 of a rounding boundary k + 0.5; such a code may differ by one.
  The number of mismatches must be at most 1e-5 of the elements, with at least
  one such mismatch tolerated on small cases.
* bf16 reconstructions: within one bf16 ulp of the oracle rounded to bf16
  (round to nearest, ties to even), where the value's float32 error allowed
  above (1e-5 of max(|o|, row RMS)) is added to that ulp: a value near zero
  may carry an absolute float32 error several bf16 ulps wide.
* Asymmetric quantiser: scales as above; a zero point may differ from the
  oracle's by one only where the oracle's pre-round value -lo/scale lies
  within 1e-4 of a .5 boundary; codes are then compared, under the code rule
  above, with round(y/scale) plus the GPU's zero point, clamped.
* Decode attention: the rule for float32 values above plus the conditioning
  of softmax on float32 scores.  A score s held in float32 (log2 units, after
  a few roundings) is off by at most 16 u |s| (u = 2^-24); a weight then moves
  by p_t ln2 (ds_t - sum_t' p_t' ds_t'), so output element d moves by at most
  2 ln2 * 16 u * (sum_t p_t |s_t|) * max_t |v_td - o_d|.  That term is added
  to the allowance of each output element (v: dequantised values in the
  original basis).
"""

from __future__ import annotations

import numpy as np

import oracle as O

REL_TOL = 1e-5
BOUNDARY = 1e-4
MISMATCH_RATE = 1e-5


def gpu_codes_to_int(codes: np.ndarray, bits: int, dim: int) -> np.ndarray:
    c = np.asarray(codes)
    if bits == 8:
        return c.reshape(-1, dim).astype(np.int64)
    return O.unpack_int4(c.reshape(-1, dim // 2))


def check_values(g: np.ndarray, o: np.ndarray, what: str, tol: float = REL_TOL) -> float:
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    if o.size == 0:
        return 0.0
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True))
    ref = np.maximum(np.abs(o), rms)
    err = np.abs(g - o)
    bad = err > tol * ref
    if np.any(bad):
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} values off; first at {tuple(i)}: "
                             f"gpu {g[tuple(i)]!r} oracle {o[tuple(i)]!r}")
    with np.errstate(invalid="ignore", divide="ignore"):
        return float(np.nanmax(np.where(ref > 0, err / ref, 0.0)))


def check_scales(g: np.ndarray, o: np.ndarray) -> float:
    g = np.asarray(g, dtype=np.float64).reshape(o.shape)
    o = np.asarray(o, dtype=np.float64)
    zero = o == 0
    assert np.all(g[zero] == 0), "all-zero groups must have scale 0"
    err = np.abs(g - o)
    ok = err <= np.maximum(REL_TOL * np.abs(o), 2.0 ** -149)
    assert np.all(ok), f"scales: {int((~ok).sum())} off, max rel err {(err / np.abs(o))[~ok].max():.3e}"
    with np.errstate(invalid="ignore", divide="ignore"):
        rel = np.where(zero, 0.0, err / np.abs(o))
    return float(rel.max()) if rel.size else 0.0


def check_codes(g_q: np.ndarray, o_q: np.ndarray, pre_round: np.ndarray, max_mismatches=None) -> int:
    """Returns the number of (allowed) boundary mismatches.  ``max_mismatches``
    overrides the count limit for inputs built to sit on ties."""
    g_q = np.asarray(g_q).reshape(o_q.shape)
    mism = g_q != o_q
    n = int(mism.sum())
    if n:
        d = O.half_boundary_distance(pre_round[mism])
        far = d > BOUNDARY
        if np.any(far):
            idx = np.argwhere(mism)[np.argmax(far)]
            raise AssertionError(f"codes: {int(far.sum())} mismatches away from a .5 boundary; e.g. "
                                 f"at {tuple(idx)} gpu {g_q[tuple(idx)]} oracle {o_q[tuple(idx)]} "
                                 f"pre-round {pre_round[tuple(idx)]!r}")
        assert np.all(np.abs(g_q[mism] - o_q[mism]) == 1)
    allowed = max(1.0, MISMATCH_RATE * o_q.size) if max_mismatches is None else max_mismatches
    assert n <= allowed, f"codes: {n} boundary mismatches > {allowed:g} allowed"
    return n


def bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bits with one rounding (to nearest, ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    normal = np.ldexp(np.round(m * 256.0) / 256.0, e)   # 8 significant bits
    sub = np.round(x * 2.0 ** 133) * 2.0 ** -133        # bf16 subnormal grid
    y = np.where(np.abs(x) < 2.0 ** -126, sub, normal).astype(np.float32)  # exact
    return (y.view(np.uint32) >> 16).astype(np.uint16)


def _ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (subnormal spacing below 2^-126)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(np.maximum(a, 2.0 ** -126))
    return np.ldexp(1.0, e - 8)


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_bf16(g_bits: np.ndarray, o: np.ndarray, what: str) -> int:
    """Returns the largest distance in bf16 steps from the rounded oracle."""
    o = np.asarray(o, dtype=np.float64)
    ref = bf16_bits_rne(o)
    g_bits = np.asarray(g_bits, dtype=np.uint16).reshape(ref.shape)
    g = decode_bf16(g_bits)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True))
    allowed = bf16_ulp(o) + REL_TOL * np.maximum(np.abs(o), rms)
    bad = np.abs(g - o) > allowed
    if np.any(bad):
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} values off by more than one bf16 ulp; "
                             f"first at {i}: gpu {g[i]!r} oracle {o[i]!r}")
    d = np.abs(_ordered(g_bits) - _ordered(ref))
    return int(d.max()) if d.size else 0


ATTN_SCORE_ULPS = 16
U32 = 2.0 ** -24


def attention_allowance(o: np.ndarray, scores: np.ndarray, values: np.ndarray, group: int) -> np.ndarray:
    """Per-element allowance of the decode-attention output (see module note).

    ``o`` [b, h, d] oracle output; ``scores`` [b, h, T] oracle scores (natural
    units); ``values`` [b, kvh, T, d] dequantised values in the original
    basis; query head h reads KV head h // group.
    """
    s2 = scores * np.log2(np.e)
    p = np.exp(scores - scores.max(axis=-1, keepdims=True))
    p /= p.sum(axis=-1, keepdims=True)
    sbar = np.sum(p * np.abs(s2), axis=-1)                        # [b, h]
    nb, nh, d = o.shape
    spread = np.empty_like(o)
    for b in range(nb):
        for h in range(nh):
            spread[b, h] = np.max(np.abs(values[b, h // group] - o[b, h]), axis=0)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True))
    return (REL_TOL * np.maximum(np.abs(o), rms)
            + 2 * np.log(2.0) * ATTN_SCORE_ULPS * U32 * sbar[..., None] * spread)


def check_attention(g: np.ndarray, o: np.ndarray, allowance: np.ndarray, what: str,
                    bf16: bool = False) -> float:
    """Compare a decode-attention output (float32 values or bf16 bits) with
    the oracle under :func:`attention_allowance`; bf16 adds one bf16 ulp.
    Returns the largest error as a fraction of the allowance."""
    o = np.asarray(o, dtype=np.float64)
    if bf16:
        gv = decode_bf16(np.asarray(g, dtype=np.uint16).reshape(o.shape))
        allowance = allowance + bf16_ulp(o)
    else:
        gv = np.asarray(g, dtype=np.float64).reshape(o.shape)
    err = np.abs(gv - o)
    bad = err > allowance
    if np.any(bad):
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} values off; first at {i}: gpu {gv[i]!r} "
                             f"oracle {o[i]!r} allowance {allowance[i]:.3e}")
    return float(np.max(err / allowance)) if err.size else 0.0


def check_asym(g_q: np.ndarray, g_scales: np.ndarray, g_zp: np.ndarray, ref: dict, bits: int,
               max_mismatches=None) -> int:
    """Asymmetric codes, scales and zero points against ``oracle.rotate_quantize_asym``.

    ``g_q``: unpacked GPU codes [rows, dim] (int); ``g_scales``, ``g_zp``
    [rows, dim/G].  Returns the number of tolerated code mismatches.
    """
    o_zp = ref["zero_points"].astype(np.int64).reshape(-1)
    gz = np.asarray(g_zp).astype(np.int64).reshape(o_zp.shape)
    check_scales(np.asarray(g_scales).reshape(ref["scales"].shape), ref["scales"])
    mz = gz != o_zp
    if np.any(mz):
        d = O.half_boundary_distance(ref["zp_pre_round"].reshape(-1)[mz])
        assert np.all(d <= BOUNDARY) and np.all(np.abs(gz[mz] - o_zp[mz]) == 1), "zero point mismatch"
    v = ref["pre_round"]
    rows, dim = v.shape
    ngroups = ref["scales"].shape[-1]
    G = dim // ngroups
    zp_full = np.repeat(gz.reshape(rows, ngroups), G, axis=1)
    nz = np.repeat(ref["scale64"].reshape(rows, ngroups) > 0, G, axis=1)
    o_q = np.where(nz, np.clip(np.round(v) + zp_full, 0, 2 ** bits - 1), 0).astype(np.int64)
    return check_codes(np.asarray(g_q).reshape(rows, dim), o_q, v, max_mismatches)
