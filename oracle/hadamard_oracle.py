"""Plain float64 CPU oracle for the online rotate-then-quantize step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code,
tables or constants with the CUDA library.

Every function is written to be checked by eye against the pages it cites.
Page names used in citations:

* [Hartmann rotation] -- "哈特曼旋转，轻量级QAT，流式注意力" (Hadamard rotation
  of Q/K, lightweight QAT, streaming attention), lzwjava.github.io.
* [QuaRot hands-on] -- "手把手教你用QuaRot实现LLM的4位量化：从原理到代码实践",
  0539edu.com.
* [Outlier nemesis] -- "旋转量化：大模型低比特量化中的离群值克星", yfxerp.com.
* [msModelSlim QuaRot] -- "QuaRot：基于旋转的离群值抑制算法说明",
  msmodelslim.readthedocs.io.
* [HyQuant] -- "HyQuant:面向 LLM 注意力的混合精度量化" (HyQuant: mixed-precision
  quantisation for LLM attention), ai-feeds.com.

Readings taken where the pages are silent or ambiguous (each is also listed
in the design notes of the repository):

* rounding is round-half-to-even (numpy ``round`` / torch ``round`` as used
  on [Outlier nemesis] §2.2 and [Hartmann rotation] §2);
* the code range is symmetric, ``[-(2^(b-1)-1), 2^(b-1)-1]`` ([Outlier
  nemesis] §2.2 clips to that range); -8 is never produced for INT4;
* an all-zero group gets scale 0 and codes 0;
* H is the orthonormal Sylvester matrix (entries +-1/sqrt(n)), as built on
  [Hartmann rotation] §1;
* the optional +-1 sign vector has the length of the row and multiplies the
  input before H (randomised Hadamard, [QuaRot hands-on] §2.1);
* the scale group is independent of the Hadamard block;
* INT4 codes are packed two per byte, even element in the low nibble.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
against closed forms, library routines, brute force or values the pages print.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "sylvester",
    "fwht",
    "rotate",
    "inverse_rotate",
    "quantize",
    "pack_int4",
    "unpack_int4",
    "rotate_quantize",
    "dequant_rotate_inv",
    "quant_error",
    "half_boundary_distance",
    "kron_rotate",
    "kron_inverse_rotate",
    "rotate_quantize_kron",
    "dequant_rotate_inv_kron",
    "quantize_asym",
    "pack_uint4",
    "unpack_uint4",
    "rotate_quantize_asym",
    "dequant_rotate_inv_asym",
    "rotate_quantize_keep",
    "dequant_rotate_inv_keep",
    "dequant_rotated",
    "kv_decode_scores",
    "kv_decode_attention",
]


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode raw bfloat16 bit patterns (uint16) to float64, exactly.

    A bfloat16 is the top half of an IEEE float32, so the decode is the
    16-bit pattern placed in the high half of a float32 word.
    """
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sylvester(n: int) -> np.ndarray:
    """Dense normalised Sylvester-Hadamard matrix H_n (float64).

    [Hartmann rotation] §1: H_1 = [1]; H_2n = [[H_n, H_n], [H_n, -H_n]] / sqrt(2);
    n must be a power of two.  The result is orthogonal (H H^T = I) with every
    entry +-1/sqrt(n).
    """
    if n < 1 or (n & (n - 1)) != 0:
        raise ValueError(f"Sylvester Hadamard needs a power of two, got {n}")
    if n == 1:
        return np.ones((1, 1), dtype=np.float64)
    h = sylvester(n // 2)
    top = np.concatenate([h, h], axis=1)
    bottom = np.concatenate([h, -h], axis=1)
    return np.concatenate([top, bottom], axis=0) / np.sqrt(2.0)


def fwht(x: np.ndarray) -> np.ndarray:
    """Fast Walsh-Hadamard transform along the last axis, float64.

    The O(n log n) butterfly that [Hartmann rotation] (summary table) and
    [QuaRot hands-on] §4.1 name as the fast way to apply H: one add/sub pass
    per bit of the index ([Outlier nemesis] §2.1: H_4 = H_2 (x) H_2, only
    additions and subtractions), then one scaling by 1/sqrt(n).  Equal to
    ``x @ sylvester(n)`` (pinned by tests).
    """
    y = np.array(x, dtype=np.float64, copy=True)
    n = y.shape[-1]
    if n < 1 or (n & (n - 1)) != 0:
        raise ValueError(f"FWHT needs a power of two, got {n}")
    lead = y.shape[:-1]
    h = 1
    while h < n:
        v = y.reshape(lead + (n // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        b = v[..., 1, :]
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        h *= 2
    return y / np.sqrt(float(n))


def _block_size(dim: int, block: int) -> int:
    B = dim if block == -1 else block
    if B < 1 or (B & (B - 1)) != 0 or dim % B != 0:
        raise ValueError(f"block {block} is not a power of two dividing dim {dim}")
    return B


def _group_size(dim: int, group: int) -> int:
    G = dim if group == -1 else group
    if G < 1 or dim % G != 0:
        raise ValueError(f"group {group} does not divide dim {dim}")
    return G


def rotate(x: np.ndarray, block: int = -1, signs=None, method: str = "dense") -> np.ndarray:
    """y = (x * s) @ H_B applied independently to each B-wide block of a row.

    * [Hartmann rotation] §1: ``Q_rot = Q @ H.T`` on the last dimension.
    * [Outlier nemesis] §2.1: for widths that are not a power of two, cut the
      row into blocks (e.g. 4096 = 32 x 128) and rotate each block on its own,
      i.e. a block-diagonal H.  ``block = -1`` means one block over the whole
      row ([msModelSlim QuaRot] YAML ``block_size: -1``).
    * [QuaRot hands-on] §2.1: randomised Hadamard = random +-1 signs, then H.

    ``method='dense'`` multiplies by the explicit matrix; ``'fwht'`` uses the
    butterfly.  Returns float64 of the same shape as ``x``.
    """
    x = np.asarray(x, dtype=np.float64)
    dim = x.shape[-1]
    B = _block_size(dim, block)
    if signs is not None:
        s = np.where(np.asarray(signs) < 0, -1.0, 1.0)
        if s.shape != (dim,):
            raise ValueError("signs must have one entry per column")
        x = x * s
    xb = x.reshape(x.shape[:-1] + (dim // B, B))
    if method == "dense":
        H = sylvester(B)
        yb = xb @ H.T
    elif method == "fwht":
        yb = fwht(xb)
    else:
        raise ValueError(method)
    return yb.reshape(x.shape)


def inverse_rotate(y: np.ndarray, block: int = -1, signs=None, method: str = "dense") -> np.ndarray:
    """x = (y @ H_B) * s, the inverse of :func:`rotate`.

    H is orthogonal and symmetric, so H^-1 = H^T = H ([Hartmann rotation] §1,
    H H^T = I); the sign flip is its own inverse and is applied after H
    ([QuaRot hands-on] §2.3: the output is transformed back where needed).
    """
    y = np.asarray(y, dtype=np.float64)
    dim = y.shape[-1]
    B = _block_size(dim, block)
    yb = y.reshape(y.shape[:-1] + (dim // B, B))
    if method == "dense":
        xb = yb @ sylvester(B)
    elif method == "fwht":
        xb = fwht(yb)
    else:
        raise ValueError(method)
    x = xb.reshape(y.shape)
    if signs is not None:
        x = x * np.where(np.asarray(signs) < 0, -1.0, 1.0)
    return x


def quantize(y: np.ndarray, bits: int, group: int = -1):
    """Symmetric absmax quantisation of the last axis, per group of G columns.

    [Hartmann rotation] §1 and [Outlier nemesis] §2.2:
    ``scale = max|x| / (2^(b-1) - 1)``; ``q = clip(round(x / scale), -qmax, qmax)``.
    [Outlier nemesis] §6.2: per-group scales (group 128 for 4-bit).

    Returns ``(q, scale64, scale32, v)``: the integer codes (int64), the float64
    scale per group, that scale rounded to float32 (what is stored), and the
    pre-round value ``v = y / scale64`` (0 for an all-zero group).
    """
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    y = np.asarray(y, dtype=np.float64)
    dim = y.shape[-1]
    G = _group_size(dim, group)
    qmax = float(2 ** (bits - 1) - 1)
    yg = y.reshape(y.shape[:-1] + (dim // G, G))
    absmax = np.max(np.abs(yg), axis=-1)
    scale64 = absmax / qmax
    safe = np.where(scale64 > 0, scale64, 1.0)
    v = np.where(scale64[..., None] > 0, yg / safe[..., None], 0.0)
    q = np.clip(np.round(v), -qmax, qmax).astype(np.int64)
    return (q.reshape(y.shape), scale64, scale64.astype(np.float32),
            v.reshape(y.shape))


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Two 4-bit two's-complement codes per byte; element 2j in the low nibble.

    [QuaRot hands-on] §2.2: INT4 takes half a byte per value.  The nibble order
    is not stated on the pages; low nibble = even index is the reading used.
    """
    q = np.asarray(q, dtype=np.int64)
    if q.shape[-1] % 2:
        raise ValueError("INT4 packing needs an even number of columns")
    nib = (q & 0xF).astype(np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_int4`: sign-extend each nibble to int64."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def rotate_quantize(x_bits: np.ndarray, block: int = -1, signs=None, bits: int = 4,
                    group: int = -1, method: str = "dense") -> dict:
    """The whole forward step on a [rows, dim] bfloat16 input (raw uint16 bits).

    Steps, in the order the pages give them: decode bf16 -> multiply by the
    sign vector -> block Hadamard ([Hartmann rotation] §1, [Outlier nemesis]
    §2.1) -> per-group absmax scale -> round/clip ([Outlier nemesis] §2.2) ->
    INT8 codes or packed INT4 codes ([QuaRot hands-on] §2.2).

    Returns a dict with ``codes`` (int8 [rows, dim] or uint8 [rows, dim/2]),
    ``q`` (int64 codes, unpacked), ``scales`` (float32 [rows, dim/G]),
    ``scale64``, ``rotated`` (float64 y) and ``pre_round`` (float64 y/scale).
    """
    x = bf16_bits_to_f64(x_bits)
    y = rotate(x, block=block, signs=signs, method=method)
    q, scale64, scale32, v = quantize(y, bits, group)
    if bits == 8:
        codes = q.astype(np.int8)
    else:
        codes = pack_int4(q)
    return {"codes": codes, "q": q, "scales": scale32, "scale64": scale64,
            "rotated": y, "pre_round": v}


def dequant_rotate_inv(codes: np.ndarray, scales: np.ndarray, dim: int, block: int = -1,
                       signs=None, bits: int = 4, group: int = -1,
                       method: str = "dense") -> np.ndarray:
    """Dequantise then undo the rotation: x_hat = ((q * scale) @ H_B) * s.

    [QuaRot hands-on] §2.2: the 4-bit KV cache is dequantised when read;
    §2.3: the final output is transformed back if needed.  ``deq = q * scale``
    is the dequantisation of [Outlier nemesis] §2.2 (``x_q * scale``).  The
    stored float32 scale is used as given.  Returns float64 [rows, dim].
    """
    if bits == 8:
        q = np.asarray(codes).astype(np.int64)
    elif bits == 4:
        q = unpack_int4(codes)
    else:
        raise ValueError("bits must be 4 or 8")
    q = q.reshape(-1, dim)
    G = _group_size(dim, group)
    s = np.asarray(scales, dtype=np.float32).astype(np.float64).reshape(q.shape[0], dim // G)
    yhat = (q.reshape(q.shape[0], dim // G, G) * s[..., None]).reshape(q.shape)
    return inverse_rotate(yhat, block=block, signs=signs, method=method)


def kron_rotate(x: np.ndarray, fa: np.ndarray, b: int, signs=None) -> np.ndarray:
    """y = (F (x) H_b) (x * s) for rows of width a * b, float64.

    [msModelSlim QuaRot], online rotation: down_proj is rotated online with a
    Kronecker-product matrix, and dimensions without a Sylvester matrix take
    stored Hadamard matrices (FAQ: add the matrix for the dimension).  F is
    the a x a factor as it multiplies (e.g. a stored Hadamard matrix over
    sqrt(a)); H_b is the normalised Sylvester matrix.  With the row viewed as
    X[a, b] (element i * b + j), y = vec(F X H_b^T).
    """
    x = np.asarray(x, dtype=np.float64)
    fa = np.asarray(fa, dtype=np.float64)
    a = fa.shape[0]
    if fa.shape != (a, a) or x.shape[-1] != a * b:
        raise ValueError("row width must be a * b with F of shape (a, a)")
    if signs is not None:
        x = x * np.where(np.asarray(signs) < 0, -1.0, 1.0)
    X = x.reshape(x.shape[:-1] + (a, b))
    Y = fa @ X @ sylvester(b).T
    return Y.reshape(x.shape)


def kron_inverse_rotate(y: np.ndarray, fa: np.ndarray, b: int, signs=None) -> np.ndarray:
    """x = (F^T (x) H_b) y, then the signs: the inverse of :func:`kron_rotate`
    for an orthogonal F (H_b is symmetric and orthogonal)."""
    y = np.asarray(y, dtype=np.float64)
    fa = np.asarray(fa, dtype=np.float64)
    a = fa.shape[0]
    Y = y.reshape(y.shape[:-1] + (a, b))
    X = fa.T @ Y @ sylvester(b).T
    x = X.reshape(y.shape)
    if signs is not None:
        x = x * np.where(np.asarray(signs) < 0, -1.0, 1.0)
    return x


def rotate_quantize_kron(x_bits: np.ndarray, fa: np.ndarray, b: int, signs=None, bits: int = 4,
                         group: int = -1) -> dict:
    """The forward step with the Kronecker rotation: decode bf16 ->
    :func:`kron_rotate` -> symmetric absmax quantisation (:func:`quantize`) ->
    codes, as :func:`rotate_quantize`."""
    y = kron_rotate(bf16_bits_to_f64(x_bits), fa, b, signs)
    q, scale64, scale32, v = quantize(y, bits, group)
    codes = q.astype(np.int8) if bits == 8 else pack_int4(q)
    return {"codes": codes, "q": q, "scales": scale32, "scale64": scale64, "rotated": y, "pre_round": v}


def dequant_rotate_inv_kron(codes: np.ndarray, scales: np.ndarray, fa: np.ndarray, b: int, signs=None,
                            bits: int = 4, group: int = -1) -> np.ndarray:
    """q * scale with the stored float32 scale, then :func:`kron_inverse_rotate`."""
    a = np.asarray(fa).shape[0]
    dim = a * b
    q = np.asarray(codes).astype(np.int64) if bits == 8 else unpack_int4(codes)
    q = q.reshape(-1, dim)
    G = _group_size(dim, group)
    s = np.asarray(scales, dtype=np.float32).astype(np.float64).reshape(q.shape[0], dim // G)
    yhat = (q.reshape(q.shape[0], dim // G, G) * s[..., None]).reshape(q.shape)
    return kron_inverse_rotate(yhat, fa, b, signs)


def quantize_asym(y: np.ndarray, bits: int, group: int = -1):
    """Asymmetric (zero-point) quantisation of the last axis, per group of G columns.

    [Hartmann rotation] §2, the FakeQuantize forward: x_int = round(x / scale)
    + zero_point, clamped to [0, 2^b - 1]; dequantised as (x_int - zero_point)
    * scale.  The page takes scale and zero point as given (learned); here
    they come from the group's range, which always holds 0 (reading):
    lo = min(0, min y), hi = max(0, max y), scale = (hi - lo) / (2^b - 1),
    zero_point = clamp(round(-lo / scale), 0, 2^b - 1).  Rounding is half to
    even.  A group of zeros gets scale 0, zero point 0 and codes 0.

    Returns ``(q, scale64, scale32, zp, v, zv)``: unsigned integer codes
    (int64), the float64 scale, that scale rounded to float32 (stored), the
    zero points (int64), the pre-round values v = y / scale64 and
    zv = -lo / scale64.
    """
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    y = np.asarray(y, dtype=np.float64)
    dim = y.shape[-1]
    G = _group_size(dim, group)
    qmax = float(2 ** bits - 1)
    yg = y.reshape(y.shape[:-1] + (dim // G, G))
    lo = np.minimum(yg.min(axis=-1), 0.0)
    hi = np.maximum(yg.max(axis=-1), 0.0)
    scale64 = (hi - lo) / qmax
    nz = scale64 > 0
    safe = np.where(nz, scale64, 1.0)
    zv = np.where(nz, -lo / safe, 0.0)
    zp = np.clip(np.round(zv), 0, qmax).astype(np.int64)
    v = np.where(nz[..., None], yg / safe[..., None], 0.0)
    q = np.clip(np.round(v) + zp[..., None], 0, qmax).astype(np.int64)
    q = np.where(nz[..., None], q, 0)
    return (q.reshape(y.shape), scale64, scale64.astype(np.float32), zp, v.reshape(y.shape), zv)


def pack_uint4(q: np.ndarray) -> np.ndarray:
    """Two unsigned 4-bit codes (0..15) per byte; element 2j in the low nibble."""
    q = np.asarray(q, dtype=np.int64)
    if q.shape[-1] % 2:
        raise ValueError("INT4 packing needs an even number of columns")
    return ((q[..., 0::2] & 0xF) | ((q[..., 1::2] & 0xF) << 4)).astype(np.uint8)


def unpack_uint4(packed: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_uint4` (values 0..15, int64)."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int64)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = (p >> 4) & 0xF
    return out


def rotate_quantize_asym(x_bits: np.ndarray, block: int = -1, signs=None, bits: int = 4,
                         group: int = -1, method: str = "dense") -> dict:
    """The forward step with the asymmetric quantiser: decode bf16 -> signs ->
    block Hadamard (as :func:`rotate_quantize`) -> :func:`quantize_asym` ->
    unsigned codes (uint8 per element for INT8, two per byte for INT4).

    Returns ``codes``, ``q``, ``scales`` (float32 [rows, dim/G]),
    ``zero_points`` (uint8 [rows, dim/G]), ``scale64``, ``rotated``,
    ``pre_round`` (y / scale64) and ``zp_pre_round`` (-lo / scale64).
    """
    x = bf16_bits_to_f64(x_bits)
    y = rotate(x, block=block, signs=signs, method=method)
    q, scale64, scale32, zp, v, zv = quantize_asym(y, bits, group)
    codes = q.astype(np.uint8) if bits == 8 else pack_uint4(q)
    return {"codes": codes, "q": q, "scales": scale32, "zero_points": zp.astype(np.uint8),
            "scale64": scale64, "rotated": y, "pre_round": v, "zp_pre_round": zv}


def dequant_rotate_inv_asym(codes: np.ndarray, scales: np.ndarray, zero_points: np.ndarray, dim: int,
                            block: int = -1, signs=None, bits: int = 4, group: int = -1,
                            method: str = "dense") -> np.ndarray:
    """x_hat = (((q - zero_point) * scale) H_B) * s with the stored float32
    scale ([Hartmann rotation] §2: (x_int - zero_point) * scale, then the
    inverse rotation as :func:`dequant_rotate_inv`).  Returns float64
    [rows, dim]."""
    q = np.asarray(codes).astype(np.int64) if bits == 8 else unpack_uint4(codes)
    q = q.reshape(-1, dim)
    G = _group_size(dim, group)
    s = np.asarray(scales, dtype=np.float32).astype(np.float64).reshape(q.shape[0], dim // G)
    z = np.asarray(zero_points).astype(np.int64).reshape(q.shape[0], dim // G)
    yhat = ((q.reshape(q.shape[0], dim // G, G) - z[..., None]) * s[..., None]).reshape(q.shape)
    return inverse_rotate(yhat, block=block, signs=signs, method=method)


def _kept_tokens(keep_slot, n_keep: int):
    """(token, slot) pairs of the kept tokens: entries in [0, n_keep)."""
    ks = np.asarray(keep_slot).astype(np.int64)
    return [(t, int(v)) for t, v in enumerate(ks) if 0 <= v < n_keep]


def rotate_quantize_keep(x_bits: np.ndarray, heads: int, tokens: int, keep_slot, n_keep: int,
                         block: int = -1, signs=None, bits: int = 4, group: int = -1,
                         method: str = "dense") -> dict:
    """HyQuant-style mixed-precision KV quantisation of [heads * tokens, dim] rows.

    [HyQuant] method, key modules: a small set of tokens (vertical-line
    tokens, which carry most of the attention mass, and a local window) stays
    in full precision and every other token is stored in low bit; the decode
    stage applies that split to the KV cache.  [Hartmann rotation] §3 (the
    first, "sink", tokens always matter) gives the other usual member of the
    kept set.  Which tokens are kept is an input here.  Row
    h * tokens + t belongs to head h and token t.  Token t is kept when
    ``keep_slot[t]`` lies in [0, n_keep): its rows are copied unchanged into
    ``kept[h, keep_slot[t]]`` (bf16 bits) and get codes 0 and scale 0.  Every
    other row is rotated and quantised exactly as :func:`rotate_quantize`.
    """
    r = rotate_quantize(x_bits, block=block, signs=signs, bits=bits, group=group, method=method)
    x = np.asarray(x_bits, dtype=np.uint16).reshape(heads * tokens, -1)
    dim = x.shape[1]
    codes, scales, q = r["codes"].copy(), r["scales"].copy(), r["q"].copy()
    kept = np.zeros((heads, n_keep, dim), dtype=np.uint16)
    keep_row = np.zeros(heads * tokens, dtype=bool)
    for t, slot in _kept_tokens(keep_slot, n_keep):
        for h in range(heads):
            row = h * tokens + t
            kept[h, slot] = x[row]
            codes[row] = 0
            scales[row] = 0.0
            q[row] = 0
            keep_row[row] = True
    return {"codes": codes, "q": q, "scales": scales, "kept": kept, "keep_row": keep_row,
            "rotated": r["rotated"], "pre_round": r["pre_round"], "scale64": r["scale64"]}


def dequant_rotate_inv_keep(codes: np.ndarray, scales: np.ndarray, kept: np.ndarray, keep_slot,
                            n_keep: int, heads: int, tokens: int, dim: int, block: int = -1,
                            signs=None, bits: int = 4, group: int = -1,
                            method: str = "dense") -> np.ndarray:
    """Reads a mixed-precision cache back: kept tokens return their bf16 rows
    exactly, every other row is dequantised and rotated back as
    :func:`dequant_rotate_inv`.  Returns float64 [heads * tokens, dim]."""
    out = dequant_rotate_inv(codes, scales, dim, block=block, signs=signs, bits=bits, group=group,
                             method=method)
    for t, slot in _kept_tokens(keep_slot, n_keep):
        for h in range(heads):
            out[h * tokens + t] = bf16_bits_to_f64(kept[h, slot])
    return out


def dequant_rotated(codes: np.ndarray, scales: np.ndarray, dim: int, bits: int = 4,
                    group: int = -1) -> np.ndarray:
    """q * scale, left in the rotated basis (no inverse rotation), float64 [..., dim].

    The dequantisation of [Outlier nemesis] §2.2 (``x_q * scale``) applied to
    stored codes; [QuaRot hands-on] §2.2 reads the 4-bit KV cache this way.
    """
    q = np.asarray(codes).astype(np.int64) if bits == 8 else unpack_int4(codes)
    lead = q.shape[:-1]
    G = _group_size(dim, group)
    s = np.asarray(scales, dtype=np.float32).astype(np.float64).reshape(lead + (dim // G,))
    return (q.reshape(lead + (dim // G, G)) * s[..., None]).reshape(lead + (dim,))


def kv_decode_scores(q_bits: np.ndarray, k_codes: np.ndarray, k_scales: np.ndarray, dim: int,
                     block: int = -1, signs=None, bits: int = 4, group: int = -1,
                     softmax_scale: float | None = None) -> np.ndarray:
    """Attention scores of one decode query per head against a rotated,
    quantised key cache: softmax_scale * q_rot . k_hat_t, float64
    [batch, n_q_heads, tokens].

    [Hartmann rotation] §1: Q_rot K_rot^T = Q K^T, so the rotated query
    against the dequantised rotated keys gives the scores of the un-rotated
    ones.  Query head h reads KV head h // (n_q_heads / n_kv_heads).
    """
    q = bf16_bits_to_f64(q_bits)
    nb, nqh, d = q.shape
    assert d == dim
    kr = dequant_rotated(k_codes, k_scales, dim, bits, group)   # [b, hk, T, d]
    nkh = kr.shape[1]
    if nqh % nkh:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    g = nqh // nkh
    if softmax_scale is None:
        softmax_scale = 1.0 / np.sqrt(dim)
    qr = rotate(q, block=block, signs=signs)
    s = np.empty((nb, nqh, kr.shape[2]))
    for b in range(nb):
        for h in range(nqh):
            s[b, h] = softmax_scale * (kr[b, h // g] @ qr[b, h])
    return s


def kv_decode_attention(q_bits: np.ndarray, k_codes: np.ndarray, k_scales: np.ndarray,
                        v_codes: np.ndarray, v_scales: np.ndarray, dim: int, block: int = -1,
                        signs=None, bits: int = 4, group: int = -1,
                        softmax_scale: float | None = None) -> np.ndarray:
    """Decode attention of one new query token per head over a quantised,
    rotated KV cache, float64.

    * [QuaRot hands-on] §2.2: K and V are rotated online and stored in 4 bits,
      then dequantised when they are read for attention.
    * Scores from :func:`kv_decode_scores` (rotated query against rotated
      keys, [Hartmann rotation] §1), softmax over the cached tokens.
    * P V_rot = (P V) H: the output is computed in the rotated basis and
      transformed back once ([QuaRot hands-on] §2.3), with H and the signs
      of :func:`inverse_rotate`.

    Shapes: ``q_bits`` bf16 bits [batch, n_q_heads, dim]; codes [batch,
    n_kv_heads, tokens, dim] (INT8) or [..., dim/2] (INT4); scales [batch,
    n_kv_heads, tokens, dim/G].  Query head h reads KV head h // (n_q_heads /
    n_kv_heads).  Returns float64 [batch, n_q_heads, dim].
    """
    s = kv_decode_scores(q_bits, k_codes, k_scales, dim, block, signs, bits, group, softmax_scale)
    vr = dequant_rotated(v_codes, v_scales, dim, bits, group)   # [b, hk, T, d]
    nb, nqh, _ = s.shape
    g = nqh // vr.shape[1]
    out = np.empty((nb, nqh, dim))
    for b in range(nb):
        for h in range(nqh):
            p = np.exp(s[b, h] - s[b, h].max())
            p /= p.sum()
            out[b, h] = p @ vr[b, h // g]
    return inverse_rotate(out, block=block, signs=signs)


def quant_error(x: np.ndarray, bits: int = 4) -> float:
    """Mean absolute error of one tensor-wide symmetric absmax quantisation.

    The error measure of [Outlier nemesis] §2.2: one scale for the whole
    input, round, clip to +-qmax, dequantise, mean |x - x_deq|.
    """
    x = np.asarray(x, dtype=np.float64)
    qmax = 2 ** (bits - 1) - 1
    scale = np.abs(x).max() / qmax
    xq = np.clip(np.round(x / scale), -qmax, qmax)
    return float(np.mean(np.abs(x - xq * scale)))


def half_boundary_distance(v: np.ndarray) -> np.ndarray:
    """Distance of each pre-round value to the nearest rounding boundary k+0.5."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    return np.abs((a - np.floor(a)) - 0.5)
