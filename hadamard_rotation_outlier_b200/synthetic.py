"""Seeded synthetic inputs for the rotate + quantize path.

This module only draws random numbers and converts them to bfloat16 bit
patterns.  It holds none of the method's arithmetic (no Hadamard transform,
no scale, no rounding to codes), so both the CUDA path and the CPU oracle can
take their inputs from it.

Workloads follow the five synthetic configurations this library is measured
on: activations with about 0.1% of channels ~100x larger (the outlier
statistic quoted on [Hartmann rotation] §1), Q/K heads and KV-cache rows with
a few outlier dimensions per head, and heavy-tailed Student-t(3) rows of a
width that is not a power of two.  Rows are generated in fixed chunks, each
from its own seed, so any row range can be regenerated without producing the
whole tensor.
"""

from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK_ROWS = 256
DEFAULT_SEED = 42


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the raw uint16 bit patterns.  Inputs must be finite.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


@dataclasses.dataclass(frozen=True)
class Tensor:
    """One input tensor of a workload: its name, row count and outliers.

    ``outlier_dims`` is the number of outlier columns per head (0 for none);
    rows ``[h * rows_per_head, (h + 1) * rows_per_head)`` belong to head h.
    ``outlier_key`` names the seed stream of the outlier columns, so that two
    tensors (Q and K of one head) can share them.
    """
    name: str
    rows: int
    heads: int = 1
    outlier_dims: int = 0
    outlier_scale: float = 1.0
    outlier_key: int = 0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    description: str
    dim: int
    block: int          # -1: one Hadamard block over the whole row
    group: int          # -1: one scale per row
    bits: int
    with_signs: bool
    dist: str           # "normal" or "student_t3"
    tensors: tuple
    dequant: bool = False
    # kept tokens (mixed precision): (n_sink, window, n_vertical) or None.
    # Rows are then [heads, tokens] over all tensors stacked (every tensor
    # has the same tokens per head), and a token's rows are kept in all heads.
    keep: tuple | None = None
    # asymmetric (zero-point) quantiser: unsigned codes + one zero point per group
    asym: bool = False
    # Kronecker rotation (F (x) H_b) with a Paley factor of order kron_a
    # (b = dim / kron_a); 0 for none
    kron_a: int = 0

    @property
    def rows(self) -> int:
        return sum(t.rows for t in self.tensors)

    @property
    def elements(self) -> int:
        return self.rows * self.dim

    def scales_per_row(self) -> int:
        return self.dim // (self.dim if self.group == -1 else self.group)

    @property
    def heads(self) -> int:
        return sum(t.heads for t in self.tensors)

    @property
    def tokens(self) -> int:
        return self.tensors[0].rows // self.tensors[0].heads

    @property
    def n_keep(self) -> int:
        if not self.keep:
            return 0
        n_sink, window, n_vertical = self.keep
        return n_sink + window + n_vertical

    def quant_bytes(self) -> int:
        """bf16 in + codes out + fp32 scales out, each byte moved once (plus,
        with kept tokens, the int32 keep table in and the kept bf16 rows out)."""
        n = self.elements
        codes = n if self.bits == 8 else n // 2
        b = 2 * n + codes + 4 * self.rows * self.scales_per_row()
        if self.keep:
            b += 4 * self.tokens + 2 * self.heads * self.n_keep * self.dim
        if self.asym:
            b += self.rows * self.scales_per_row()
        return b

    def dequant_bytes(self, out_bytes_per_elem: int = 2) -> int:
        """codes + fp32 scales in + reconstructed values out (plus the keep
        table and the kept bf16 rows in)."""
        n = self.elements
        codes = n if self.bits == 8 else n // 2
        b = codes + 4 * self.rows * self.scales_per_row() + out_bytes_per_elem * n
        if self.keep:
            b += 4 * self.tokens + 2 * self.heads * self.n_keep * self.dim
        if self.asym:
            b += self.rows * self.scales_per_row()
        return b

    def with_rows(self, rows_per_tensor: int) -> "Workload":
        """The same recipe with fewer rows per tensor (for oracle-sized tests).

        Head structure is kept: rows are spread over the same number of heads.
        """
        ts = []
        for t in self.tensors:
            r = max(t.heads, (rows_per_tensor // t.heads) * t.heads)
            ts.append(dataclasses.replace(t, rows=r))
        return dataclasses.replace(self, tensors=tuple(ts))


WORKLOADS = {
    "c1_tok256_h4096_b128_int4": Workload(
        name="c1_tok256_h4096_b128_int4",
        description="256 tokens x hidden 4096, N(0,1) with 4 seeded channels x100; "
                    "block Hadamard 128 (32 blocks), no signs; per-token INT4",
        dim=4096, block=128, group=-1, bits=4, with_signs=False, dist="normal",
        tensors=(Tensor("x", 256, 1, 4, 100.0, 1),)),
    "c2_qk_h32_s8192_d128_int8": Workload(
        name="c2_qk_h32_s8192_d128_int8",
        description="Q and K [1,32,8192,128], N(0,1) with 2 outlier dims per head x50 "
                    "(shared by Q and K); full 128-point Hadamard; per token-head INT8",
        dim=128, block=-1, group=-1, bits=8, with_signs=False, dist="normal",
        tensors=(Tensor("q", 32 * 8192, 32, 2, 50.0, 2),
                 Tensor("k", 32 * 8192, 32, 2, 50.0, 2))),
    "c3_tok16384_h4096_full_signs_int4": Workload(
        name="c3_tok16384_h4096_full_signs_int4",
        description="16384 tokens x hidden 4096, N(0,1) with 4 channels (0.1%) x100; "
                    "seeded signs then full 4096-point Hadamard; per-token INT4",
        dim=4096, block=-1, group=-1, bits=4, with_signs=True, dist="normal",
        tensors=(Tensor("x", 16384, 1, 4, 100.0, 3),)),
    "c4_kv_h8_t131072_d128_int4_g128": Workload(
        name="c4_kv_h8_t131072_d128_int4_g128",
        description="K and V [8,131072,128], N(0,1), K with 4 outlier dims per head x30; "
                    "128-point Hadamard; INT4 group 128; then dequant + inverse",
        dim=128, block=128, group=128, bits=4, with_signs=False, dist="normal",
        tensors=(Tensor("k", 8 * 131072, 8, 4, 30.0, 4),
                 Tensor("v", 8 * 131072, 8, 0, 1.0, 5)),
        dequant=True),
    "c4k_kv_h8_t131072_d128_int4_g128_keep196": Workload(
        name="c4k_kv_h8_t131072_d128_int4_g128_keep196",
        description="the KV-cache workload with HyQuant-style mixed precision: 4 sink tokens, 64 "
                    "seeded vertical-line tokens and a 128-token window stay bf16, the rest INT4; "
                    "then read back (kept rows exact, the rest dequantised + inverse)",
        dim=128, block=128, group=128, bits=4, with_signs=False, dist="normal",
        tensors=(Tensor("k", 8 * 131072, 8, 4, 30.0, 4),
                 Tensor("v", 8 * 131072, 8, 0, 1.0, 5)),
        dequant=True, keep=(4, 128, 64)),
    "c4a_kv_h8_t131072_d128_uint4_g128_asym": Workload(
        name="c4a_kv_h8_t131072_d128_uint4_g128_asym",
        description="the KV-cache workload with the asymmetric quantiser: unsigned INT4 codes, one "
                    "fp32 scale and one uint8 zero point per 128-column group; then dequant + inverse",
        dim=128, block=128, group=128, bits=4, with_signs=False, dist="normal",
        tensors=(Tensor("k", 8 * 131072, 8, 4, 30.0, 4),
                 Tensor("v", 8 * 131072, 8, 0, 1.0, 5)),
        dequant=True, asym=True),
    "c6_tok8192_d5120_kron20x256_int4_g128": Workload(
        name="c6_tok8192_d5120_kron20x256_int4_g128",
        description="8192 tokens x 5120 (no Sylvester matrix of that width), N(0,1) with 5 channels "
                    "x100; seeded signs, Kronecker rotation (Paley S_20 / sqrt(20)) x (H_256) with the "
                    "factor given as the stored +-1 matrix S_20; INT4 group 128",
        dim=5120, block=256, group=128, bits=4, with_signs=True, dist="normal",
        tensors=(Tensor("x", 8192, 1, 5, 100.0, 7),), kron_a=20),
    "c5_tok32768_w11008_b128_signs_int4_g128": Workload(
        name="c5_tok32768_w11008_b128_signs_int4_g128",
        description="32768 tokens x 11008 (86 blocks of 128), Student-t(3); seeded signs, "
                    "block Hadamard 128; INT4 group 128",
        dim=11008, block=128, group=128, bits=4, with_signs=True, dist="student_t3",
        tensors=(Tensor("x", 32768, 1, 0, 1.0, 6),)),
}

WORKLOAD_ORDER = list(WORKLOADS)


def outlier_columns(t: Tensor, dim: int, seed: int = DEFAULT_SEED) -> np.ndarray:
    """Seeded outlier column indices, shape [heads, outlier_dims] (sorted)."""
    if t.outlier_dims == 0:
        return np.zeros((t.heads, 0), dtype=np.int64)
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x0D11, t.outlier_key]))
    cols = [np.sort(rng.choice(dim, size=t.outlier_dims, replace=False)) for _ in range(t.heads)]
    return np.stack(cols).astype(np.int64)


def signs(wl: Workload, seed: int = DEFAULT_SEED):
    """The seeded +-1 sign vector of a workload (int8 [dim]) or None."""
    if not wl.with_signs:
        return None
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x5160, wl.dim]))
    return (rng.integers(0, 2, size=wl.dim) * 2 - 1).astype(np.int8)


def _chunk_values(dist: str, dim: int, n_rows: int, ss: np.random.SeedSequence) -> np.ndarray:
    rng = np.random.default_rng(ss)
    if dist == "normal":
        return rng.standard_normal((n_rows, dim), dtype=np.float32)
    if dist == "student_t3":
        return rng.standard_t(3, size=(n_rows, dim)).astype(np.float32)
    raise ValueError(dist)


def _chunk(wl: Workload, ti: int, c: int, seed: int, cols: np.ndarray) -> np.ndarray:
    t = wl.tensors[ti]
    r0 = c * CHUNK_ROWS
    r1 = min(t.rows, r0 + CHUNK_ROWS)
    ss = np.random.SeedSequence([seed, 0xDA7A, ti, c])
    v = _chunk_values(wl.dist, wl.dim, r1 - r0, ss)
    if t.outlier_dims:
        rows_per_head = t.rows // t.heads
        heads = np.arange(r0, r1) // rows_per_head
        for h in np.unique(heads):
            sel = heads == h
            v[np.ix_(sel, cols[h])] *= np.float32(t.outlier_scale)
    return f32_to_bf16_bits(v)


def tensor_rows(wl: Workload, ti: int, r0: int, r1: int, seed: int = DEFAULT_SEED,
                threads: int | None = None) -> np.ndarray:
    """Rows [r0, r1) of tensor ``ti`` as bfloat16 bits (uint16 [r1-r0, dim])."""
    t = wl.tensors[ti]
    if not (0 <= r0 <= r1 <= t.rows):
        raise ValueError("row range out of bounds")
    out = np.empty((r1 - r0, wl.dim), dtype=np.uint16)
    if r1 == r0:
        return out
    cols = outlier_columns(t, wl.dim, seed)
    c0, c1 = r0 // CHUNK_ROWS, (r1 - 1) // CHUNK_ROWS + 1

    def work(c):
        a = _chunk(wl, ti, c, seed, cols)
        lo = max(r0, c * CHUNK_ROWS)
        hi = min(r1, c * CHUNK_ROWS + a.shape[0])
        out[lo - r0:hi - r0] = a[lo - c * CHUNK_ROWS:hi - c * CHUNK_ROWS]

    n = c1 - c0
    nthreads = threads or min(n, os.cpu_count() or 1, 32)
    if nthreads <= 1:
        for c in range(c0, c1):
            work(c)
    else:
        with ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(work, range(c0, c1)))
    return out


def tensor(wl: Workload, ti: int, seed: int = DEFAULT_SEED) -> np.ndarray:
    """A whole input tensor as bfloat16 bits (uint16 [rows, dim])."""
    return tensor_rows(wl, ti, 0, wl.tensors[ti].rows, seed)


def random_bf16(rows: int, dim: int, seed: int, dist: str = "normal",
                outlier_cols=(), outlier_scale: float = 100.0) -> np.ndarray:
    """Free-form seeded bf16 input for shape sweeps (uint16 [rows, dim])."""
    ss = np.random.SeedSequence([seed, 0xF4EE, rows, dim])
    v = _chunk_values(dist, dim, rows, ss)
    if len(outlier_cols):
        v[:, np.asarray(outlier_cols)] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(v)


def random_signs(dim: int, seed: int) -> np.ndarray:
    """Seeded +-1 int8 sign vector of length ``dim``."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x5161, dim]))
    return (rng.integers(0, 2, size=dim) * 2 - 1).astype(np.int8)


# ------------------------------------------------------------------ decode

@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """One decode step of attention over a rotated INT4 KV cache.

    ``batch`` sequences, each with ``n_q_heads`` query heads (one new token)
    and ``n_kv_heads`` cached heads of ``tokens`` rows at head dim ``dim``.
    """
    name: str
    description: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    tokens: int
    dim: int = 128
    with_signs: bool = False

    def attn_bytes(self, out_bytes_per_elem: int = 2) -> int:
        """bf16 query in + K and V codes + K and V row scales in + output,
        each byte moved once."""
        rows = self.batch * self.n_kv_heads * self.tokens
        q = self.batch * self.n_q_heads * self.dim
        return 2 * q + 2 * rows * (self.dim // 2) + 2 * rows * 4 + out_bytes_per_elem * q


DECODE_WORKLOADS = {
    "d1_decode_q32_kv8_t131072_d128_int4": DecodeWorkload(
        name="d1_decode_q32_kv8_t131072_d128_int4",
        description="one decode step: 32 query heads, 8 KV heads (4 per group), the "
                    "131072-token INT4 cache of K and V [8,131072,128]",
        batch=1, n_q_heads=32, n_kv_heads=8, tokens=131072),
}


def decode_query(batch: int, n_q_heads: int, dim: int, seed: int, outlier_dims: int = 2,
                 outlier_scale: float = 50.0) -> np.ndarray:
    """Seeded query rows, bf16 bits [batch, n_q_heads, dim]: N(0,1) with
    ``outlier_dims`` seeded columns per head scaled by ``outlier_scale``."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x0E7A, batch, n_q_heads, dim]))
    v = rng.standard_normal((batch, n_q_heads, dim), dtype=np.float32)
    for h in range(n_q_heads):
        cols = rng.choice(dim, size=outlier_dims, replace=False)
        v[:, h, cols] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(v)


def random_int4_cache(batch: int, n_kv_heads: int, stride: int, dim: int, seed: int,
                      scale_range=(0.25, 0.75)):
    """Seeded packed INT4 cache rows and positive float32 row scales.

    Each code is an independent draw of binomial(14, 1/2) - 7 (values -7..7,
    standard deviation 1.87), taken as the number of set bits among 14 random
    bits minus 7, and stored as 4-bit two's complement with element 2j in the
    low nibble of byte j.  Returns ``(codes uint8 [batch, n_kv_heads, stride,
    dim/2], scales float32 [batch, n_kv_heads, stride])``.
    """
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0xCAC4, batch, n_kv_heads, stride, dim]))
    shape = (batch, n_kv_heads, stride, dim // 2)
    ones = np.array([bin(v).count("1") - 7 for v in range(1 << 14)], dtype=np.int8)
    lo = ones[rng.integers(0, 1 << 14, size=shape, dtype=np.uint16)]
    hi = ones[rng.integers(0, 1 << 14, size=shape, dtype=np.uint16)]
    codes = ((lo.view(np.uint8) & 0xF) | ((hi.view(np.uint8) & 0xF) << 4)).astype(np.uint8)
    scales = rng.uniform(scale_range[0], scale_range[1],
                         size=(batch, n_kv_heads, stride)).astype(np.float32)
    return codes, scales


def random_int8_cache(batch: int, n_kv_heads: int, stride: int, dim: int, seed: int,
                      scale_range=(0.004, 0.012)):
    """Seeded INT8 cache rows and positive float32 row scales.

    Each code is the sum of four independent uniform draws from -31..31
    (values -124..124, standard deviation about 36), stored as int8.  Returns
    ``(codes int8 [batch, n_kv_heads, stride, dim], scales float32 [batch,
    n_kv_heads, stride])``.
    """
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0xCAC8, batch, n_kv_heads, stride, dim]))
    shape = (batch, n_kv_heads, stride, dim)
    codes = np.zeros(shape, np.int16)
    for _ in range(4):
        codes += rng.integers(-31, 32, size=shape, dtype=np.int16)
    scales = rng.uniform(scale_range[0], scale_range[1],
                         size=(batch, n_kv_heads, stride)).astype(np.float32)
    return codes.astype(np.int8), scales


def vertical_tokens(tokens: int, n: int, seed: int, skip_head: int = 0, skip_tail: int = 0) -> np.ndarray:
    """Seeded distinct token indices standing in for vertical-line tokens,
    drawn from [skip_head, tokens - skip_tail) and sorted."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x7E47, tokens, n]))
    lo, hi = skip_head, tokens - skip_tail
    return np.sort(rng.choice(np.arange(lo, hi), size=min(n, max(0, hi - lo)), replace=False))


def paley_hadamard(q: int) -> np.ndarray:
    """A +-1 Hadamard matrix of order q + 1 for a prime q = 3 (mod 4), by the
    Paley construction (quadratic residues of GF(q)); int8 [q + 1, q + 1].

    Stands in for the stored Hadamard matrices that widths without a
    Sylvester matrix need (those files are not available here).
    """
    res = {(i * i) % q for i in range(1, q)}
    chi = np.array([0] + [1 if v in res else -1 for v in range(1, q)], dtype=np.int64)
    idx = (np.arange(q)[None, :] - np.arange(q)[:, None]) % q
    S = np.zeros((q + 1, q + 1), dtype=np.int64)
    S[0, 1:] = 1
    S[1:, 0] = -1
    S[1:, 1:] = chi[idx]
    return (S + np.eye(q + 1, dtype=np.int64)).astype(np.int8)
