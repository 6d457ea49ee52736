"""Thin ctypes binding of libhadq.so (include/hadq.h), same names as the C ABI.

This module only marshals arguments: it checks tensor dtypes, devices and
contiguity, resolves the row count, allocates outputs with torch when the
caller passes none, and calls the C entry point on the current CUDA stream.
Every step of the computation runs in the library's CUDA kernels.  There is
no fallback: if the library is missing or cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhadq.so")

HADQ_OK, HADQ_ERR_INVALID_ARG, HADQ_ERR_UNSUPPORTED, HADQ_ERR_MISALIGNED, HADQ_ERR_CUDA, HADQ_ERR_DEVICE = range(6)
HADQ_OUT_BF16, HADQ_OUT_F32 = 0, 1
PATH_NAMES = {0: "none", 1: "blocked", 2: "full4096", 3: "generic", 4: "chunk", 5: "wide4096", 6: "wide4096_mma", 7: "chunk_mma", 8: "h4096_tc"}
KRON_VARIANTS = {0: "smem", 1: "reg16", 2: "mma"}
MAX_DIM = 32768

EXPORTED = ("hadq_rotate_quantize", "hadq_dequant_rotate_inv", "hadq_rotate_quantize_kron",
            "hadq_dequant_rotate_inv_kron", "hadq_rotate_quantize_kron_pm1", "hadq_dequant_rotate_inv_kron_pm1", "hadq_rotate_quantize_asym",
            "hadq_dequant_rotate_inv_asym", "hadq_rotate_quantize_keep",
            "hadq_dequant_rotate_inv_keep", "hadq_kv_decode_attention",
            "hadq_kv_decode_workspace_size", "hadq_kv_decode_attention_noalloc", "hadq_plan", "hadq_kron_plan", "hadq_device_status", "hadq_selftest_bounded_wait", "hadq_status_str", "hadq_last_error",
            "hadq_launch_count", "hadq_version")


class HadqError(RuntimeError):
    """A non-OK status returned by the library."""

    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libhadq.so (once) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libhadq.so not found at {path}; build it with "
                           "`python -m hadamard_rotation_outlier_b200.build`")
    lib = ctypes.CDLL(path)
    c_i64, c_i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
    lib.hadq_rotate_quantize.argtypes = [vp, c_i64, c_i32, c_i32, vp, c_i32, c_i32, vp, vp, vp, vp]
    lib.hadq_rotate_quantize.restype = ctypes.c_int
    lib.hadq_dequant_rotate_inv.argtypes = [vp, vp, c_i64, c_i32, c_i32, vp, c_i32, c_i32, vp,
                                            ctypes.c_int, vp]
    lib.hadq_dequant_rotate_inv.restype = ctypes.c_int
    lib.hadq_rotate_quantize_kron.argtypes = [vp, c_i64, c_i32, vp, c_i32, vp, c_i32, c_i32, vp, vp, vp, vp]
    lib.hadq_rotate_quantize_kron.restype = ctypes.c_int
    lib.hadq_dequant_rotate_inv_kron.argtypes = [vp, vp, c_i64, c_i32, vp, c_i32, vp, c_i32, c_i32, vp,
                                                 ctypes.c_int, vp]
    lib.hadq_dequant_rotate_inv_kron.restype = ctypes.c_int
    lib.hadq_rotate_quantize_kron_pm1.argtypes = lib.hadq_rotate_quantize_kron.argtypes
    lib.hadq_rotate_quantize_kron_pm1.restype = ctypes.c_int
    lib.hadq_dequant_rotate_inv_kron_pm1.argtypes = lib.hadq_dequant_rotate_inv_kron.argtypes
    lib.hadq_dequant_rotate_inv_kron_pm1.restype = ctypes.c_int
    lib.hadq_rotate_quantize_asym.argtypes = [vp, c_i64, c_i32, c_i32, vp, c_i32, c_i32, vp, vp, vp, vp]
    lib.hadq_rotate_quantize_asym.restype = ctypes.c_int
    lib.hadq_dequant_rotate_inv_asym.argtypes = [vp, vp, vp, c_i64, c_i32, c_i32, vp, c_i32, c_i32, vp,
                                                 ctypes.c_int, vp]
    lib.hadq_dequant_rotate_inv_asym.restype = ctypes.c_int
    lib.hadq_rotate_quantize_keep.argtypes = [vp, c_i64, c_i64, c_i32, c_i32, vp, c_i32, c_i32, vp, c_i32,
                                              vp, vp, vp, vp]
    lib.hadq_rotate_quantize_keep.restype = ctypes.c_int
    lib.hadq_dequant_rotate_inv_keep.argtypes = [vp, vp, vp, vp, c_i32, c_i64, c_i64, c_i32, c_i32, vp, c_i32,
                                                 c_i32, vp, ctypes.c_int, vp]
    lib.hadq_dequant_rotate_inv_keep.restype = ctypes.c_int
    lib.hadq_kv_decode_attention.argtypes = [vp, vp, vp, vp, vp, c_i32, c_i32, c_i32, c_i64, c_i64,
                                             c_i32, c_i32, vp, c_i32, c_i32, ctypes.c_float, vp,
                                             ctypes.c_int, vp, ctypes.c_size_t, vp]
    lib.hadq_kv_decode_attention.restype = ctypes.c_int
    lib.hadq_kv_decode_attention_noalloc.argtypes = [vp, vp, vp, vp, vp, c_i32, c_i32, c_i32, c_i64, c_i64,
                                                     c_i32, c_i32, vp, c_i32, c_i32, ctypes.c_float, vp,
                                                     ctypes.c_int, vp]
    lib.hadq_kv_decode_attention_noalloc.restype = ctypes.c_int
    lib.hadq_kv_decode_workspace_size.argtypes = [c_i32, c_i32, c_i32, c_i64,
                                                  ctypes.POINTER(ctypes.c_size_t)]
    lib.hadq_kv_decode_workspace_size.restype = ctypes.c_int
    lib.hadq_plan.argtypes = [c_i32, c_i64, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                              ctypes.POINTER(ctypes.c_int)]
    lib.hadq_plan.restype = ctypes.c_int
    lib.hadq_kron_plan.argtypes = [c_i32, c_i64, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.POINTER(ctypes.c_int)]
    lib.hadq_kron_plan.restype = ctypes.c_int
    lib.hadq_device_status.argtypes = [vp]
    lib.hadq_device_status.restype = ctypes.c_int
    lib.hadq_selftest_bounded_wait.argtypes = [vp, vp]
    lib.hadq_selftest_bounded_wait.restype = ctypes.c_int
    lib.hadq_status_str.argtypes = [ctypes.c_int]
    lib.hadq_status_str.restype = ctypes.c_char_p
    lib.hadq_last_error.argtypes = []
    lib.hadq_last_error.restype = ctypes.c_char_p
    lib.hadq_launch_count.argtypes = []
    lib.hadq_launch_count.restype = c_i64
    lib.hadq_version.argtypes = []
    lib.hadq_version.restype = c_i32
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != HADQ_OK:
        lib = load_library()
        msg = lib.hadq_status_str(status).decode()
        detail = lib.hadq_last_error().decode()
        raise HadqError(status, f"{msg}: {detail}" if detail else msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t, name, dtype, device, numel=None):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()}")


def _resolve(dim, block, group):
    G = dim if group == -1 else group
    return G


def hadq_status_str(status: int) -> str:
    return load_library().hadq_status_str(status).decode()


def hadq_last_error() -> str:
    return load_library().hadq_last_error().decode()


def hadq_launch_count() -> int:
    return int(load_library().hadq_launch_count())


def hadq_version() -> int:
    return int(load_library().hadq_version())


def hadq_selftest_bounded_wait(scratch, stream=None) -> int:
    """Run the bounded-wait self-test on `scratch` (a CUDA uint8 tensor of at
    least 40976 bytes); returns the status (HADQ_ERR_DEVICE expected)."""
    _need(scratch, "scratch", torch.uint8, scratch.device)
    if scratch.numel() < 40976:
        raise ValueError("scratch must hold at least 40976 bytes")
    return int(load_library().hadq_selftest_bounded_wait(_ptr(scratch), _stream(stream)))


def hadq_device_status(stream=None) -> None:
    """Synchronise the stream; raise HadqError if a bounded wait inside a
    tcgen05 kernel ran out since the last call (the record is cleared)."""
    _check(load_library().hadq_device_status(_stream(stream)))


def hadq_plan(direction: int, rows: int, dim: int, block: int = -1, bits: int = 4, group: int = -1,
              has_signs: bool = False, aligned16: bool = True) -> str:
    """Host-only: validate sizes and name the kernel family a call would use."""
    path = ctypes.c_int(0)
    _check(load_library().hadq_plan(direction, rows, dim, block, bits, group, int(has_signs),
                                    int(aligned16), ctypes.byref(path)))
    return PATH_NAMES[path.value]


def hadq_kron_plan(direction: int, rows: int, a: int, b: int, bits: int = 4, group: int = -1,
                   aligned16: bool = True) -> str:
    """Host-only: validate the sizes of a Kronecker call and name the kernel
    variant it would launch ("smem", "reg16" or "mma")."""
    v = ctypes.c_int(0)
    _check(load_library().hadq_kron_plan(direction, rows, a, b, bits, group, int(aligned16), ctypes.byref(v)))
    return KRON_VARIANTS[v.value]


def hadq_rotate_quantize(x: torch.Tensor, block: int = -1, signs: torch.Tensor | None = None,
                         bits: int = 4, group: int = -1, codes: torch.Tensor | None = None,
                         scales: torch.Tensor | None = None, rotated_out: torch.Tensor | None = None,
                         stream=None):
    """Rotate then quantise the last dimension of a bf16 CUDA tensor.

    Returns ``(codes, scales)``: int8 ``[..., dim]`` (bits 8) or uint8
    ``[..., dim/2]`` (bits 4), and float32 ``[..., dim/G]``.  ``rotated_out``
    (float32, same shape as ``x``) receives the rotated values if given.
    """
    lib = load_library()
    if x.dtype != torch.bfloat16:
        raise TypeError(f"x must be bfloat16, got {x.dtype}")
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    dim = x.shape[-1]
    rows = x.numel() // dim if dim else 0
    lead = tuple(x.shape[:-1])
    dev = x.device
    G = _resolve(dim, block, group)
    if G <= 0 or dim % G:
        _check(lib.hadq_plan(0, rows, dim, block, bits, group, 0, 1, None))
    cshape = lead + ((dim,) if bits == 8 else (dim // 2,))
    cdtype = torch.int8 if bits == 8 else torch.uint8
    if codes is None:
        codes = torch.empty(cshape, dtype=cdtype, device=dev)
    else:
        _need(codes, "codes", cdtype, dev, rows * cshape[-1])
    if scales is None:
        scales = torch.empty(lead + (dim // G,), dtype=torch.float32, device=dev)
    else:
        _need(scales, "scales", torch.float32, dev, rows * (dim // G))
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    if rotated_out is not None:
        _need(rotated_out, "rotated_out", torch.float32, dev, x.numel())
    _check(lib.hadq_rotate_quantize(_ptr(x), rows, dim, block, _ptr(signs), bits, group,
                                    _ptr(codes), _ptr(scales), _ptr(rotated_out), _stream(stream)))
    return codes, scales


def hadq_dequant_rotate_inv(codes: torch.Tensor, scales: torch.Tensor, dim: int, block: int = -1,
                            signs: torch.Tensor | None = None, bits: int = 4, group: int = -1,
                            out: torch.Tensor | None = None, out_dtype: torch.dtype = torch.bfloat16,
                            stream=None) -> torch.Tensor:
    """Dequantise codes and undo the rotation; returns ``[..., dim]`` bf16 or fp32."""
    lib = load_library()
    if not codes.is_cuda or not codes.is_contiguous():
        raise ValueError("codes must be a contiguous CUDA tensor")
    dev = codes.device
    per_row = dim if bits == 8 else dim // 2
    if per_row <= 0:
        _check(lib.hadq_plan(1, 0, dim, block, bits, group, 0, 1, None))
    rows = codes.numel() // per_row
    lead = tuple(codes.shape[:-1]) if codes.shape[-1] == per_row else (rows,)
    G = _resolve(dim, block, group)
    if G <= 0 or dim % G:
        _check(lib.hadq_plan(1, rows, dim, block, bits, group, 0, 1, None))
    _need(scales, "scales", torch.float32, dev, rows * (dim // G))
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")
    if out is None:
        out = torch.empty(lead + (dim,), dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev, rows * dim)
    code = HADQ_OUT_F32 if out_dtype == torch.float32 else HADQ_OUT_BF16
    _check(lib.hadq_dequant_rotate_inv(_ptr(codes), _ptr(scales), rows, dim, block, _ptr(signs), bits,
                                       group, _ptr(out), code, _stream(stream)))
    return out


def hadq_kv_decode_workspace_size(batch: int, n_q_heads: int, n_kv_heads: int, tokens: int) -> int:
    """Host-only: workspace bytes :func:`hadq_kv_decode_attention` needs (any GPU)."""
    n = ctypes.c_size_t(0)
    _check(load_library().hadq_kv_decode_workspace_size(batch, n_q_heads, n_kv_heads, tokens,
                                                        ctypes.byref(n)))
    return int(n.value)


def hadq_kv_decode_attention(q: torch.Tensor, k_codes: torch.Tensor, k_scales: torch.Tensor,
                             v_codes: torch.Tensor, v_scales: torch.Tensor, tokens: int | None = None,
                             block: int = -1, signs: torch.Tensor | None = None, bits: int = 4,
                             group: int = -1, softmax_scale: float | None = None,
                             out: torch.Tensor | None = None, out_dtype: torch.dtype = torch.bfloat16,
                             workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One decode step of attention over a rotated INT4 or INT8 KV cache.

    ``q``: bf16 ``[batch, n_q_heads, dim]``.  ``k_codes``/``v_codes``: uint8
    ``[batch, n_kv_heads, token_stride, dim/2]`` (INT4) or uint8/int8 ``[...,
    dim]`` (INT8, ``bits=8``); ``k_scales``/``v_scales``:
    float32 ``[batch, n_kv_heads, token_stride, dim/group]`` (one scale per row
    for group 128 or -1, which may drop the trailing 1).
    ``tokens`` (default ``token_stride``) rows of each head are attended over.
    ``workspace``: a zero-filled uint8 CUDA tensor of at least
    :func:`hadq_kv_decode_workspace_size` bytes, reused across calls (one is
    allocated when omitted).  Returns ``[batch, n_q_heads, dim]`` bf16 or fp32.
    """
    lib = load_library()
    if q.dtype != torch.bfloat16:
        raise TypeError(f"q must be bfloat16, got {q.dtype}")
    if q.dim() != 3 or not q.is_cuda or not q.is_contiguous():
        raise ValueError("q must be a contiguous CUDA tensor [batch, n_q_heads, dim]")
    batch, nqh, dim = q.shape
    dev = q.device
    if k_codes.dim() != 4 or v_codes.shape != k_codes.shape:
        raise ValueError("k_codes and v_codes must be [batch, n_kv_heads, token_stride, dim*bits/8] alike")
    nkv, stride = k_codes.shape[1], k_codes.shape[2]
    if k_codes.shape[0] != batch:
        raise ValueError("k_codes batch differs from q")
    per_row = k_codes.shape[3]
    if tokens is None:
        tokens = stride
    for name, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        if t.dtype == torch.int8:  # INT8 caches may come as int8
            t = t.view(torch.uint8)
        _need(t, name, torch.uint8, dev)
    per_scale = dim // _resolve(dim, block, group) if group != 0 and dim % _resolve(dim, block, group) == 0 else 1
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _need(t, name, torch.float32, dev, batch * nkv * stride * per_scale)
    if per_row * 8 != dim * bits:
        raise ValueError(f"codes rows hold {per_row} bytes, expected dim*bits/8 = {dim * bits // 8}")
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    if softmax_scale is None:
        softmax_scale = 1.0 / float(dim) ** 0.5
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")
    if out is None:
        out = torch.empty((batch, nqh, dim), dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev, batch * nqh * dim)
    need = hadq_kv_decode_workspace_size(batch, nqh, nkv, tokens) if batch else 0
    if workspace is None:
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=dev)
    else:
        _need(workspace, "workspace", torch.uint8, dev)
    code = HADQ_OUT_F32 if out_dtype == torch.float32 else HADQ_OUT_BF16
    _check(lib.hadq_kv_decode_attention(_ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes),
                                        _ptr(v_scales), batch, nqh, nkv, tokens, stride, dim, block,
                                        _ptr(signs), bits, group, float(softmax_scale), _ptr(out), code,
                                        _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def hadq_kv_decode_attention_noalloc(q: torch.Tensor, k_codes: torch.Tensor, k_scales: torch.Tensor,
                                     v_codes: torch.Tensor, v_scales: torch.Tensor, out: torch.Tensor,
                                     tokens: int | None = None, block: int = -1,
                                     signs: torch.Tensor | None = None, bits: int = 4, group: int = -1,
                                     softmax_scale: float | None = None, stream=None) -> torch.Tensor:
    """:func:`hadq_kv_decode_attention` on the library's static scratch.

    Nothing is allocated: ``out`` (bf16 or fp32 ``[batch, n_q_heads, dim]``)
    is required and the partials use the scratch the library holds.
    """
    lib = load_library()
    if q.dtype != torch.bfloat16 or q.dim() != 3 or not q.is_cuda or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 CUDA tensor [batch, n_q_heads, dim]")
    batch, nqh, dim = q.shape
    dev = q.device
    if k_codes.dim() != 4 or v_codes.shape != k_codes.shape or k_codes.shape[0] != batch:
        raise ValueError("k_codes and v_codes must be [batch, n_kv_heads, token_stride, dim*bits/8] alike")
    nkv, stride = k_codes.shape[1], k_codes.shape[2]
    for name, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        if t.dtype == torch.int8:  # INT8 caches may come as int8
            t = t.view(torch.uint8)
        _need(t, name, torch.uint8, dev)
    if k_codes.shape[3] * 8 != dim * bits:
        raise ValueError(f"codes rows hold {k_codes.shape[3]} bytes, expected dim*bits/8 = {dim * bits // 8}")
    per_scale = dim // _resolve(dim, block, group) if group != 0 and dim % _resolve(dim, block, group) == 0 else 1
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _need(t, name, torch.float32, dev, batch * nkv * stride * per_scale)
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, dev, batch * nqh * dim)
    if softmax_scale is None:
        softmax_scale = 1.0 / float(dim) ** 0.5
    code = HADQ_OUT_F32 if out.dtype == torch.float32 else HADQ_OUT_BF16
    _check(lib.hadq_kv_decode_attention_noalloc(
        _ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales), batch, nqh, nkv,
        stride if tokens is None else tokens, stride, dim, block, _ptr(signs), bits, group,
        float(softmax_scale), _ptr(out), code, _stream(stream)))
    return out


def hyquant_keep_slots(tokens: int, n_sink: int = 0, window: int = 0, vertical=()):
    """Host helper: the keep table of a HyQuant-style token set.

    Kept tokens are the first ``n_sink`` tokens, the last ``window`` tokens and
    the ``vertical`` token indices; each gets its rank among the kept tokens
    (ascending token order) as its slot.  Returns ``(keep_slot int32
    [tokens] with -1 for quantised tokens, n_keep)``.
    """
    import numpy as np
    kept = set(range(min(n_sink, tokens))) | set(range(max(0, tokens - window), tokens))
    for t in vertical:
        if not 0 <= int(t) < tokens:
            raise ValueError(f"vertical token {t} outside [0, {tokens})")
        kept.add(int(t))
    slots = np.full(tokens, -1, dtype=np.int32)
    for rank, t in enumerate(sorted(kept)):
        slots[t] = rank
    return slots, len(kept)


def hadq_rotate_quantize_keep(x: torch.Tensor, keep_slot: torch.Tensor, n_keep: int, block: int = -1,
                              signs: torch.Tensor | None = None, bits: int = 4, group: int = -1,
                              codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                              kept: torch.Tensor | None = None, stream=None):
    """Mixed-precision rotate+quantise of a bf16 ``[heads, tokens, dim]`` tensor.

    ``keep_slot``: int32 CUDA tensor ``[tokens]``; token t is kept when
    ``keep_slot[t]`` is in ``[0, n_keep)``.  Returns ``(codes, scales, kept)``
    with ``kept`` bf16 ``[heads, n_keep, dim]``; kept rows get codes 0 and
    scale 0.
    """
    lib = load_library()
    if x.dtype != torch.bfloat16 or x.dim() != 3 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor [heads, tokens, dim]")
    heads, tokens, dim = x.shape
    dev = x.device
    _need(keep_slot, "keep_slot", torch.int32, dev, tokens)
    G = _resolve(dim, block, group)
    if G <= 0 or dim % G:
        _check(lib.hadq_plan(0, heads * tokens, dim, block, bits, group, 0, 1, None))
    cdim = dim if bits == 8 else dim // 2
    cdt = torch.int8 if bits == 8 else torch.uint8
    if codes is None:
        codes = torch.empty((heads, tokens, cdim), dtype=cdt, device=dev)
    else:
        _need(codes, "codes", cdt, dev, heads * tokens * cdim)
    if scales is None:
        scales = torch.empty((heads, tokens, dim // G), dtype=torch.float32, device=dev)
    else:
        _need(scales, "scales", torch.float32, dev, heads * tokens * (dim // G))
    if kept is None:
        kept = torch.empty((heads, n_keep, dim), dtype=torch.bfloat16, device=dev)
    else:
        _need(kept, "kept", torch.bfloat16, dev, heads * n_keep * dim)
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    _check(lib.hadq_rotate_quantize_keep(_ptr(x), heads, tokens, dim, block, _ptr(signs), bits, group,
                                         _ptr(keep_slot), n_keep, _ptr(codes), _ptr(scales),
                                         _ptr(kept) if n_keep else None, _stream(stream)))
    return codes, scales, kept


def hadq_dequant_rotate_inv_keep(codes: torch.Tensor, scales: torch.Tensor, kept: torch.Tensor,
                                 keep_slot: torch.Tensor, n_keep: int, dim: int, block: int = -1,
                                 signs: torch.Tensor | None = None, bits: int = 4, group: int = -1,
                                 out: torch.Tensor | None = None, out_dtype: torch.dtype = torch.bfloat16,
                                 stream=None) -> torch.Tensor:
    """Reads a mixed-precision cache back to ``[heads, tokens, dim]`` bf16 or
    fp32: kept tokens return their stored bf16 rows exactly."""
    lib = load_library()
    if codes.dim() != 3 or not codes.is_cuda or not codes.is_contiguous():
        raise ValueError("codes must be a contiguous CUDA tensor [heads, tokens, dim or dim/2]")
    heads, tokens, _ = codes.shape
    dev = codes.device
    _need(keep_slot, "keep_slot", torch.int32, dev, tokens)
    _need(kept, "kept", torch.bfloat16, dev, heads * n_keep * dim)
    G = _resolve(dim, block, group)
    if G <= 0 or dim % G:
        _check(lib.hadq_plan(1, heads * tokens, dim, block, bits, group, 0, 1, None))
    _need(scales, "scales", torch.float32, dev, heads * tokens * (dim // G))
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")
    if out is None:
        out = torch.empty((heads, tokens, dim), dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev, heads * tokens * dim)
    code = HADQ_OUT_F32 if out_dtype == torch.float32 else HADQ_OUT_BF16
    _check(lib.hadq_dequant_rotate_inv_keep(_ptr(codes), _ptr(scales), _ptr(kept) if n_keep else None,
                                            _ptr(keep_slot), n_keep, heads, tokens, dim, block, _ptr(signs),
                                            bits, group, _ptr(out), code, _stream(stream)))
    return out


def hadq_rotate_quantize_asym(x: torch.Tensor, block: int = -1, signs: torch.Tensor | None = None,
                              bits: int = 4, group: int = -1, codes: torch.Tensor | None = None,
                              scales: torch.Tensor | None = None, zero_points: torch.Tensor | None = None,
                              stream=None):
    """Rotate, then quantise with a zero point (unsigned codes).

    Returns ``(codes, scales, zero_points)``: uint8 ``[..., dim]`` (bits 8) or
    ``[..., dim/2]`` (bits 4), float32 ``[..., dim/G]`` and uint8 ``[..., dim/G]``.
    """
    lib = load_library()
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    dim = x.shape[-1]
    rows = x.numel() // dim if dim else 0
    lead = tuple(x.shape[:-1])
    dev = x.device
    G = _resolve(dim, block, group)
    if G <= 0 or dim % G:
        _check(lib.hadq_plan(0, rows, dim, block, bits, group, 0, 1, None))
    cdim = dim if bits == 8 else dim // 2
    if codes is None:
        codes = torch.empty(lead + (cdim,), dtype=torch.uint8, device=dev)
    else:
        _need(codes, "codes", torch.uint8, dev, rows * cdim)
    if scales is None:
        scales = torch.empty(lead + (dim // G,), dtype=torch.float32, device=dev)
    else:
        _need(scales, "scales", torch.float32, dev, rows * (dim // G))
    if zero_points is None:
        zero_points = torch.empty(lead + (dim // G,), dtype=torch.uint8, device=dev)
    else:
        _need(zero_points, "zero_points", torch.uint8, dev, rows * (dim // G))
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    _check(lib.hadq_rotate_quantize_asym(_ptr(x), rows, dim, block, _ptr(signs), bits, group, _ptr(codes),
                                         _ptr(scales), _ptr(zero_points), _stream(stream)))
    return codes, scales, zero_points


def hadq_dequant_rotate_inv_asym(codes: torch.Tensor, scales: torch.Tensor, zero_points: torch.Tensor,
                                 dim: int, block: int = -1, signs: torch.Tensor | None = None,
                                 bits: int = 4, group: int = -1, out: torch.Tensor | None = None,
                                 out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """(codes - zero_point) * scale, then the inverse rotation; ``[..., dim]``."""
    lib = load_library()
    if not codes.is_cuda or not codes.is_contiguous():
        raise ValueError("codes must be a contiguous CUDA tensor")
    dev = codes.device
    per_row = dim if bits == 8 else dim // 2
    if per_row <= 0:
        _check(lib.hadq_plan(1, 0, dim, block, bits, group, 0, 1, None))
    rows = codes.numel() // per_row
    lead = tuple(codes.shape[:-1]) if codes.shape[-1] == per_row else (rows,)
    G = _resolve(dim, block, group)
    if G <= 0 or dim % G:
        _check(lib.hadq_plan(1, rows, dim, block, bits, group, 0, 1, None))
    _need(scales, "scales", torch.float32, dev, rows * (dim // G))
    _need(zero_points, "zero_points", torch.uint8, dev, rows * (dim // G))
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")
    if out is None:
        out = torch.empty(lead + (dim,), dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev, rows * dim)
    code = HADQ_OUT_F32 if out_dtype == torch.float32 else HADQ_OUT_BF16
    _check(lib.hadq_dequant_rotate_inv_asym(_ptr(codes), _ptr(scales), _ptr(zero_points), rows, dim, block,
                                            _ptr(signs), bits, group, _ptr(out), code, _stream(stream)))
    return out


def hadq_rotate_quantize_kron(x: torch.Tensor, fa: torch.Tensor, b: int, signs: torch.Tensor | None = None,
                              bits: int = 4, group: int = -1, codes: torch.Tensor | None = None,
                              scales: torch.Tensor | None = None, rotated_out: torch.Tensor | None = None,
                              stream=None):
    """Kronecker rotation (F (x) H_b) then quantisation of a bf16 ``[..., a * b]``
    tensor; ``fa``: float32 CUDA ``[a, a]`` (as it multiplies).  Returns
    ``(codes, scales)`` as :func:`hadq_rotate_quantize`."""
    return _kron_forward(False, x, fa, b, signs, bits, group, codes, scales, rotated_out, stream)


def hadq_rotate_quantize_kron_pm1(x: torch.Tensor, sa: torch.Tensor, b: int, signs: torch.Tensor | None = None,
                                  bits: int = 4, group: int = -1, codes: torch.Tensor | None = None,
                                  scales: torch.Tensor | None = None, rotated_out: torch.Tensor | None = None,
                                  stream=None):
    """As :func:`hadq_rotate_quantize_kron` with the factor given as a +-1
    matrix: ``sa`` int8 CUDA ``[a, a]``, F = sa / sqrt(a)."""
    return _kron_forward(True, x, sa, b, signs, bits, group, codes, scales, rotated_out, stream)


def _kron_forward(pm1, x, fa, b, signs, bits, group, codes, scales, rotated_out, stream):
    lib = load_library()
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    if fa.dim() != 2 or fa.shape[0] != fa.shape[1]:
        raise ValueError("fa must be a square [a, a] matrix")
    a = fa.shape[0]
    dim = x.shape[-1]
    if dim != a * b:
        raise ValueError(f"rows of {dim} columns do not match a * b = {a * b}")
    dev = x.device
    _need(fa, "sa" if pm1 else "fa", torch.int8 if pm1 else torch.float32, dev)
    rows = x.numel() // dim
    lead = tuple(x.shape[:-1])
    G = _resolve(dim, b, group)
    if G <= 0 or dim % G:
        _check(lib.hadq_plan(0, rows, dim, b, bits, group, 0, 1, None))
    cshape = lead + ((dim,) if bits == 8 else (dim // 2,))
    cdtype = torch.int8 if bits == 8 else torch.uint8
    if codes is None:
        codes = torch.empty(cshape, dtype=cdtype, device=dev)
    else:
        _need(codes, "codes", cdtype, dev, rows * cshape[-1])
    if scales is None:
        scales = torch.empty(lead + (dim // G,), dtype=torch.float32, device=dev)
    else:
        _need(scales, "scales", torch.float32, dev, rows * (dim // G))
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    if rotated_out is not None:
        _need(rotated_out, "rotated_out", torch.float32, dev, x.numel())
    fn = lib.hadq_rotate_quantize_kron_pm1 if pm1 else lib.hadq_rotate_quantize_kron
    _check(fn(_ptr(x), rows, a, _ptr(fa), b, _ptr(signs), bits, group, _ptr(codes), _ptr(scales), _ptr(rotated_out),
              _stream(stream)))
    return codes, scales


def hadq_dequant_rotate_inv_kron(codes: torch.Tensor, scales: torch.Tensor, fa: torch.Tensor, b: int,
                                 signs: torch.Tensor | None = None, bits: int = 4, group: int = -1,
                                 out: torch.Tensor | None = None, out_dtype: torch.dtype = torch.bfloat16,
                                 stream=None) -> torch.Tensor:
    """Inverse of :func:`hadq_rotate_quantize_kron`: ``[..., a * b]`` bf16 or fp32."""
    return _kron_inverse(False, codes, scales, fa, b, signs, bits, group, out, out_dtype, stream)


def hadq_dequant_rotate_inv_kron_pm1(codes: torch.Tensor, scales: torch.Tensor, sa: torch.Tensor, b: int,
                                     signs: torch.Tensor | None = None, bits: int = 4, group: int = -1,
                                     out: torch.Tensor | None = None, out_dtype: torch.dtype = torch.bfloat16,
                                     stream=None) -> torch.Tensor:
    """Inverse of :func:`hadq_rotate_quantize_kron_pm1` (``sa`` int8 +-1 ``[a, a]``)."""
    return _kron_inverse(True, codes, scales, sa, b, signs, bits, group, out, out_dtype, stream)


def _kron_inverse(pm1, codes, scales, fa, b, signs, bits, group, out, out_dtype, stream):
    lib = load_library()
    if not codes.is_cuda or not codes.is_contiguous():
        raise ValueError("codes must be a contiguous CUDA tensor")
    a = fa.shape[0]
    dim = a * b
    dev = codes.device
    _need(fa, "sa" if pm1 else "fa", torch.int8 if pm1 else torch.float32, dev, a * a)
    per_row = dim if bits == 8 else dim // 2
    rows = codes.numel() // per_row
    lead = tuple(codes.shape[:-1]) if codes.shape[-1] == per_row else (rows,)
    G = _resolve(dim, b, group)
    if G <= 0 or dim % G:
        _check(lib.hadq_plan(1, rows, dim, b, bits, group, 0, 1, None))
    _need(scales, "scales", torch.float32, dev, rows * (dim // G))
    if signs is not None:
        _need(signs, "signs", torch.int8, dev, dim)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")
    if out is None:
        out = torch.empty(lead + (dim,), dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev, rows * dim)
    code = HADQ_OUT_F32 if out_dtype == torch.float32 else HADQ_OUT_BF16
    fn = lib.hadq_dequant_rotate_inv_kron_pm1 if pm1 else lib.hadq_dequant_rotate_inv_kron
    _check(fn(_ptr(codes), _ptr(scales), rows, a, _ptr(fa), b, _ptr(signs), bits, group, _ptr(out), code,
              _stream(stream)))
    return out
