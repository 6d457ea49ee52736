"""Device-resident workload steps: what one pass of the hot path launches.

A step is one rotate+quantise launch over every input row of a workload (the
tensors of a workload, e.g. Q and K, are stored back to back in one bf16
buffer because they share one recipe), followed, for workloads that read
their codes back (the KV cache), by one dequantise+inverse launch to bf16.
Buffers are allocated once with torch; the launches go through the C ABI.
"""

from __future__ import annotations

import numpy as np
import torch

from . import binding as B
from . import synthetic as S


def bits_to_bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bit patterns (numpy) -> bf16 torch tensor on ``device``."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def bf16_tensor_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class WorkloadStep:
    """Inputs, outputs and launches of one workload on one device."""

    def __init__(self, wl: S.Workload, device="cuda", seed: int = S.DEFAULT_SEED,
                 x_bits: np.ndarray | None = None, pinned_host: bool = False):
        self.wl = wl
        self.device = torch.device(device)
        dim = wl.dim
        if x_bits is None:
            x_bits = np.concatenate([S.tensor(wl, i, seed) for i in range(len(wl.tensors))], axis=0)
        assert x_bits.shape == (wl.rows, dim)
        self.rows = wl.rows
        host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16)
        if pinned_host:
            self.x_host = host.pin_memory()
        else:
            self.x_host = None
        self.x = host.to(self.device)
        s = S.signs(wl, seed)
        self.signs = None if s is None else torch.from_numpy(s).to(self.device)
        G = dim if wl.group == -1 else wl.group
        cdim = dim if wl.bits == 8 else dim // 2
        cdt = torch.int8 if wl.bits == 8 else torch.uint8
        if wl.asym:
            cdt = torch.uint8
        self.codes = torch.empty((self.rows, cdim), dtype=cdt, device=self.device)
        self.scales = torch.empty((self.rows, dim // G), dtype=torch.float32, device=self.device)
        self.zero_points = (torch.empty((self.rows, dim // G), dtype=torch.uint8, device=self.device)
                            if wl.asym else None)
        self.out = (torch.empty((self.rows, dim), dtype=torch.bfloat16, device=self.device)
                    if wl.dequant else None)
        self.sa = None   # the stored +-1 factor S_a of a Kronecker workload (F = S_a / sqrt(a))
        if wl.kron_a:
            self.sa = torch.from_numpy(S.paley_hadamard(wl.kron_a - 1)).to(self.device)
        self.keep_slot = self.kept = None
        if wl.keep:
            n_sink, window, n_vertical = wl.keep
            vert = S.vertical_tokens(wl.tokens, n_vertical, seed, n_sink, window)
            slots, n_keep = B.hyquant_keep_slots(wl.tokens, n_sink, window, vert)
            assert n_keep == wl.n_keep
            self.keep_slot_host = slots
            self.keep_slot = torch.from_numpy(slots).to(self.device)
            self.kept = torch.empty((wl.heads, n_keep, dim), dtype=torch.bfloat16, device=self.device)

    @property
    def launches_per_step(self) -> int:
        return 2 if self.wl.dequant else 1

    @property
    def bytes_per_step(self) -> int:
        """Algorithmic bytes of one step (each byte read or written once)."""
        b = self.wl.quant_bytes()
        if self.wl.dequant:
            b += self.wl.dequant_bytes(2)
        return b

    def quantize(self, stream=None, rotated_out=None):
        wl = self.wl
        if wl.kron_a:
            B.hadq_rotate_quantize_kron_pm1(self.x, self.sa, wl.dim // wl.kron_a, signs=self.signs, bits=wl.bits,
                                        group=wl.group, codes=self.codes, scales=self.scales,
                                        rotated_out=rotated_out, stream=stream)
            return
        if wl.asym:
            B.hadq_rotate_quantize_asym(self.x, block=wl.block, signs=self.signs, bits=wl.bits, group=wl.group,
                                        codes=self.codes, scales=self.scales, zero_points=self.zero_points,
                                        stream=stream)
            return
        if wl.keep:
            h, t = wl.heads, wl.tokens
            B.hadq_rotate_quantize_keep(self.x.view(h, t, wl.dim), self.keep_slot, wl.n_keep, block=wl.block,
                                        signs=self.signs, bits=wl.bits, group=wl.group,
                                        codes=self.codes.view(h, t, -1), scales=self.scales.view(h, t, -1),
                                        kept=self.kept, stream=stream)
            return
        B.hadq_rotate_quantize(self.x, block=wl.block, signs=self.signs, bits=wl.bits, group=wl.group,
                               codes=self.codes, scales=self.scales, rotated_out=rotated_out,
                               stream=stream)

    def dequantize(self, stream=None, out=None, out_dtype=torch.bfloat16):
        wl = self.wl
        out = self.out if out is None else out
        if wl.asym:
            return B.hadq_dequant_rotate_inv_asym(self.codes, self.scales, self.zero_points, wl.dim,
                                                  block=wl.block, signs=self.signs, bits=wl.bits, group=wl.group,
                                                  out=out, out_dtype=out_dtype, stream=stream)
        if wl.keep:
            h, t = wl.heads, wl.tokens
            return B.hadq_dequant_rotate_inv_keep(self.codes.view(h, t, -1), self.scales.view(h, t, -1),
                                                  self.kept, self.keep_slot, wl.n_keep, wl.dim, block=wl.block,
                                                  signs=self.signs, bits=wl.bits, group=wl.group,
                                                  out=out.view(h, t, wl.dim), out_dtype=out_dtype,
                                                  stream=stream)
        return B.hadq_dequant_rotate_inv(self.codes, self.scales, wl.dim, block=wl.block,
                                         signs=self.signs, bits=wl.bits, group=wl.group,
                                         out=out, out_dtype=out_dtype, stream=stream)

    def step(self, stream=None):
        self.quantize(stream)
        if self.wl.dequant:
            self.dequantize(stream)
