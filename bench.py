#!/usr/bin/env python
"""Benchmark of the fused Hadamard rotate + quantise step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the hot path over the workload's whole batch: one
rotate+quantise launch over every input row (plus, for the KV-cache workload,
one dequantise+inverse launch to bf16).  The decode workload
(``--workload d1_decode_q32_kv8_t131072_d128_int4``) instead times one decode
step of attention over the rotated INT4 KV cache: one launch that reads every
cached K/V code and scale once.  Inputs are resident in HBM before the
timed region.  Between timed steps a 256 MiB buffer is written to flush the
126 MB L2; that write sits outside the CUDA events that time each step.  The
default workload is the largest of the five synthetic configurations: 32768
tokens x 11008 columns of Student-t(3) bf16 values, seeded signs, 86 blocks of
the 128-point Hadamard, INT4 codes with one fp32 scale per 128 columns.

The same line carries ``per_config``: every one of the five configurations
(and the KV-cache dequantiser) timed the same way, plus a ``sustained``
figure per kernel taken back to back with no flush, where each launch also
pays the write-back of the previous launch's outputs still dirty in L2.
Fractions are given against the measured copy bandwidth and against the
nominal 8 TB/s of the B200's HBM3e.

Multi-GPU (torchrun, one process per GPU): rows are independent, so every rank
runs its own copy of the workload with no data-path collective ("weak"
scaling); the process group only provides the barrier and the max over ranks
of the timed duration.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
instead (rank 0 only, bounded samples of the same workload).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "c5_tok32768_w11008_b128_signs_int4_g128"
PER_CONFIG = ["c1_tok256_h4096_b128_int4", "c2_qk_h32_s8192_d128_int8", "c3_tok16384_h4096_full_signs_int4",
              "c4_kv_h8_t131072_d128_int4_g128", "c5_tok32768_w11008_b128_signs_int4_g128"]
METRIC = "fused Hadamard+quantize GB/s (bf16 in→int4/int8 out), % of B200 HBM peak"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, vendor figure
L2_FLUSH_BYTES = 256 << 20
KERNEL_NAMES = {"blocked": "rq_blocked_kernel", "full4096": "rq_full4096_kernel",
                "generic": "rq_generic_kernel", "chunk": "rq_chunk_kernel",
                "wide4096": "rq_wide4096_kernel", "wide4096_mma": "rq_h4096_mma_kernel",
                "chunk_mma": "rq_chunk_mma_kernel", "h4096_tc": "rq_h4096_tc_kernel", "none": None}
KRON_KERNELS = {"smem": "rq_kron_kernel", "reg16": "rq_kron16_kernel", "mma": "rq_kron_tc_kernel"}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="target CPU time of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-per-config", action="store_true",
                   help="time only the headline workload")
    p.add_argument("--config-steps", type=int, default=50,
                   help="timed steps per per_config entry (flushed and back to back each)")
    return p.parse_args(argv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


from hadamard_rotation_outlier_b200.records import (KERNEL_SOURCES, kernel_source_hash,  # noqa: E402,F401
                                                    recorded_parity, recorded_traffic, workload_family)


# ------------------------------------------------------------------ clocks

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Reads SM clock and clock-event reasons through NVML while the GPU works."""

    def __init__(self, device_index: int):
        self.ok = False
        self.sm = []
        self.reasons = set()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report clocks as unavailable
            self.ok = False

    def sample(self):
        if not self.ok:
            return
        try:
            self.sm.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
            r = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in _REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def poll_until(self, event, min_samples: int = 3):
        """Sample while ``event`` (a CUDA event recorded after the work) is pending."""
        n = 0
        while not event.query() or n < min_samples:
            self.sample()
            n += 1
            if event.query() and n >= min_samples:
                break
            time.sleep(0.0005)

    def summary(self):
        if not self.ok or not self.sm:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml_unavailable"]}
        return {"sm_mhz": float(statistics.median(self.sm)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.sm)}


# ------------------------------------------------------------ CPU oracle

def cpu_threads() -> int:
    """Threads of the BLAS pool the oracle's matrix products run on."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def single_thread(fn, *a, **kw):
    """``fn(*a, **kw)`` with the BLAS pool limited to one thread."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(1):
        return fn(*a, **kw)


def oracle_sample_rate(wl, target_s: float, seed: int = 42):
    """Time the oracle on a bounded row sample of ``wl``; returns (GB/s, info)."""
    import oracle as O
    from hadamard_rotation_outlier_b200 import synthetic as S

    signs = S.signs(wl, seed)
    t0 = wl.tensors[0]

    fa = None
    if wl.kron_a:
        fa = S.paley_hadamard(wl.kron_a - 1).astype(np.float64) / np.sqrt(wl.kron_a)

    def run(nrows):
        x = S.tensor_rows(wl, 0, 0, nrows, seed)
        t = time.perf_counter()
        if wl.kron_a:
            O.rotate_quantize_kron(x, fa, wl.dim // wl.kron_a, signs, wl.bits, wl.group)
        elif wl.asym:
            r = O.rotate_quantize_asym(x, block=wl.block, signs=signs, bits=wl.bits, group=wl.group)
            O.dequant_rotate_inv_asym(r["codes"], r["scales"], r["zero_points"], wl.dim, block=wl.block,
                                      signs=signs, bits=wl.bits, group=wl.group)
        elif wl.keep:  # the sample's rows as one head of consecutive tokens, first n_sink kept
            slots = np.full(nrows, -1, np.int32)
            slots[:min(nrows, wl.keep[0])] = np.arange(min(nrows, wl.keep[0]))
            r = O.rotate_quantize_keep(x, 1, nrows, slots, wl.keep[0], block=wl.block, signs=signs,
                                       bits=wl.bits, group=wl.group)
            O.dequant_rotate_inv_keep(r["codes"], r["scales"], r["kept"], slots, wl.keep[0], 1, nrows, wl.dim,
                                      block=wl.block, signs=signs, bits=wl.bits, group=wl.group)
        else:
            r = O.rotate_quantize(x, block=wl.block, signs=signs, bits=wl.bits, group=wl.group)
            if wl.dequant:
                O.dequant_rotate_inv(r["codes"], r["scales"], wl.dim, block=wl.block, signs=signs,
                                     bits=wl.bits, group=wl.group)
        return time.perf_counter() - t

    n = min(t0.rows, max(1, (1 << 20) // wl.dim))
    dt = run(n)
    while dt < 0.2 * target_s and n < t0.rows:
        n = min(t0.rows, int(n * min(8.0, max(2.0, 0.5 * target_s / max(dt, 1e-3)))))
        dt = run(n)
    # a whole first tensor that still takes less than half the target: repeat it
    passes = 1
    while dt < 0.5 * target_s and passes < 64:
        dt += run(n)
        passes += 1
    frac = n * passes / wl.rows
    nbytes = wl.quant_bytes() * frac + (wl.dequant_bytes(2) * frac if wl.dequant else 0)
    info = {"rows": n, "passes": passes, "seconds": round(dt, 3), "bytes": int(nbytes)}
    return nbytes / dt / 1e9, info


# -------------------------------------------------------------- GPU arm

def _dist_setup(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(world, value: float, device="cuda") -> float:
    """Max of a per-rank duration over all ranks (the job's time)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class L2Flush:
    """Evicts the 126 MB L2 between steps: writes one 256 MiB buffer, then reads
    another so that the written (dirty) lines are flushed to HBM here, not
    during the next timed step."""

    def __init__(self, device):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.sink = torch.zeros((), dtype=torch.float32, device=device)

    def __call__(self):
        self.w.fill_(1)
        self.sink.copy_(self.r.sum())


def hold_cycles(steps: int, host_us_per_step: float = 150.0, clock_ghz: float = 2.0) -> int:
    """Device-sleep length that covers the host enqueueing `steps` steps."""
    return int((2000.0 + steps * host_us_per_step) * 1e3 * clock_ghz)


def aggregate_gbs(world: int, bytes_per_step: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: every rank processes its own batch (weak scaling)."""
    return world * bytes_per_step * steps / (total_ms * 1e-3) / 1e9


DECODE_METRIC = ("decode attention over the rotated INT4 KV cache, GB/s (bf16 query + K/V codes + "
                 "K/V scales in, bf16 out), % of B200 HBM peak")


def decode_oracle_rate(dw, target_s: float, seed: int = 71):
    """Time the oracle's decode attention on a bounded token sample of ``dw``
    (one KV head and its query heads); returns (GB/s, info)."""
    import oracle as O
    from hadamard_rotation_outlier_b200 import synthetic as S

    g = dw.n_q_heads // dw.n_kv_heads
    q = S.decode_query(1, g, dw.dim, seed)

    def run(tokens):
        kc, ks = S.random_int4_cache(1, 1, tokens, dw.dim, seed + 1)
        vc, vs = S.random_int4_cache(1, 1, tokens, dw.dim, seed + 2)
        t = time.perf_counter()
        O.kv_decode_attention(q, kc, ks, vc, vs, dw.dim, 128, None, 4, 128)
        return time.perf_counter() - t

    n = 4096
    dt = run(n)
    while dt < 0.2 * target_s and n < dw.tokens:
        n = min(dw.tokens, int(n * min(8.0, max(2.0, 0.5 * target_s / max(dt, 1e-3)))))
        dt = run(n)
    nbytes = 2 * g * dw.dim + 2 * n * (dw.dim // 2) + 2 * n * 4 + 2 * g * dw.dim
    info = {"tokens": n, "q_heads": g, "seconds": round(dt, 3), "bytes": int(nbytes)}
    return nbytes / dt / 1e9, info


def run_decode(args):
    """One decode step of attention per timed step (see the module note)."""
    import torch
    from hadamard_rotation_outlier_b200 import binding as B
    from hadamard_rotation_outlier_b200 import synthetic as S
    from hadamard_rotation_outlier_b200.build import build

    dw = S.DECODE_WORKLOADS[args.workload]
    world, rank, local = _dist_setup(args)
    if rank == 0:
        build()
    _barrier(world)
    B.load_library()
    warmup = max(3, args.warmup)
    steps = max(1, args.steps)
    dev = torch.device("cuda", local if world > 1 else 0)
    seed = 71 + rank
    kc, ks = S.random_int4_cache(dw.batch, dw.n_kv_heads, dw.tokens, dw.dim, seed)
    vc, vs = S.random_int4_cache(dw.batch, dw.n_kv_heads, dw.tokens, dw.dim, seed + 1000)
    qbits = S.decode_query(dw.batch, dw.n_q_heads, dw.dim, seed)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    k_codes, k_scales, v_codes, v_scales = to_dev(kc), to_dev(ks), to_dev(vc), to_dev(vs)
    q = to_dev(qbits.view(np.int16)).view(torch.bfloat16)
    out = torch.empty((dw.batch, dw.n_q_heads, dw.dim), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(B.hadq_kv_decode_workspace_size(dw.batch, dw.n_q_heads, dw.n_kv_heads, dw.tokens),
                     dtype=torch.uint8, device=dev)
    flusher = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step(qt, o, s):
        B.hadq_kv_decode_attention(qt, k_codes, k_scales, v_codes, v_scales, tokens=dw.tokens, block=128,
                                   bits=4, group=128, out=o, workspace=ws, stream=s)

    for _ in range(warmup):
        flusher()
        step(q, out, stream)
    torch.cuda.synchronize(dev)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    done = torch.cuda.Event()
    clocks = ClockSampler(dev.index)
    _barrier(world)
    torch.cuda.synchronize(dev)
    n0 = B.hadq_launch_count()
    torch.cuda._sleep(hold_cycles(steps))
    for i in range(steps):
        flusher()
        starts[i].record(stream)
        step(q, out, stream)
        ends[i].record(stream)
    done.record(stream)
    clocks.poll_until(done)
    torch.cuda.synchronize(dev)
    _barrier(world)
    launches = B.hadq_launch_count() - n0
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_ms = _max_over_ranks(world, sum(step_ms))

    # ---- end to end: the new query from pinned host memory, the output back ----
    h_q = torch.from_numpy(qbits.view(np.int16)).pin_memory()
    h_out = torch.empty(out.shape, dtype=torch.bfloat16, pin_memory=True)
    q_dev = torch.empty_like(q)

    def e2e_step():
        q_dev.view(torch.int16).copy_(h_q, non_blocking=True)
        step(q_dev, out, stream)
        h_out.copy_(out, non_blocking=True)

    for _ in range(2):
        flusher()
        e2e_step()
    torch.cuda.synchronize(dev)
    e_ms = 0.0
    for _ in range(args.e2e_steps):
        flusher()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms += a.elapsed_time(b)
    e_ms = _max_over_ranks(world, e_ms)

    if rank != 0:
        return None
    nbytes = dw.attn_bytes()
    value = aggregate_gbs(world, nbytes, steps, total_ms)
    avg_ms = sum(step_ms) / steps
    peak, peak_kind = measured_peaks()
    achieved = nbytes / (avg_ms * 1e-3) / 1e9
    out_line = {
        "metric": DECODE_METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(total_ms / steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": dw.name, "description": dw.description, "batch": dw.batch,
            "n_q_heads": dw.n_q_heads, "n_kv_heads": dw.n_kv_heads, "tokens": dw.tokens, "dim": dw.dim,
            "bytes_per_step": nbytes,
            "cache": "seeded INT4 codes binomial(14,1/2)-7, row scales uniform [0.25, 0.75]",
            "l2": "flushed between steps outside the timed events: 256 MiB written, then 256 MiB read",
            "parallelism": f"dp{world} (independent sequences, no collective)",
        },
        "roofline": {
            "bound": "hbm", "kernel": "kv_decode_attn_kernel", "achieved": round(achieved, 1),
            "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs (copy)", "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": recorded_traffic(dw.name, "attn"),
            "algorithmic_bytes_per_launch": nbytes, "avg_launch_ms": round(avg_ms, 5),
        },
        "e2e": {"value": round(world * nbytes * args.e2e_steps / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(q.numel() * 2), "d2h_bytes_per_step": int(out.numel() * 2),
                "steps": args.e2e_steps, "ms_per_step": round(e_ms / args.e2e_steps, 4),
                "note": "the KV cache is decode state resident in HBM; each step uploads the new query "
                        "and downloads the attention output"},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline:
        rate, info = decode_oracle_rate(dw, args.cpu_seconds)
        out_line["cpu_baseline"] = {
            "value": round(rate, 4), "unit": "GB/s", "cores": host_cores(), "blas_threads": cpu_threads(),
            "kind": "oracle",
            "sample": f"{info['q_heads']} query heads over {info['tokens']} cached tokens of one KV head "
                      f"through the float64 oracle in {info['seconds']} s"}
    return out_line


class TimedRuns:
    """CUDA-event durations of the launches of one workload step.

    ``flushed``: the L2 is flushed before every step (outside the events), so
    each launch starts cold and leaves its dirty lines behind.  Back to back
    (``flushed=False``) each launch also pays the write-back of the previous
    launch's outputs, the figure a long stream of such steps sustains.  The
    stream is held by a bounded device sleep while the host enqueues, so no
    event brackets host launch latency.
    """

    def __init__(self, st, stream, steps: int, flusher=None, clocks=None):
        import torch
        wl = st.wl
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3 if wl.dequant else 2)]
              for _ in range(steps)]
        done = torch.cuda.Event()
        torch.cuda.synchronize(stream.device)
        torch.cuda._sleep(hold_cycles(steps))
        for e in ev:
            if flusher is not None:
                flusher()
            e[0].record(stream)
            st.quantize(stream)
            e[1].record(stream)
            if wl.dequant:
                st.dequantize(stream)
                e[2].record(stream)
        done.record(stream)
        if clocks is not None:
            clocks.poll_until(done)
        torch.cuda.synchronize(stream.device)
        self.quant_ms = [e[0].elapsed_time(e[1]) for e in ev]
        self.dequant_ms = [e[1].elapsed_time(e[2]) for e in ev] if wl.dequant else []
        self.step_ms = [q + d for q, d in zip(self.quant_ms, self.dequant_ms or [0.0] * steps)]


def kernel_name(wl) -> str:
    from hadamard_rotation_outlier_b200 import binding as B
    if wl.kron_a:
        return KRON_KERNELS[B.hadq_kron_plan(0, wl.rows, wl.kron_a, wl.dim // wl.kron_a, wl.bits, wl.group)]
    if wl.asym:
        return "rq_chunk_asym_kernel"
    if wl.keep:  # the kept-token calls run KEEP instances: the tensor-core quantiser for 128-point
        # blocks with a scale per block, else the chunk kernel
        return "rq_chunk_mma_kernel" if wl.block == 128 and wl.group == 128 else "rq_chunk_kernel"
    return KERNEL_NAMES[B.hadq_plan(0, wl.rows, wl.dim, wl.block, wl.bits, wl.group, wl.with_signs, True)]


def dequant_kernel_name(wl) -> str:
    from hadamard_rotation_outlier_b200 import binding as B
    if wl.asym:
        return "dq_chunk_asym_kernel"
    if wl.keep:
        return "dq_chunk_kernel"
    path = B.hadq_plan(1, wl.rows, wl.dim, wl.block, wl.bits, wl.group, wl.with_signs, True)
    return {"chunk_mma": "dq_chunk_mma_kernel", "chunk": "dq_chunk_kernel", "blocked": "dq_blocked_kernel",
            "generic": "dq_generic_kernel"}.get(path, path)


def bandwidth(nbytes: int, ms: float, peak: float) -> dict:
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"avg_launch_ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
            "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4)}


def config_entry(wl, flushed: TimedRuns, sustained: TimedRuns, peak: float) -> dict:
    """One per_config entry: the quantise kernel (and the dequantiser) of a
    workload, flushed and back to back."""
    avg = lambda v: sum(v) / len(v)
    q_bytes = wl.quant_bytes()
    fam = workload_family(wl)
    e = {"workload": wl.name, "kernel": kernel_name(wl), "bytes": q_bytes,
         **bandwidth(q_bytes, avg(flushed.quant_ms), peak),
         "rows_per_s": round(wl.rows / (avg(flushed.quant_ms) * 1e-3), 1),
         "traffic": recorded_traffic(wl.name, fam),
         "sustained": bandwidth(q_bytes, avg(sustained.quant_ms), peak),
         "parity": recorded_parity(wl.name, fam)}
    if wl.dequant:
        d_bytes = wl.dequant_bytes(2)
        e["dequant"] = {"kernel": dequant_kernel_name(wl), "bytes": d_bytes,
                        **bandwidth(d_bytes, avg(flushed.dequant_ms), peak),
                        "sustained": bandwidth(d_bytes, avg(sustained.dequant_ms), peak)}
    return e


def run_ours(args):
    import torch
    from hadamard_rotation_outlier_b200 import binding as B
    from hadamard_rotation_outlier_b200 import synthetic as S
    from hadamard_rotation_outlier_b200.build import build
    from hadamard_rotation_outlier_b200.steps import WorkloadStep

    if args.workload not in S.WORKLOADS:
        raise SystemExit(f"unknown workload {args.workload}; choose from {list(S.WORKLOADS)}")
    world, rank, local = _dist_setup(args)
    if rank == 0:
        build()
    _barrier(world)
    B.load_library()
    wl = S.WORKLOADS[args.workload]
    warmup = max(3, args.warmup)
    steps = max(1, args.steps)
    dev = torch.device("cuda", local if world > 1 else 0)
    peak, peak_kind = measured_peaks()

    st = WorkloadStep(wl, dev, pinned_host=True)
    flusher = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(warmup):
        flusher()
        st.step(stream)
    torch.cuda.synchronize(dev)

    # ---- device-resident timed region ----
    clocks = ClockSampler(dev.index)
    _barrier(world)
    torch.cuda.synchronize(dev)
    n0 = B.hadq_launch_count()
    timed = TimedRuns(st, stream, steps, flusher, clocks)
    _barrier(world)
    launches = B.hadq_launch_count() - n0
    total_ms = _max_over_ranks(world, sum(timed.step_ms))

    # ---- the same launches back to back, no flush (sustained) ----
    sustained = TimedRuns(st, stream, min(steps, max(1, args.config_steps)))

    # ---- end to end through the public API with host buffers ----
    e2e = run_e2e(st, stream, args.e2e_steps, world)

    headline = config_entry(wl, timed, sustained, peak) if rank == 0 else None
    del st

    # ---- every configuration the target is stated on ----
    per_config = None
    if not args.no_per_config:
        per_config = []
        for name in PER_CONFIG:
            if name == wl.name:
                per_config.append(headline)
                continue
            cw = S.WORKLOADS[name]
            cs = WorkloadStep(cw, dev)
            for _ in range(3):
                flusher()
                cs.step(stream)
            n = max(1, args.config_steps)
            f = TimedRuns(cs, stream, n, flusher)
            b = TimedRuns(cs, stream, n)
            if rank == 0:
                per_config.append(config_entry(cw, f, b, peak))
            del cs
            torch.cuda.empty_cache()
        _barrier(world)

    if rank != 0:
        return None
    bytes_step = wl.quant_bytes() + (wl.dequant_bytes(2) if wl.dequant else 0)
    value = aggregate_gbs(world, bytes_step, steps, total_ms)
    q_ms = sum(timed.quant_ms) / steps
    achieved = wl.quant_bytes() / (q_ms * 1e-3) / 1e9
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": round(total_ms / steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": wl.name, "description": wl.description, "rows": wl.rows, "dim": wl.dim,
            "block": wl.block, "group": wl.group, "bits": wl.bits, "signs": wl.with_signs,
            "dequant_in_step": wl.dequant, "bytes_per_step": bytes_step,
            "rows_per_s": round(world * wl.rows * steps / (total_ms * 1e-3), 1),
            "l2": "flushed between steps outside the timed events: 256 MiB written, then 256 MiB read "
                  "so the flush's own dirty lines are written back before the step (L2 left clean)",
            "parallelism": f"dp{world} (independent rows, no collective)",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": headline["kernel"],
            "achieved": round(achieved, 1), "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs (copy)",
            "unit": "GB/s", "frac": round(achieved / peak, 4),
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "nominal_peak": NOMINAL_HBM_GBS,
            "traffic": headline["traffic"],
            "algorithmic_bytes_per_launch": wl.quant_bytes(), "avg_launch_ms": round(q_ms, 5),
        },
        "sustained": {**headline["sustained"],
                      "note": "the same launches back to back with no L2 flush: each pays the write-back "
                              "of the previous launch's dirty lines"},
        "parity": headline["parity"],
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    if wl.dequant:
        out["roofline"]["dequant_achieved"] = headline["dequant"]["gbs"]
    if per_config is not None:
        out["per_config"] = per_config
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    return out


def cpu_baseline(wl, target_s: float) -> dict:
    """The oracle on a bounded row sample, on every BLAS thread and on one."""
    r, info = oracle_sample_rate(wl, target_s)
    r1, info1 = single_thread(oracle_sample_rate, wl, max(1.0, target_s / 2))
    return {"value": round(r, 4), "unit": "GB/s", "cores": host_cores(), "blas_threads": cpu_threads(),
            "kind": "oracle",
            "sample": f"{info['passes']} pass(es) over {info['rows']} rows of {wl.name} "
                      f"through the float64 oracle in {info['seconds']} s",
            "single_thread": {"value": round(r1, 4), "unit": "GB/s",
                              "sample": f"{info1['passes']} pass(es) over {info1['rows']} rows in "
                                        f"{info1['seconds']} s, BLAS limited to one thread"}}


def run_e2e(st, stream, steps: int, world: int, nchunks: int = 8):
    """Same metric through the public API with host buffers.

    Every step copies the bf16 input from pinned host memory, runs the step's
    launches and copies every output (codes, scales and, for the KV-cache
    workload, the bf16 reconstruction) back to pinned host memory.  The batch
    is cut into row chunks alternating over two streams so that host-to-device
    copies, kernels and device-to-host copies overlap.
    """
    import torch
    wl = st.wl
    dev = st.x.device
    h_codes = torch.empty(st.codes.shape, dtype=st.codes.dtype, pin_memory=True)
    h_scales = torch.empty(st.scales.shape, dtype=torch.float32, pin_memory=True)
    h_out = torch.empty(st.out.shape, dtype=st.out.dtype, pin_memory=True) if wl.dequant else None
    h_kept = torch.empty(st.kept.shape, dtype=st.kept.dtype, pin_memory=True) if wl.keep else None
    h_zp = torch.empty(st.zero_points.shape, dtype=torch.uint8, pin_memory=True) if wl.asym else None
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    rows = st.rows
    per = -(-rows // nchunks)
    if wl.keep:  # kept-token calls take whole heads
        per = -(-wl.heads // nchunks) * wl.tokens
    from hadamard_rotation_outlier_b200 import binding as B

    def one_step():
        ev0 = torch.cuda.Event()
        ev0.record(stream)
        tails = []
        for c in range(nchunks):
            r0, r1 = c * per, min(rows, (c + 1) * per)
            if r0 >= r1:
                break
            s = streams[c % 2]
            s.wait_event(ev0)
            with torch.cuda.stream(s):
                st.x[r0:r1].copy_(st.x_host[r0:r1], non_blocking=True)
                if wl.keep:
                    h0, h1, t = r0 // wl.tokens, r1 // wl.tokens, wl.tokens
                    B.hadq_rotate_quantize_keep(st.x[r0:r1].view(h1 - h0, t, wl.dim), st.keep_slot, wl.n_keep,
                                                block=wl.block, signs=st.signs, bits=wl.bits, group=wl.group,
                                                codes=st.codes[r0:r1].view(h1 - h0, t, -1),
                                                scales=st.scales[r0:r1].view(h1 - h0, t, -1),
                                                kept=st.kept[h0:h1], stream=s)
                    B.hadq_dequant_rotate_inv_keep(st.codes[r0:r1].view(h1 - h0, t, -1),
                                                   st.scales[r0:r1].view(h1 - h0, t, -1), st.kept[h0:h1],
                                                   st.keep_slot, wl.n_keep, wl.dim, block=wl.block,
                                                   signs=st.signs, bits=wl.bits, group=wl.group,
                                                   out=st.out[r0:r1].view(h1 - h0, t, wl.dim), stream=s)
                    h_out[r0:r1].copy_(st.out[r0:r1], non_blocking=True)
                    h_kept[h0:h1].copy_(st.kept[h0:h1], non_blocking=True)
                elif wl.kron_a:
                    B.hadq_rotate_quantize_kron_pm1(st.x[r0:r1], st.sa, wl.dim // wl.kron_a, signs=st.signs,
                                                    bits=wl.bits, group=wl.group, codes=st.codes[r0:r1],
                                                    scales=st.scales[r0:r1], stream=s)
                elif wl.asym:
                    B.hadq_rotate_quantize_asym(st.x[r0:r1], block=wl.block, signs=st.signs, bits=wl.bits,
                                                group=wl.group, codes=st.codes[r0:r1], scales=st.scales[r0:r1],
                                                zero_points=st.zero_points[r0:r1], stream=s)
                    B.hadq_dequant_rotate_inv_asym(st.codes[r0:r1], st.scales[r0:r1], st.zero_points[r0:r1],
                                                   wl.dim, block=wl.block, signs=st.signs, bits=wl.bits,
                                                   group=wl.group, out=st.out[r0:r1], stream=s)
                    h_out[r0:r1].copy_(st.out[r0:r1], non_blocking=True)
                else:
                    B.hadq_rotate_quantize(st.x[r0:r1], block=wl.block, signs=st.signs, bits=wl.bits,
                                           group=wl.group, codes=st.codes[r0:r1], scales=st.scales[r0:r1],
                                           stream=s)
                    if wl.dequant:
                        B.hadq_dequant_rotate_inv(st.codes[r0:r1], st.scales[r0:r1], wl.dim, block=wl.block,
                                                  signs=st.signs, bits=wl.bits, group=wl.group,
                                                  out=st.out[r0:r1], stream=s)
                        h_out[r0:r1].copy_(st.out[r0:r1], non_blocking=True)
                h_codes[r0:r1].copy_(st.codes[r0:r1], non_blocking=True)
                h_scales[r0:r1].copy_(st.scales[r0:r1], non_blocking=True)
                if h_zp is not None:
                    h_zp[r0:r1].copy_(st.zero_points[r0:r1], non_blocking=True)
            e = torch.cuda.Event()
            e.record(s)
            tails.append(e)
        for e in tails:
            stream.wait_event(e)

    for _ in range(2):
        one_step()
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(steps):
        one_step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    _barrier(world)
    ms = _max_over_ranks(world, start.elapsed_time(end))
    h2d = st.x.numel() * 2
    d2h = h_codes.numel() * h_codes.element_size() + h_scales.numel() * 4
    if h_out is not None:
        d2h += h_out.numel() * 2
    if h_kept is not None:
        d2h += h_kept.numel() * 2
    if h_zp is not None:
        d2h += h_zp.numel()
    return {"value": round(world * st.bytes_per_step * steps / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4), "chunks": nchunks}


# ------------------------------------------------------------ reference arm

REFERENCE_BUDGET_S = 120.0


def reference_step_seconds(args) -> float:
    """CPU time of one reference-arm step: the whole run (warm-up and timed
    steps) stays near two minutes, each step between 0.3 s and half the
    baseline target."""
    n = max(1, args.steps) + max(0, args.warmup)
    return max(0.3, min(args.cpu_seconds / 2, REFERENCE_BUDGET_S / n))


def run_reference(args):
    """The CPU oracle as it stands, timed on this host's cores (rank 0 only).

    Exactly ``--steps`` timed steps after ``--warmup`` untimed ones; each step
    is one bounded row sample of the workload (see reference_step_seconds)."""
    from hadamard_rotation_outlier_b200 import synthetic as S
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return None
    if args.workload in S.DECODE_WORKLOADS:
        return run_reference_decode(args, S.DECODE_WORKLOADS[args.workload], world)
    wl = S.WORKLOADS[args.workload]
    steps = max(1, args.steps)
    target = reference_step_seconds(args)
    for _ in range(max(0, args.warmup)):
        oracle_sample_rate(wl, target)
    infos = [oracle_sample_rate(wl, target)[1] for _ in range(steps)]
    total_bytes = sum(i["bytes"] for i in infos)
    total_s = sum(i["seconds"] for i in infos)
    value = total_bytes / total_s / 1e9
    sample = (f"{steps} steps, each {infos[0]['passes']} pass(es) over {infos[0]['rows']} rows of {wl.name} "
              f"through the float64 oracle (numpy, dense matrix products), about {target:.1f} s of CPU each")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": round(total_s / steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "rows": wl.rows, "dim": wl.dim, "block": wl.block,
                   "group": wl.group, "bits": wl.bits, "signs": wl.with_signs},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": host_cores(),
                         "blas_threads": cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_reference_decode(args, dw, world):
    steps = max(1, args.steps)
    target = reference_step_seconds(args)
    for _ in range(max(0, args.warmup)):
        decode_oracle_rate(dw, target)
    infos = [decode_oracle_rate(dw, target)[1] for _ in range(steps)]
    total_bytes = sum(i["bytes"] for i in infos)
    total_s = sum(i["seconds"] for i in infos)
    value = total_bytes / total_s / 1e9
    sample = (f"{steps} steps, each {infos[0]['q_heads']} query heads over {infos[0]['tokens']} cached "
              f"tokens of one KV head through the float64 oracle")
    return {
        "impl": "reference", "metric": DECODE_METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": round(total_s / steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": dw.name, "batch": dw.batch, "n_q_heads": dw.n_q_heads,
                   "n_kv_heads": dw.n_kv_heads, "tokens": dw.tokens, "dim": dw.dim},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": host_cores(),
                         "blas_threads": cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        out = run_reference(args)
    else:
        from hadamard_rotation_outlier_b200 import synthetic as S
        out = run_decode(args) if args.workload in S.DECODE_WORKLOADS else run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)
    if args.impl == "ours" and int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
