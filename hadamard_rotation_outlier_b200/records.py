"""Committed measurement records and the kernel sources they are valid for.

Some figures in a benchmark line come from runs other than the timed one:
the DRAM bytes of the timed kernel (one ncu capture) and the number of code
mismatches over every element of a workload (the full-size parity test).  Each
is stored in a text file under ``profiles/`` as lines

    workload  source_hash  value...

where ``source_hash`` hashes the device sources of the kernel family that
produced it.  A record is used only while those sources still hash the same,
so a kernel change retires its old figures by itself.

This module only reads files and hashes them; it holds none of the method's
arithmetic.
"""

from __future__ import annotations

import hashlib
import os

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)

# Device sources each kernel family is built from.
KERNEL_SOURCES = {
    "quant": ["hadq_common.cuh", "hadq_chunk.cuh", "hadq_blocked.cuh", "hadq_full4096.cuh",
              "hadq_generic.cuh", "hadq_mma.cuh", "hadq_chunk_mma.cuh", "k_blocked.cu", "k_chunk.cu",
              "k_chunk_dq4.cu", "k_chunk_dq8.cu", "k_chunk_mma.cu", "k_full4096.cu", "k_generic.cu",
              "hadq_dq_mma.cuh", "k_dq_mma.cu"],
    "attn": ["hadq_common.cuh", "hadq_attn.cuh", "k_attn.cu"],
    "keep": ["hadq_common.cuh", "hadq_chunk.cuh", "hadq_mma.cuh", "hadq_chunk_mma.cuh", "k_keep_rq.cu",
             "k_keep_dq.cu"],
    "asym": ["hadq_common.cuh", "hadq_chunk.cuh", "hadq_asym.cuh", "k_asym.cu"],
    "kron": ["hadq_common.cuh", "hadq_generic.cuh", "hadq_mma.cuh", "hadq_kron.cuh", "k_kron.cu"],
    "h4096": ["hadq_common.cuh", "hadq_chunk.cuh", "hadq_mma.cuh", "hadq_h4096.cuh", "k_h4096.cu"],
    "h4096tc": ["hadq_common.cuh", "hadq_tc.cuh", "hadq_h4096_tc.cuh", "k_h4096_tc.cu"],
}

TRAFFIC_FILE = "dram_traffic.txt"
PARITY_FILE = "parity_counts.txt"


def workload_family(wl) -> str:
    """Kernel family whose sources a workload's timed kernels are built from."""
    from . import binding as B
    if getattr(wl, "kron_a", 0):
        return "kron"
    if getattr(wl, "asym", False):
        return "asym"
    if getattr(wl, "keep", None):
        return "keep"
    if not hasattr(wl, "block"):
        return "attn"
    path = B.hadq_plan(0, wl.rows, wl.dim, wl.block, wl.bits, wl.group, wl.with_signs, True)
    if path == "wide4096_mma":
        return "h4096"
    if path == "h4096_tc":
        return "h4096tc"
    return "quant"


def kernel_source_hash(family: str, root: str | None = None) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(root or ROOT, "hadamard_rotation_outlier_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[family]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def read_record(filename: str, workload: str, source_hash: str, root: str | None = None):
    """Fields after the hash of the last line ``workload source_hash ...`` of
    ``profiles/<filename>``, or None when no line matches."""
    path = os.path.join(root or ROOT, "profiles", filename)
    try:
        with open(path) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    found = None
    for ln in lines:
        if not ln.strip() or ln.lstrip().startswith("#"):
            continue
        parts = ln.split()
        if len(parts) >= 3 and parts[0] == workload and parts[1] == source_hash:
            found = parts[2:]
    return found


def recorded_traffic(workload: str, family: str, root: str | None = None):
    """DRAM bytes per launch of the workload's timed quantise kernel, or None."""
    f = read_record(TRAFFIC_FILE, workload, kernel_source_hash(family, root), root)
    return int(f[0]) if f else None


def recorded_parity(workload: str, family: str, root: str | None = None):
    """Code mismatches over every element of the workload, from the full-size
    parity test, as a dict, or None when there is no record for the current
    kernel sources."""
    f = read_record(PARITY_FILE, workload, kernel_source_hash(family, root), root)
    if not f:
        return None
    kv = dict(item.split("=", 1) for item in f if "=" in item)
    out = {"mismatches": int(kv["mismatches"]), "elements": int(kv["elements"])}
    out["rate"] = out["mismatches"] / out["elements"]
    for k in ("far", "scale_bad", "max_scale_rel", "bf16_bad", "when"):
        if k in kv:
            out[k] = kv[k] if k == "when" else float(kv[k]) if "." in kv[k] or "e" in kv[k] else int(kv[k])
    return out


def parity_line(workload: str, family: str, counts: dict, when: str) -> str:
    """One record line of ``profiles/parity_counts.txt``."""
    items = " ".join(f"{k}={counts[k]}" for k in ("mismatches", "elements", "far", "scale_bad",
                                                   "max_scale_rel", "bf16_bad") if k in counts)
    return f"{workload} {kernel_source_hash(family)} {items} when={when}"
