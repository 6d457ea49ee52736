"""Host-side pieces of bench.py that need no GPU: the reference arm's JSON
line (it times the oracle on the host), the kernel-family source hashes and
the committed DRAM-traffic lookup."""

import json
import os
import re
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from hadamard_rotation_outlier_b200 import records as R  # noqa: E402
from hadamard_rotation_outlier_b200 import synthetic as S  # noqa: E402

REQUIRED = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "gpu_launches")


def _line(capsys, argv):
    bench.main(argv)
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1, out
    return json.loads(out[0])


@pytest.mark.parametrize("workload", ["c2_qk_h32_s8192_d128_int8", "d1_decode_q32_kv8_t131072_d128_int4"])
def test_reference_arm_line(capsys, workload):
    d = _line(capsys, ["--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "0",
                       "--cpu-seconds", "0.5"])
    for k in REQUIRED:
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == workload
    assert d["gpu_launches"] == 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] == d["cpu_baseline"]["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["sample"]


def test_every_workload_has_a_kernel_family_with_sources():
    csrc = os.path.join(bench.ROOT, "hadamard_rotation_outlier_b200", "csrc")
    for fam, files in R.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (fam, f)
        assert len(R.kernel_source_hash(fam)) == 16
    for wl in S.WORKLOADS.values():
        assert R.workload_family(wl) in R.KERNEL_SOURCES
    for dw in S.DECODE_WORKLOADS.values():
        assert R.workload_family(dw) == "attn"


def test_kernel_families_cover_every_included_header():
    # a record stays valid only while its kernels' sources are unchanged, so a
    # family must list every header its translation units include (directly
    # or through other headers); the declarations header holds no device code
    csrc = os.path.join(bench.ROOT, "hadamard_rotation_outlier_b200", "csrc")

    def included(name, seen):
        with open(os.path.join(csrc, name)) as f:
            for h in re.findall(r'#include "([^"]+)"', f.read()):
                if os.path.exists(os.path.join(csrc, h)) and h not in seen:
                    seen.add(h)
                    included(h, seen)
        return seen

    for fam, files in R.KERNEL_SOURCES.items():
        need = set()
        for f in files:
            if f.endswith(".cu"):
                need |= included(f, set())
        assert not need - set(files) - {"hadq_kernels.h"}, (fam, sorted(need - set(files)))


def test_records_follow_the_source_hash(tmp_path, monkeypatch):
    # a committed figure is used while the family's sources hash the same
    wl = S.WORKLOADS["c2_qk_h32_s8192_d128_int8"]
    fam = R.workload_family(wl)
    got = R.recorded_traffic(wl.name, fam)
    assert got is None or got > 0
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / R.TRAFFIC_FILE).write_text(f"# comment\n{wl.name} 0000000000000000 123\n"
                                       f"{wl.name} 1111111111111111 456\n")
    (prof / R.PARITY_FILE).write_text(
        f"{wl.name} 0000000000000000 mismatches=3 elements=1000000 far=0 scale_bad=0 "
        f"max_scale_rel=2.5e-07 when=2026-01-01T00:00Z\n")
    monkeypatch.setattr(R, "kernel_source_hash", lambda family, root=None: "abcdabcdabcdabcd")
    assert R.recorded_traffic(wl.name, fam, root=str(tmp_path)) is None
    assert R.recorded_parity(wl.name, fam, root=str(tmp_path)) is None
    monkeypatch.setattr(R, "kernel_source_hash", lambda family, root=None: "0000000000000000")
    assert R.recorded_traffic(wl.name, fam, root=str(tmp_path)) == 123
    p = R.recorded_parity(wl.name, fam, root=str(tmp_path))
    assert p["mismatches"] == 3 and p["elements"] == 1000000 and p["rate"] == 3e-6
    assert p["far"] == 0 and p["max_scale_rel"] == 2.5e-7 and p["when"] == "2026-01-01T00:00Z"


def test_parity_line_round_trips(tmp_path, monkeypatch):
    wl = S.WORKLOADS["c5_tok32768_w11008_b128_signs_int4_g128"]
    fam = R.workload_family(wl)
    line = R.parity_line(wl.name, fam, {"mismatches": 7, "elements": 360710144, "far": 0, "scale_bad": 0,
                                        "max_scale_rel": 3.1e-07}, "2026-12-02T10:00Z")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / R.PARITY_FILE).write_text(line + "\n")
    h = R.kernel_source_hash(fam)
    monkeypatch.setattr(R, "kernel_source_hash", lambda family, root=None: h)
    p = R.recorded_parity(wl.name, fam, root=str(tmp_path))
    assert p["mismatches"] == 7 and p["elements"] == 360710144 and p["max_scale_rel"] == 3.1e-07


class _Runs:
    def __init__(self, q, d=()):
        self.quant_ms, self.dequant_ms = list(q), list(d)


def test_per_config_entry_fractions():
    wl = S.WORKLOADS["c4_kv_h8_t131072_d128_int4_g128"]
    e = bench.config_entry(wl, _Runs([0.1, 0.1], [0.2, 0.2]), _Runs([0.125], [0.25]), 6543.4)
    q = wl.quant_bytes()
    assert e["workload"] == wl.name and e["bytes"] == q
    assert e["gbs"] == round(q / 1e-4 / 1e9, 1)
    assert e["frac"] == round(q / 1e-4 / 1e9 / 6543.4, 4)
    assert e["frac_of_nominal"] == round(q / 1e-4 / 1e9 / bench.NOMINAL_HBM_GBS, 4)
    assert e["sustained"]["avg_launch_ms"] == 0.125
    assert e["dequant"]["bytes"] == wl.dequant_bytes(2) and e["dequant"]["avg_launch_ms"] == 0.2
    assert e["kernel"].startswith("rq_") and e["dequant"]["kernel"].startswith("dq_")
    assert set(bench.PER_CONFIG) <= set(S.WORKLOADS) and bench.DEFAULT_WORKLOAD in bench.PER_CONFIG


def test_reference_arm_runs_the_requested_steps(capsys):
    d = _line(capsys, ["--impl", "reference", "--workload", "c1_tok256_h4096_b128_int4", "--steps", "4",
                       "--warmup", "1", "--cpu-seconds", "0.6"])
    assert d["steps"] == 4 and d["warmup"] == 1
    assert d["cpu_baseline"]["cores"] == bench.host_cores()
    args = bench.parse_args(["--steps", "20", "--warmup", "5"])
    assert 0.3 <= bench.reference_step_seconds(args) <= args.cpu_seconds / 2
    assert bench.reference_step_seconds(args) * 25 <= bench.REFERENCE_BUDGET_S + 1e-9
