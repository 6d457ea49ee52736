"""Host-side pieces of bench.py that need no GPU: the reference arm's JSON
line (it times the oracle on the host), the kernel-family source hashes and
the committed DRAM-traffic lookup."""

import json
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
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
    for fam, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (fam, f)
        assert len(bench.kernel_source_hash(fam)) == 16
    for wl in S.WORKLOADS.values():
        assert bench.workload_family(wl) in bench.KERNEL_SOURCES


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    # the committed figure is used while the family's sources hash the same
    wl = S.WORKLOADS["c2_qk_h32_s8192_d128_int8"]
    fam = bench.workload_family(wl)
    got = bench.recorded_traffic(wl.name, fam)
    assert got is None or got > 0
    # a line with another hash is ignored
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.txt").write_text(f"{wl.name} 0000000000000000 123\n"
                                           f"{wl.name} {bench.kernel_source_hash(fam)} 456\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda family: "abcdabcdabcdabcd")
    assert bench.recorded_traffic(wl.name, fam) is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda family: "0000000000000000")
    assert bench.recorded_traffic(wl.name, fam) == 123
