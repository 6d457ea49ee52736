import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """Print the full-size code-mismatch counts, when that test ran."""
    fp = sys.modules.get("full_parity")
    summary = getattr(fp, "SUMMARY", None)
    if not summary:
        return
    tr = terminalreporter
    tr.section("code mismatches over every element (limit 1e-5 of the elements)")
    for name, t in summary.items():
        line = (f"{name}: {t['mismatches']} mismatches / {t['elements']} elements = "
                f"{t['mismatches'] / t['elements']:.2e}; away from a boundary {t['far']}; "
                f"scales off {t['scale_bad']} (max rel {t['max_scale_rel']:.2e})")
        if "bf16_bad" in t:
            line += f"; bf16 reconstructions off {t['bf16_bad']}, exact {t['bf16_exact']}"
        tr.write_line(line)


def read_golden(name):
    """Parse a ``name = v1, v2, ...`` fixture file into {name: [floats]}."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split("=", 1)
            out[key.strip()] = [float(v) for v in val.split(",")]
    return out


@pytest.fixture(scope="session")
def golden_pages():
    return read_golden("pages_printed_values.txt")


@pytest.fixture(scope="session")
def golden_hand():
    return read_golden("hand_worked_examples.txt")
