"""The comparison rules of tests/parity.py catch planted mistakes (CPU only)."""

import numpy as np
import pytest

import oracle as O
from hadamard_rotation_outlier_b200 import synthetic as S

from parity import check_asym


def _ref(bits=4, group=128):
    x = S.random_bf16(6, 256, 31, outlier_cols=[7], outlier_scale=20.0)
    return O.rotate_quantize_asym(x, block=128, bits=bits, group=group)


def test_asym_rule_accepts_the_oracle_itself():
    r = _ref()
    assert check_asym(r["q"], r["scales"], r["zero_points"], r, 4) == 0


def test_asym_rule_catches_a_shifted_code():
    r = _ref()
    q = r["q"].copy()
    q[2, 10] = (q[2, 10] + 2) % 16
    with pytest.raises(AssertionError):
        check_asym(q, r["scales"], r["zero_points"], r, 4)


def test_asym_rule_catches_a_wrong_zero_point():
    r = _ref(bits=8)
    zp = r["zero_points"].copy()
    zp[1, 0] += 1                                  # not at a .5 boundary
    with pytest.raises(AssertionError):
        check_asym(r["q"], r["scales"], zp, r, 8)


def test_asym_rule_catches_a_wrong_scale():
    r = _ref()
    s = r["scales"].copy()
    s[3, 1] *= 1.001
    with pytest.raises(AssertionError):
        check_asym(r["q"], s, r["zero_points"], r, 4)
