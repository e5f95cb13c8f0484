"""Pins for the oracle's binary16 conversions (IEEE 754 binary16 definition).

Checked against things other than the oracle itself: numpy's float16 casts
(a library routine) over all 65536 bit patterns and over random binary64
values spanning subnormals to overflow, and hand-derived tie cases
(tests/golden/fp16_rounding.txt).
"""
import numpy as np
import pytest

import oracle
from golden_io import fp16_rounding


def _h2d_all():
    lib = oracle._load()
    return np.array([lib.orc_half_to_double(int(b)) for b in range(65536)])


def test_half_to_double_exhaustive_matches_numpy():
    ref = np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float64)
    got = _h2d_all()
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    # signed zeros keep their sign
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


def test_round_trip_every_non_nan_pattern():
    lib = oracle._load()
    vals = _h2d_all()
    for b in range(65536):
        if not np.isnan(vals[b]):
            assert lib.orc_double_to_half(float(vals[b])) == b, hex(b)


@pytest.mark.parametrize("lo_exp,hi_exp", [(-30, -14), (-14, 0), (0, 17), (-9, 5)])
def test_double_to_half_matches_numpy_rounding(lo_exp, hi_exp):
    rng = np.random.default_rng(1234 + lo_exp)
    n = 40000
    d = rng.choice([-1.0, 1.0], n) * np.exp2(rng.uniform(lo_exp, hi_exp, n))
    # also exact midpoints between adjacent binary16 values (the tie cases)
    h = rng.integers(0, 0x7BFF, n // 4).astype(np.uint16)
    a = h.view(np.float16).astype(np.float64)
    b = (h + 1).view(np.float16).astype(np.float64)
    d = np.concatenate([d, (a + b) / 2, -(a + b) / 2])
    lib = oracle._load()
    got = np.array([lib.orc_double_to_half(float(v)) for v in d], dtype=np.uint16)
    with np.errstate(over="ignore"):
        ref = d.astype(np.float16).view(np.uint16)
    assert (got == ref).all()


def test_hand_derived_rounding_cases():
    for v, bits in fp16_rounding():
        assert oracle.double_to_half(v) == bits, (v.hex(), hex(bits))


def test_special_values():
    assert oracle.double_to_half(float("inf")) == 0x7C00
    assert oracle.double_to_half(float("-inf")) == 0xFC00
    assert (oracle.double_to_half(float("nan")) & 0x7C00) == 0x7C00
    assert oracle.double_to_half(1e300) == 0x7C00
    assert oracle.double_to_half(1e-300) == 0x0000
