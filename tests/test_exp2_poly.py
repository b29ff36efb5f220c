"""The attention kernels' 2^x on the FMA pipe (exp2_fma in sm100.cuh):
Cody-Waite range reduction x = n + f with n = round(x), 2^f on [-1/2, 1/2] by
a degree-3 polynomial with constant term 1, the exponent added as an integer.
The coefficients are read from the CUDA source and the same float32 steps are
replayed here, then checked against NumPy's exp2 (float64): the relative error
stays below the bound the coefficients were chosen for, far below the bf16
rounding of P (2^-9), and a masked key (x = -inf) gives exactly 0."""

import os
import re

import numpy as np
import pytest

from tests.conftest import ROOT

SRC = os.path.join(ROOT, "block_sparse_local_nb_b200", "csrc", "sm100.cuh")


def _coefficients():
    text = open(SRC).read()
    got = {}
    for name in ("kExp2C1", "kExp2C2", "kExp2C3"):
        m = re.search(name + r"\s*=\s*([0-9.eE+-]+)f", text)
        assert m, name
        got[name] = np.float32(float(m.group(1)))
    return got["kExp2C1"], got["kExp2C2"], got["kExp2C3"]


def _exp2_fma(x):
    """float32 replay of the kernel's steps."""
    c1, c2, c3 = _coefficients()
    x = np.minimum(np.maximum(np.asarray(x, np.float32), np.float32(-127)), np.float32(64))
    M = np.float32(12582912.0)
    t = (x + M).astype(np.float32)
    n = (t - M).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + np.float32(1)).astype(np.float32)
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_polynomial_relative_error_on_the_reduced_range():
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    got = _exp2_fma(f).astype(np.float64)
    want = np.exp2(f.astype(np.float64))
    assert np.max(np.abs(got - want) / want) < 1.1e-4


@pytest.mark.parametrize("lo,hi", [(-126.0, -100.0), (-30.0, 0.0), (0.0, 8.0), (8.0, 64.0)])
def test_range_reduction_keeps_the_relative_error(lo, hi):
    x = np.linspace(lo, hi, 100003, dtype=np.float32)
    got = _exp2_fma(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.all(got > 0)
    assert np.max(np.abs(got - want) / want) < 1.1e-4


def test_masked_and_clamped_inputs():
    assert _exp2_fma(np.array([-np.inf, -127.0, -500.0], np.float32)).tolist() == [0.0, 0.0, 0.0]
    # between -127 and -126.5 the result is a tiny non-negative denormal, never garbage
    tiny = _exp2_fma(np.linspace(-127.0, -126.0, 1001, dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)
    # the upper clamp: never above 2^64, so a chunk sum past 2^64 flags a recompute
    assert _exp2_fma(np.array([64.0, 100.0, np.inf], np.float32)).tolist() == [2.0 ** 64] * 3


def test_integer_values_are_exact_powers_of_two():
    n = np.arange(-126, 65, dtype=np.float32)
    assert np.array_equal(_exp2_fma(n).astype(np.float64), np.exp2(n.astype(np.float64)))
