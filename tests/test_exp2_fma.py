"""Host check of the FMA-pipe exp2 that the forward softmax uses for part of
its exponentials (`exp2_fma2` in block_sparse_local_b200/csrc/device_ptx.cuh).

The four cubic coefficients are read from the header and the routine is
emulated step by step in float32 / int32 arithmetic (shifter rounding,
cubic by Horner, exponent insertion by integer add, clamp at zero); the
result is compared with numpy's float64 exp2.  A wrong coefficient, a wrong
shifter or a wrong shift count fails the relative-error bound; the clamp
must turn x <= -127 and -inf into exactly +0.
"""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(__file__), "..", "block_sparse_local_b200", "csrc",
                      "device_ptx.cuh")


def _coeffs():
    text = open(HEADER).read()
    c = {}
    for k in range(4):
        m = re.search(rf"constexpr float kExp2C{k} = ([0-9.eE+-]+)f;", text)
        assert m, f"kExp2C{k} not found"
        c[k] = np.float32(float(m.group(1)))
    return c


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 inputs; one rounding to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_emulated(x):
    c = _coeffs()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    n = (t - shifter).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    p = _fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = _fma32(p, f, np.full_like(f, c[1]))
    p = _fma32(p, f, np.full_like(f, c[0]))
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    bits = ((bits + 2**31) % 2**32 - 2**31).astype(np.int32)   # int32 wrap-around
    bits = np.maximum(bits, 0)
    return bits.view(np.float32)


def test_relative_error_over_softmax_range():
    # arguments of the softmax: x = s * log2(e)/sqrt(d) - reference <= 8;
    # below -125.5 the result is subnormal and only its order of magnitude
    # holds (irrelevant next to a row maximum of 1)
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_fma_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()     # bf16 rounding of P is 2^-9 = 2.0e-3


def test_integers_and_halves():
    # x = n exactly and x = n + 1/2 (the ends of the reduced interval)
    n = np.arange(-126, 120, dtype=np.float32)
    for x in (n, n + np.float32(0.5), n - np.float32(0.5)):
        x = x[x >= -125]
        got = exp2_fma_emulated(x).astype(np.float64)
        ref = np.exp2(x.astype(np.float64))
        assert (np.abs(got - ref) / ref).max() < 1.0e-4


def test_masked_and_underflow_give_zero():
    x = np.array([-np.inf, -1e30, -1000.0, -200.0, -127.0], dtype=np.float32)
    got = exp2_fma_emulated(x)
    assert np.all(got == 0.0) and not np.any(np.signbit(got))


def test_never_negative_or_nan_below_range():
    x = np.linspace(-140.0, -120.0, 20001, dtype=np.float32)
    got = exp2_fma_emulated(x)
    assert np.all(np.isfinite(got)) and np.all(got >= 0.0)
    assert np.all(got <= np.exp2(-119.0))
