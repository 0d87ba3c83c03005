"""Host check of the cubic 2^x used for part of the softmax exponentials
(exp2_poly in device_ptx.cuh): its coefficients are the ones the Remez
script produces, and the kernel's float32 steps, emulated bit for bit in
NumPy, stay within the stated relative error on the range the softmax uses
and give a finite non-negative value everywhere, -inf included."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_local_b200", "csrc")
sys.path.insert(0, CSRC)
import gen_exp2_poly  # noqa: E402


def _header_coefficients():
    src = open(os.path.join(CSRC, "device_ptx.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"0x([0-9a-f]{8})u", body)
    # Horner order in the source: c3, c2, c1, c0
    c3, c2, c1, c0 = (np.uint32(int(h, 16)).view(np.float32) for h in hexes)
    return [c0, c1, c2, c3]


def _emulate(x, c):
    f32 = np.float32
    x = np.maximum(np.asarray(x, dtype=f32), f32(-126.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    f = (x - (t - magic).astype(f32)).astype(f32)
    # fmaf rounds once: the float32 product is exact in float64
    p = (np.float64(c[3]) * f + np.float64(c[2])).astype(f32)
    p = (p.astype(np.float64) * f + np.float64(c[1])).astype(f32)
    p = (p.astype(np.float64) * f + np.float64(c[0])).astype(f32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(f32)


def test_header_holds_the_remez_coefficients():
    want = [np.float32(v) for v in gen_exp2_poly.coefficients()]
    got = _header_coefficients()
    assert [g.view(np.uint32) for g in got] == [w.view(np.uint32) for w in want]


def test_relative_error_on_the_softmax_range():
    c = _header_coefficients()
    x = np.linspace(-60.0, 9.0, 400001, dtype=np.float32)
    y = _emulate(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 8e-5
    # exact at integers up to the cubic's error at f = 0
    xi = np.arange(-60, 10, dtype=np.float32)
    assert np.all(np.abs(_emulate(xi, c) / np.exp2(xi.astype(np.float64)) - 1) < 8e-5)


def test_finite_and_non_negative_everywhere():
    c = _header_coefficients()
    x = np.concatenate([np.array([-np.inf, -1e30, -1000.0, -127.0, -126.5, -126.0, -125.5],
                                 dtype=np.float32),
                        np.linspace(-130, 10, 10001, dtype=np.float32)])
    y = _emulate(x, c)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    assert np.all(y[x <= -126] < 1e-37)
