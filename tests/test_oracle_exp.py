"""Pins for the routing exp (Cody-Waite reduction + degree-7 Taylor).

Checked against exp in double precision (an independent library routine),
against its own defining properties (exp(0) = 1, monotonicity), and against
hand-checked points in tests/golden/exp_points.txt.
"""
import math
import os
import struct

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32_from_bits(bits):
    return np.asarray(bits, dtype=np.uint32).view(np.float32)


def _ulp_error(f, exact):
    f = np.asarray(f, np.float64)
    e = np.asarray(exact, np.float64)
    expo = np.floor(np.log2(np.abs(e)))
    ulp = np.exp2(np.maximum(expo, -126) - 23)
    return np.abs(f - e) / ulp


def test_special_values(orc):
    assert orc.exp_portable(np.float32(0.0))[()] == np.float32(1.0)
    assert orc.exp_portable(np.float32(-0.0))[()] == np.float32(1.0)
    assert orc.exp_portable(np.float32(-np.inf))[()] == 0.0
    assert orc.exp_portable(np.float32(np.nan))[()] == 0.0
    assert orc.exp_portable(np.float32(-87.5))[()] == 0.0
    v = orc.exp_portable(np.float32(-87.0))[()]
    assert v >= np.finfo(np.float32).tiny  # still a normal float


def test_ulp_sweep_whole_domain(orc):
    # every 127th float in [-87, -0]: ~8.8M points spread over the domain
    top = struct.unpack("<I", struct.pack("<f", 87.0))[0]
    mags = np.arange(0, top + 1, 127, dtype=np.uint32)
    x = _f32_from_bits(mags | np.uint32(0x80000000))
    f = orc.exp_portable(x)
    err = _ulp_error(f, np.exp(x.astype(np.float64)))
    assert err.max() <= 2.0, f"max ulp error {err.max()} at x={x[err.argmax()]}"


def test_ulp_dense_windows(orc):
    # consecutive floats around the reduction boundaries (r near +-ln2/2) and near -87
    for c in [-0.3466, -1.0397, -10.0, -43.6, -86.99, -1e-6]:
        b = struct.unpack("<I", struct.pack("<f", abs(c)))[0]
        x = _f32_from_bits(np.arange(b - 20000, b + 20000, dtype=np.uint32) | np.uint32(0x80000000))
        x = x[x >= -87.0]
        f = orc.exp_portable(x)
        assert _ulp_error(f, np.exp(x.astype(np.float64))).max() <= 2.0


def test_monotone(orc):
    # walking down consecutive floats, exp never increases
    for start in [0, 0x3E000000, 0x3F300000, 0x40A00000, 0x42AD0000]:
        f = orc.exp_portable_neg_bits(start, 200000)
        assert np.all(np.diff(f.astype(np.float64)) <= 0.0)


def test_golden_points(orc):
    # x, then e^x to 9 significant digits: worked by hand from e = 2.718281828...
    with open(os.path.join(GOLDEN, "exp_points.txt")) as fh:
        rows = [l.split() for l in fh if l.strip() and not l.startswith("#")]
    for xs, ys in rows:
        x, y = np.float32(float(xs)), float(ys)
        f = float(orc.exp_portable(x))
        assert abs(f - y) <= 2.5e-7 * y, (xs, f, y)
