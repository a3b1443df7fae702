"""The softmax's FMA-pipe 2^x (ex2_poly2 in csrc/tc_common.cuh), emulated
step by step in float32 with the constants read from the source: its error
against exact 2^x must stay far below the bf16 rounding of P (2^-9)."""
import re
from pathlib import Path

import numpy as np

SRC = Path(__file__).resolve().parents[1] / "block_sparse_attention_reorder_b200" / "csrc" / "tc_common.cuh"


def _coeffs():
    body = SRC.read_text()
    body = body[body.index("ex2_poly2"):]
    m = re.search(r"c0 = ([0-9.eE+-]+)f, c1 = ([0-9.eE+-]+)f, c2 = ([0-9.eE+-]+)f, c3 = ([0-9.eE+-]+)f", body)
    assert m, "coefficients not found"
    return [np.float32(float(x)) for x in m.groups()]


def _fma32(a, b, c):
    # float32 fma: the float64 product of two float32 values is exact, one rounding after the add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _ex2_poly(x):
    c0, c1, c2, c3 = _coeffs()
    M = np.float32(12582912.0)
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + M).astype(np.float32)
    n = (t - M).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32),
                        np.float32([0.0, -0.0, 0.5, -0.5, 1.5, -2.5, 7.999, -124.99])])
    got = _ex2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 2e-4  # bf16 keeps 2^-9 = 2e-3


def test_monotone_and_clamped():
    x = np.linspace(-140.0, 8.0, 200_001, dtype=np.float32)
    y = _ex2_poly(x)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert np.all(y[x <= -125] == y[0])  # clamped: 2^-125 stands in for smaller values
    # relative steps stay within the polynomial error (no jumps at integer boundaries)
    r = y[1:].astype(np.float64) / y[:-1]
    step = np.exp2(np.diff(np.maximum(x, -125).astype(np.float64)))
    assert np.max(np.abs(r / step - 1)) < 4e-4
