"""The e4m3 quantiser's division-free quotient, checked on the CPU.

The e4m3 code of a value x in a tile with scale s is defined (FPSAttention
page, Approach: per-tile e4m3 quantisation) by the IEEE fp32 quotient
fl(x / s). The kernels compute it without a division, by Markstein's FMA
correction: with y = fl(1 / s) correctly rounded,

    p = fl(x * y),   t = fl(p * s - x),   q = fl(p + t * (-y)),

the two last steps single-rounded FMAs (t is minus the residual x - p * s, and
this form keeps the sign of x = -0), and they take the plain division in
tiles whose scale is below 2^-92 or above 2^126. Here the three roundings are
redone exactly in numpy (products of two fp32 values are exact in fp64; the
last sum is rounded to fp32 from an exact two-term sum) and the codes from q
are compared with the oracle's codes from fl(x / s), for every bf16 x with
|x| <= amax, both signs and both zeros, across a few hundred tile amax values
(random ones, ones just above the 2^-92 bound, and the bf16 extremes).
"""
import numpy as np

from oracle import e4m3

GUARD_MIN, GUARD_MAX = 2.0 ** -92, 2.0 ** 126


def _rn32_of_sum(a, b):
    """float32 nearest (ties to even) to the exact a + b, for fp64 a, b."""
    hi = a + b
    bb = hi - a
    lo = (a - (hi - bb)) + (b - bb)  # Knuth's two-sum: hi + lo == a + b exactly
    r32 = hi.astype(np.float32)
    r = r32.astype(np.float64)
    up = np.nextafter(r32, np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(r32, np.float32(-np.inf)).astype(np.float64)
    # Only an hi exactly halfway between two fp32 values can round the wrong
    # way; the sign of lo then decides (lo == 0: the tie went to even already).
    out = r.copy()
    go_up = (hi == (r + up) / 2) & (lo > 0)
    go_dn = (hi == (r + dn) / 2) & (lo < 0)
    out[go_up] = up[go_up]
    out[go_dn] = dn[go_dn]
    return out


def _fma_quotient(x, scale, y):
    p = (x * y).astype(np.float32).astype(np.float64)
    t = (p * scale - x).astype(np.float32).astype(np.float64)
    return _rn32_of_sum(p, t * -y)


def _bf16_from_bits(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def test_two_sum_rounding_helper():
    # Halfway cases, and sums whose fp64 rounding lands on a halfway point
    # (2^-24 (1 + 2^-52) and 2^-24 (1 - 2^-53) are fp64 values; added to 1
    # they round to 1 + 2^-24 and leave the rest in lo).
    one = np.float64(1.0)
    half_ulp = 2.0 ** -24
    a = np.array([one, one, one, one + 2.0 ** -23])
    b = np.array([half_ulp, half_ulp * (1 + 2.0 ** -52), half_ulp * (1 - 2.0 ** -53), half_ulp])
    got = _rn32_of_sum(a, b)
    assert got[0] == 1.0                       # tie to even
    assert got[1] == 1.0 + 2.0 ** -23          # just above halfway
    assert got[2] == 1.0                       # just below halfway
    assert got[3] == 1.0 + 2.0 ** -22          # tie to even, upwards


def test_fma_quotient_codes_equal_division_codes():
    rng = np.random.default_rng(11)
    xs_pos = _bf16_from_bits(np.arange(0, 0x7F80)).astype(np.float64)  # +0, subnormals, normals
    guard_bits = int(np.float32(448.0 * GUARD_MIN).view(np.uint32) >> 16)
    amax_bits = np.concatenate([
        rng.integers(guard_bits, 0x7F80, 200),
        np.arange(guard_bits, guard_bits + 40),
        [0x3F80, 0x43E0, 0x3F00, 0x7F7F],  # 1, 448, 0.5, bf16 max
    ])
    checked = 0
    for amax in _bf16_from_bits(amax_bits).astype(np.float64):
        scale = np.float64(np.float32(amax / 448.0))  # fl(amax / 448): fp64 quotient rounded once more is exact
        y = np.float64(np.float32(1.0 / scale))       # correctly rounded reciprocal, same argument
        assert GUARD_MIN <= scale <= GUARD_MAX
        x = xs_pos[xs_pos <= amax]
        x = np.concatenate([x, -x])                   # -x of +0 is -0
        want = e4m3.encode((x / scale).astype(np.float32))
        got = e4m3.encode(_fma_quotient(x, scale, y).astype(np.float32))
        bad = np.flatnonzero(want != got)
        assert bad.size == 0, (amax, x[bad[:4]], want[bad[:4]], got[bad[:4]])
        checked += x.size
    assert checked > 5_000_000


def test_below_the_bound_the_correction_can_fail():
    """Why the kernels divide in tiles with a scale below 2^-92: there the
    residual can fall in the fp32 subnormal range and lose bits."""
    amax = np.float64(_bf16_from_bits([0x1170])[0])  # ~1.9e-28 -> scale ~2^-101
    scale = np.float64(np.float32(amax / 448.0))
    y = np.float64(np.float32(1.0 / scale))
    assert scale < GUARD_MIN
    xs = _bf16_from_bits(np.arange(0, 0x7F80)).astype(np.float64)
    x = xs[xs <= amax]
    want = (x / scale).astype(np.float32)
    got = _fma_quotient(x, scale, y).astype(np.float32)
    assert np.count_nonzero(want != got) > 0
