"""Oracle: OCP FP8 E4M3 ("e4m3fn") encode/decode and per-tile quantisation.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The FPSAttention page (Approach) quantises Q and K to FP8 at the same 3D
tile granularity as the sparsity. The pages do not give the format details,
so this module takes the plainest reading:

* format: OCP 8-bit E4M3 with no infinities: sign bit, 4 exponent bits with
  bias 7, 3 mantissa bits; exponent field 0 is subnormal
  (value = m/8 * 2^-6); S.1111.111 is NaN; the largest finite value is 448;
* encode: round to nearest, ties to even mantissa, saturating finite values
  (and infinities) beyond 448 to +-448; NaN -> 0x7F;
* one fp32 scale per (batch, head, tile) over all tile-volume x D values,
  padded slots (zeros) included: scale = fp32(amax) / 448 as an fp32
  division, amax = 0 -> scale = 1; code = encode(fp32(x / scale)) with the
  division rounded to nearest in fp32; dequantised value = scale * decode.

Parity: the decode table is pinned exhaustively against the format
definition written out independently in the test, encode against torch's
float8_e4m3fn cast (in range) and against round trips of every
representable value (tests/test_oracle_e4m3.py).
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def decode(code: int) -> float:
    """Value of one e4m3 code (0..255)."""
    s = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** (1 - 7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def decode_table() -> np.ndarray:
    return np.array([decode(c) for c in range(256)], dtype=np.float64)


_POS = np.array([decode(c) for c in range(0x7F)], dtype=np.float64)  # 0..448 ascending


def encode(x) -> np.ndarray:
    """fp32 array -> uint8 e4m3 codes, round-to-nearest-even, satfinite.

    Magnitudes are clamped to 448, then the nearest of the 127 non-negative
    finite values is taken; at an exact midpoint the code with the even
    mantissa (even code) wins. The sign bit is copied from the input, so
    negative values that round to zero give 0x80. NaN gives 0x7F.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    nan = np.isnan(x)
    sign = np.where(np.signbit(x), 0x80, 0x00)
    a = np.minimum(np.abs(np.where(nan, 0.0, x)), E4M3_MAX)
    hi = np.searchsorted(_POS, a, side="left")  # first table value >= a
    hi_c = np.minimum(hi, len(_POS) - 1)
    lo_c = np.maximum(hi - 1, 0)
    exact = _POS[hi_c] == a
    dlo = a - _POS[lo_c]
    dhi = _POS[hi_c] - a
    pick_lo = (dlo < dhi) | ((dlo == dhi) & (lo_c % 2 == 0))
    code = np.where(exact | (hi == 0), hi_c, np.where(pick_lo, lo_c, hi_c))
    out = (sign | code).astype(np.uint8)
    return np.where(nan, np.uint8(0x7F), out).astype(np.uint8)


def tile_scale(x_tile_f32: np.ndarray) -> np.float32:
    """fp32 scale of one tile: amax / 448 (amax = 0 -> 1)."""
    amax = np.float32(np.max(np.abs(x_tile_f32))) if x_tile_f32.size else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(E4M3_MAX))


def quantize_tiled(x_tiled: np.ndarray):
    """Tiled [B, heads, Nblk, vol, D] values (bf16-exact) -> (codes u8, scales f32)."""
    x = x_tiled.astype(np.float32)
    B, Hh, nb, vol, D = x.shape
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty((B, Hh, nb), dtype=np.float32)
    for b in range(B):
        for h in range(Hh):
            for t in range(nb):
                s = tile_scale(x[b, h, t])
                scales[b, h, t] = s
                q = (x[b, h, t] / s).astype(np.float32)  # IEEE fp32 division
                codes[b, h, t] = encode(q)
    return codes, scales


def dequantize_tiled(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """fp64 values scale * decode(code)."""
    tab = decode_table()
    return tab[codes] * scales.astype(np.float64)[..., None, None]
