"""Pins for the oracle's e4m3 encoder/decoder and per-tile quantiser (CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import e4m3


def test_decode_table_from_format_definition():
    """Every code against sign * 2^(e-bias) * (1.m), written with ldexp."""
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        v = e4m3.decode(c)
        if e == 15 and m == 7:
            assert math.isnan(v)
            continue
        mag = math.ldexp(m, -9) if e == 0 else math.ldexp(8 + m, e - 10)
        assert v == (-mag if s else mag), hex(c)
    assert e4m3.decode(0x7E) == 448.0 and e4m3.decode(0x38) == 1.0
    assert e4m3.decode(0x08) == 2.0 ** -6 and e4m3.decode(0x01) == 2.0 ** -9


def test_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(e4m3.decode_table(), ref)


def test_encode_round_trips_every_finite_value():
    tab = e4m3.decode_table()
    finite = [c for c in range(256) if not math.isnan(tab[c])]
    np.testing.assert_array_equal(e4m3.encode(tab[finite].astype(np.float32)),
                                  np.array(finite, dtype=np.uint8))


def test_encode_matches_torch_in_range_including_midpoints():
    tab = e4m3.decode_table()[:127]
    mids = ((tab[1:] + tab[:-1]) / 2).astype(np.float32)
    rng = np.random.default_rng(3)
    rand = (rng.standard_normal(20000) * rng.choice([1e-3, 0.1, 10, 100], 20000)).astype(np.float32)
    x = np.concatenate([mids, -mids, rand, np.nextafter(mids, np.float32(0)),
                        np.nextafter(mids, np.float32(1000))]).astype(np.float32)
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(e4m3.encode(x), ref)


def test_encode_saturates_and_nan():
    x = np.array([449.0, 464.0, 1e9, np.inf, -np.inf, -500.0, np.nan, -1e-30], dtype=np.float32)
    np.testing.assert_array_equal(e4m3.encode(x), [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F, 0x80])


def test_tile_quantiser_error_bound_and_zero_tile():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1, 2, 3, 64, 16)).astype(np.float32)
    x[0, 1, 2] = 0.0
    codes, scales = e4m3.quantize_tiled(x)
    assert scales[0, 1, 2] == 1.0 and np.all(codes[0, 1, 2] == 0)
    deq = e4m3.dequantize_tiled(codes, scales)
    for b, h, t in np.ndindex(1, 2, 3):
        s = float(scales[b, h, t])
        if not np.any(x[b, h, t]):
            continue
        assert s == np.float32(np.float32(np.abs(x[b, h, t]).max()) / np.float32(448))
        err = np.abs(deq[b, h, t] - x[b, h, t])
        # 3 mantissa bits: relative half-ulp 2^-4 for normals, 2^-10 * s absolute below 2^-6
        bound = np.maximum(np.abs(x[b, h, t]) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
        assert np.all(err <= bound)
        # the tile maximum maps to +-448 (code 0x7E / 0xFE)
        assert np.abs(deq[b, h, t]).max() == pytest.approx(448 * s, rel=1e-6)
