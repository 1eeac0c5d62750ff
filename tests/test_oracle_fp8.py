"""Pins of the oracle's E4M3 encoder/decoder against things other than itself.

* torch's CPU cast to ``float8_e4m3fn`` (a library special case): every bf16 bit pattern and a
  million random floats, wherever torch's cast is defined the same way (finite results; torch does
  not saturate, so values that round past 448 are compared with the saturation rule instead);
* the format's closed forms: largest finite 448, smallest subnormal 2**-9, round-trip of all
  representable values, ties to even at representable midpoints.
"""

import numpy as np
import pytest
import torch

from oracle.fp8 import E4M3_MAX, e4m3_decode, e4m3_decode_table, e4m3_encode, e4m3_round

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _torch_codes(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_table_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = e4m3_decode_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])


def test_closed_forms():
    t = e4m3_decode_table()
    finite = t[~np.isnan(t)]
    assert finite.max() == 448.0 and finite.min() == -448.0
    assert np.min(np.abs(finite[finite != 0])) == 2.0 ** -9
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    # round trip of every representable value (both zeros keep their sign bit)
    for c in range(256):
        if np.isnan(t[c]):
            continue
        assert e4m3_encode(np.copysign(t[c], -1.0 if c & 0x80 else 1.0)) == c


def test_ties_to_even_and_saturation():
    # midpoints between neighbours round to the even mantissa
    assert e4m3_encode(1.0 + 1 / 16) == 0x38          # 1.0625 -> 1.0 (mantissa 000)
    assert e4m3_encode(1.0 + 3 / 16) == 0x3A          # 1.1875 -> 1.25 (mantissa 010)
    assert e4m3_encode(2.0 ** -10) == 0x00            # half the smallest subnormal -> 0
    assert e4m3_encode(1.5 * 2.0 ** -9) == 0x02       # 1.5 ulp -> 2 ulp
    assert e4m3_encode(-(2.0 ** -11)) == 0x80         # rounds to zero from below: signed zero
    # saturation instead of overflow
    for v, c in [(448.0, 0x7E), (464.0, 0x7E), (479.99, 0x7E), (480.0, 0x7E), (1e30, 0x7E),
                 (-1e30, 0xFE), (-500.0, 0xFE)]:
        assert e4m3_encode(v) == c, v
    assert e4m3_encode(np.nan) & 0x7F == 0x7F


def _compare_with_torch(x: np.ndarray):
    ours = e4m3_encode(x)
    ref = _torch_codes(x)
    rounded = e4m3_round(x)
    in_range = np.isfinite(x) & (np.abs(x) < 464.0)   # torch and satfinite agree up to the 448/480 midpoint
    assert np.array_equal(ours[in_range], ref[in_range])
    big = np.isfinite(x) & (np.abs(x) >= 464.0)
    assert np.all(np.abs(rounded[big]) == E4M3_MAX)
    assert np.all((ours[big] & 0x7F) == 0x7E)


def test_all_bf16_patterns_against_torch():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    x = bits.view(np.float32).astype(np.float64)
    _compare_with_torch(x)


def test_random_floats_against_torch():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(400_000) * 4.0,
        rng.standard_normal(300_000) * 0.01,
        (rng.random(300_000) - 0.5) * 1000.0,
    ]).astype(np.float32).astype(np.float64)
    _compare_with_torch(x)


def test_decode_encode_consistency():
    rng = np.random.default_rng(8)
    x = rng.standard_normal(10_000) * 30
    assert np.array_equal(e4m3_decode(e4m3_encode(x)), e4m3_round(x))
