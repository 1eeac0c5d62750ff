"""OCP FP8 E4M3 ("fn" flavour) encoder and decoder, written from the format's definition.

Test infrastructure only: nothing in the product path imports this module.

Format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits. Exponent field 0 holds the
subnormals ``m / 8 * 2**-6``; fields 1..15 hold ``(1 + m / 8) * 2**(e - 7)``, except that the
pattern ``S.1111.111`` is NaN (there is no infinity). Largest finite magnitude: 448.

Encoding rule used for the projected-key scoring cache (JSSA summary, picx.dev, section 3.4
"Projected Scoring Cache": the cache is kept in FP8; the JSSA repository README, section 4 notes:
r bytes per token and KV head, so there is no room for a per-token scale): a direct cast with
round-to-nearest, ties to even, saturating to +-448 instead of overflowing.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_decode_table() -> np.ndarray:
    """Value of each of the 256 codes (float64; NaN for the two NaN codes)."""
    out = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            out[c] = np.nan
        elif e == 0:
            out[c] = s * (m / 8.0) * 2.0 ** -6
        else:
            out[c] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


_TABLE = e4m3_decode_table()


def e4m3_decode(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_round(y) -> np.ndarray:
    """Nearest E4M3 value (ties to even, saturating at +-448), as float64. NaN stays NaN."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    with np.errstate(divide="ignore", invalid="ignore"):
        _, e = np.frexp(a)               # a = f * 2**e with f in [0.5, 1)
    binade = np.maximum(e - 1, -6)       # a in [2**binade, 2**(binade+1)); subnormals share -6
    quantum = np.ldexp(1.0, binade - 3)  # spacing of representable values in that binade
    v = np.rint(a / quantum) * quantum   # exact scaling; rint rounds half to even
    v = np.minimum(v, E4M3_MAX)
    return np.where(np.isnan(y), np.nan, np.copysign(v, y))


def e4m3_encode(y) -> np.ndarray:
    """Codes (uint8) of ``e4m3_round(y)``. The sign bit follows the sign of ``y``, so values that
    round to zero from below give 0x80."""
    y = np.asarray(y, dtype=np.float64)
    v = np.abs(e4m3_round(y))
    nan = np.isnan(v)
    v = np.where(nan, 0.0, v)
    with np.errstate(divide="ignore"):
        f, e = np.frexp(v)               # v = f * 2**e
    expo = e - 1                         # v = (2f) * 2**expo with 2f in [1, 2)
    normal = v >= 2.0 ** -6
    field = np.where(normal, expo + 7, 0)
    mant = np.where(normal, (2.0 * f - 1.0) * 8.0, v / 2.0 ** -9)
    code = (field.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    code = np.where(nan, E4M3_NAN, code)
    code = code | np.where(np.signbit(y), 0x80, 0)
    return code.astype(np.uint8)
