"""bfloat16 rounding, encoding and decoding, written from the format's definition.

Test infrastructure only: nothing in the product path imports this module.

The scoring-cache ablation keeps the projected keys as bf16(M k), two bytes per dimension,
instead of E4M3 (the pages keep them in FP8 for the byte count: JSSA README, section 4 notes;
JSSA summary, section 3.4). Format: 1 sign bit, 8 exponent bits with bias 127 (the float32
exponent), 7 mantissa bits: ``(1 + m / 128) * 2**(e - 127)`` for e in 1..254, subnormals
``m / 128 * 2**-126`` for e = 0, infinity and NaN at e = 255. Rounding from float64: nearest, ties
to even, overflowing to infinity.
"""

from __future__ import annotations

import numpy as np

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def bf16_round(y) -> np.ndarray:
    """Nearest bf16 value (ties to even) of float64 ``y``, as float64. NaN stays NaN."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        _, e = np.frexp(a)                 # a = f * 2**e with f in [0.5, 1)
        binade = np.maximum(e - 1, -126)   # a in [2**binade, 2**(binade+1)); subnormals share -126
        quantum = np.ldexp(1.0, binade - 7)
        v = np.rint(a / quantum) * quantum  # exact scaling; rint rounds half to even
        v = np.where(v > BF16_MAX, np.inf, v)
    return np.where(np.isnan(y), np.nan, np.copysign(v, y))


def bf16_encode(y) -> np.ndarray:
    """Bit patterns (uint16) of ``bf16_round(y)``: the high half of the float32 with that value."""
    v = bf16_round(y).astype(np.float32)  # exact: every bf16 value is a float32
    return (v.view(np.uint32) >> 16).astype(np.uint16)


def bf16_decode(bits) -> np.ndarray:
    """Value (float64) of each bf16 bit pattern."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):  # NaN patterns widen to NaN (numpy flags the cast)
        return b.view(np.float32).astype(np.float64)
