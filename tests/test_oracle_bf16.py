"""Pins of the oracle's bf16 rounding (the scoring-cache ablation) to things other than itself:
torch's CPU float32 -> bfloat16 cast (one round-to-nearest-even rounding, exact reference for
float32 inputs), the format's closed forms, and float64 inputs just off a midpoint, where a
double rounding through float32 would go the wrong way."""

import numpy as np
import torch

from oracle.bf16 import BF16_MAX, bf16_decode, bf16_encode, bf16_round


def test_decode_all_patterns_against_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = bf16_decode(bits)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_random_float32_against_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-30, 30, 200000),
                        rng.standard_normal(1000) * 1e-39]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_encode(x.astype(np.float64)), ref)


def test_closed_forms():
    assert bf16_round(1.0) == 1.0
    assert bf16_round(1.0 + 2.0 ** -8) == 1.0                    # tie to even (down)
    assert bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6    # tie to even (up)
    assert bf16_round(BF16_MAX) == BF16_MAX
    assert np.isinf(bf16_round(BF16_MAX * (1 + 2.0 ** -8)))
    assert bf16_round(2.0 ** -133) == 2.0 ** -133                # smallest subnormal
    assert bf16_round(-3.0) == -3.0


def test_float64_just_off_a_midpoint():
    # 1 + 2^-8 is the midpoint between 1 and 1 + 2^-7: a hair above must round up, a hair
    # below down. Through float32 both hairs vanish and ties-to-even would give 1 for both.
    up = 1.0 + 2.0 ** -8 + 2.0 ** -40
    down = 1.0 + 2.0 ** -8 - 2.0 ** -40
    assert bf16_round(up) == 1.0 + 2.0 ** -7
    assert bf16_round(down) == 1.0
    assert bf16_encode(np.array([up]))[0] == 0x3F81


def test_bf16_scores_with_a_coordinate_basis():
    # a basis that selects coordinates leaves bf16 keys exactly representable, so the bf16
    # scoring cache holds the keys' own coordinates and the scores are plain dot products
    from oracle import jssa as O
    rng = np.random.default_rng(16)
    d, r = 32, 8
    k = torch.from_numpy(rng.standard_normal((50, d))).to(torch.bfloat16).double().numpy()
    dims = rng.choice(d, size=r, replace=False)
    m = np.zeros((r, d))
    m[np.arange(r), dims] = 1.0
    codes = O.store_codes_bf16(k, m)
    assert np.array_equal(bf16_decode(codes), k[:, dims])  # the cache holds the coordinates
    p = rng.standard_normal(r)
    want = np.array([sum(float(k[t, dims[j]]) * p[j] for j in range(r)) for t in range(k.shape[0])])
    assert np.allclose(O.scores_bf16(codes, p), want, rtol=1e-12, atol=1e-12)
