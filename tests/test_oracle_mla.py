"""Pins of the oracle's multi-head latent attention pieces to things other than themselves:
the scoring row of the block basis against separately computed latent projection and rotary
part, and the latent attention (576-dim keys, their first 512 dims as values, 16 heads sharing
one latent head) against torch's CPU scaled_dot_product_attention in float64."""

import numpy as np
import torch

from oracle import jssa as O


def test_mla_scoring_row_is_projected_latent_then_rope():
    rng = np.random.default_rng(11)
    m_lat = rng.standard_normal((64, 512))
    c = rng.standard_normal(512)
    kr = rng.standard_normal(64)
    row = O.mla_scoring_basis(m_lat) @ np.concatenate([c, kr])
    assert np.allclose(row[:64], np.einsum("rd,d->r", m_lat, c), rtol=0, atol=1e-12)
    assert np.array_equal(row[64:], kr)


def test_mla_latent_attention_against_torch_sdpa():
    rng = np.random.default_rng(12)
    L, heads, ps = 300, 16, 64
    kv = rng.standard_normal((L, 576))
    q = rng.standard_normal((1, heads, 576))
    pages = -(-L // ps)
    cache = np.zeros((pages, ps, 1, 576))
    cache.reshape(-1, 576)[:L] = kv
    bt = np.arange(pages)[None]
    idx = np.arange(L, dtype=np.int32)[None, None]
    count = np.array([[L]], dtype=np.int32)
    scale = 1.0 / np.sqrt(576.0)
    got = O.indexed_attend_step(q, cache, cache[..., :512], bt, idx, count, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[0])[:, None], torch.from_numpy(kv)[None].expand(heads, L, 576),
        torch.from_numpy(kv[:, :512])[None].expand(heads, L, 512), scale=scale)
    assert np.allclose(got[0], ref[:, 0].numpy(), rtol=1e-12, atol=1e-12)
