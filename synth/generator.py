"""Seeded low-rank synthetic activations and paged KV caches.

Recipe (the workloads' stated generator): for each layer and KV head, keys are ``k = A_k z + mu``
and queries are ``q = A_q z'`` with ``z, z' ~ N(0, I)``. ``A_k = U_k diag(sigma) V_k^T`` and
``A_q = U_q diag(sigma) V_q^T`` with ``sigma_i = 1 / (1 + i / 8)``; ``U_k`` and ``U_q`` share their
first 48 columns (a seeded random orthonormal block) and are completed independently. ``mu = 2 u``
with ``u`` a seeded unit vector. Every query head draws its own ``z'``. Values are ``N(0, 1)``.
Everything is rounded to bf16 exactly once, when it is generated.

Pages: each sequence's logical pages are mapped to physical pages by a seeded random permutation
of the whole page pool, so consecutive logical pages are scattered in memory.

Nothing here computes a step of the sparse-attention method; the same tensors feed the CPU
oracle and the CUDA library.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes of one synthetic decode workload (one attention layer unless ``layers`` says more)."""

    name: str
    seed: int
    batch: int
    h_q: int
    h_kv: int
    d: int
    seq_len: int
    page_size: int
    rank: int
    budget: int
    calib_samples: int
    layers: int = 1
    window: int = -1

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def pages_per_seq(self) -> int:
        return -(-self.seq_len // self.page_size)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads named for this method's decode path. ``tiny`` is small enough for the oracle
# to finish in seconds; ``llama128k`` is the 128K-context layer the throughput metric is quoted on
# (batch and budget are swept around the defaults given here).
WORKLOADS = {
    "tiny": Workload("tiny", 1000, batch=1, h_q=8, h_kv=2, d=128, seq_len=2048, page_size=16,
                     rank=32, budget=128, calib_samples=4096),
    "llama32k": Workload("llama32k", 1001, batch=8, h_q=32, h_kv=8, d=128, seq_len=32768,
                         page_size=16, rank=32, budget=2048, calib_samples=32768),
    "llama128k": Workload("llama128k", 1002, batch=16, h_q=32, h_kv=8, d=128, seq_len=131072,
                          page_size=16, rank=32, budget=2048, calib_samples=32768),
    "hybrid": Workload("hybrid", 1003, batch=8, h_q=16, h_kv=8, d=256, seq_len=65536,
                       page_size=16, rank=64, budget=2048, calib_samples=32768, layers=6,
                       window=1024),
}

N_SHARED = 48


def _seed_state(*key: int) -> int:
    """A 63-bit seed derived from an integer key tuple (stable across runs and machines)."""
    ss = np.random.SeedSequence([int(k) & 0xFFFFFFFF for k in key])
    return int(ss.generate_state(2, dtype=np.uint32).astype(np.uint64).dot([1, 1 << 31])) & ((1 << 63) - 1)


def numpy_rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) & 0xFFFFFFFF for k in key]))


def torch_generator(device, *key: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed_state(*key))
    return g


def _random_orthonormal(rng: np.random.Generator, n: int, m: int) -> np.ndarray:
    q, r = np.linalg.qr(rng.standard_normal((n, m)))
    return q * np.sign(np.diag(r))[None, :]


def _complete(rng: np.random.Generator, shared: np.ndarray, d: int) -> np.ndarray:
    """Orthonormal d x d matrix whose first columns are exactly ``shared``."""
    k = shared.shape[1]
    q, _ = np.linalg.qr(np.hstack([shared, rng.standard_normal((d, d - k))]))
    q[:, :k] = shared
    # Re-orthogonalise the completion against the exact shared block (one Gram-Schmidt pass).
    rest = q[:, k:] - shared @ (shared.T @ q[:, k:])
    rest, _ = np.linalg.qr(rest)
    return np.hstack([shared, rest])


def singular_values(d: int) -> np.ndarray:
    return 1.0 / (1.0 + np.arange(d, dtype=np.float64) / 8.0)


def layer_factors(seed: int, layer: int, h_kv: int, d: int, n_shared: int = N_SHARED) -> dict:
    """Per-KV-head mixing matrices ``A_k``, ``A_q`` (fp64, ``[h_kv, d, d]``) and key mean ``mu``."""
    sigma = singular_values(d)
    a_k = np.empty((h_kv, d, d))
    a_q = np.empty((h_kv, d, d))
    mu = np.empty((h_kv, d))
    for h in range(h_kv):
        rng = numpy_rng(seed, layer, h, 1)
        shared = _random_orthonormal(rng, d, n_shared)
        u_k = _complete(rng, shared, d)
        u_q = _complete(rng, shared, d)
        v_k = _random_orthonormal(rng, d, d)
        v_q = _random_orthonormal(rng, d, d)
        a_k[h] = (u_k * sigma[None, :]) @ v_k.T
        a_q[h] = (u_q * sigma[None, :]) @ v_q.T
        u = rng.standard_normal(d)
        mu[h] = 2.0 * u / np.linalg.norm(u)
    return {"A_k": a_k, "A_q": a_q, "mu": mu}


def _mix(a: torch.Tensor, z: torch.Tensor) -> torch.Tensor:
    """``out[n, h, e] = sum_j a[h, e, j] z[n, h, j]`` (the generator's linear mixing)."""
    return torch.einsum("hej,nhj->nhe", a, z)


def _keys(factors: dict, n: int, gen: torch.Generator, device) -> torch.Tensor:
    a_k = torch.as_tensor(factors["A_k"], dtype=torch.float32, device=device)
    mu = torch.as_tensor(factors["mu"], dtype=torch.float32, device=device)
    h_kv, d = mu.shape
    z = torch.randn((n, h_kv, d), generator=gen, device=device, dtype=torch.float32)
    return (_mix(a_k, z) + mu[None]).to(torch.bfloat16).contiguous()


def _queries(factors: dict, n: int, group: int, gen: torch.Generator, device) -> torch.Tensor:
    a_q = torch.as_tensor(factors["A_q"], dtype=torch.float32, device=device)
    h_kv, d, _ = a_q.shape
    z = torch.randn((n, h_kv * group, d), generator=gen, device=device, dtype=torch.float32)
    a_rep = a_q.repeat_interleave(group, dim=0)  # query head i uses KV head i // group
    return _mix(a_rep, z).to(torch.bfloat16).contiguous()


def sample_calibration(factors: dict, n: int, group: int, seed: int, layer: int = 0,
                       device="cpu") -> tuple:
    """``n`` calibration samples: queries ``[n, h_kv*group, d]`` and keys ``[n, h_kv, d]`` (bf16)."""
    gk = torch_generator(device, seed, layer, 2)
    gq = torch_generator(device, seed, layer, 3)
    return _queries(factors, n, group, gq, device), _keys(factors, n, gk, device)


def sample_decode_queries(factors: dict, batch: int, group: int, seed: int, layer: int = 0,
                          step: int = 0, device="cpu") -> torch.Tensor:
    """One decode step's queries ``[batch, h_kv*group, d]`` (bf16)."""
    g = torch_generator(device, seed, layer, 4, step)
    return _queries(factors, batch, group, g, device)


def page_permutation(seed: int, layer: int, num_pages: int) -> np.ndarray:
    return numpy_rng(seed, layer, 5).permutation(num_pages).astype(np.int64)


def build_paged_kv(factors: dict, seq_lens: Sequence[int], page_size: int, seed: int,
                   layer: int = 0, device="cpu", extra_pages: int = 0,
                   chunk_pages: int = 2048, with_scoring_pages: bool = True) -> dict:
    """A paged bf16 KV cache holding one sequence per entry of ``seq_lens``.

    Layout: ``k_cache``/``v_cache`` are ``[num_pages, page_size, h_kv, d]``; ``block_table`` is
    ``int32 [batch, max_pages]`` (unused entries point at page 0 and are never read);
    ``seq_lens`` is ``int32 [batch]``. Logical page ``i`` of sequence ``b`` lives in physical
    page ``block_table[b, i]``. Every slot of every page holds seeded data (including slots past
    a sequence's end), so an over-read shows up as a wrong result rather than as zeros.
    """
    mu = factors["mu"]
    h_kv, d = mu.shape
    seq_lens = [int(x) for x in seq_lens]
    batch = len(seq_lens)
    npp = [max(1, -(-L // page_size)) for L in seq_lens]
    max_pages = max(npp)
    num_pages = sum(npp) + extra_pages
    perm = page_permutation(seed, layer, num_pages)
    bt = np.zeros((batch, max_pages), dtype=np.int32)
    start = 0
    for b in range(batch):
        bt[b, : npp[b]] = perm[start : start + npp[b]]
        start += npp[b]
    k_cache = torch.empty((num_pages, page_size, h_kv, d), dtype=torch.bfloat16, device=device)
    v_cache = torch.empty_like(k_cache)
    bt_dev = torch.as_tensor(bt, device=device, dtype=torch.int64)
    for b in range(batch):
        gk = torch_generator(device, seed, layer, 6, b)
        gv = torch_generator(device, seed, layer, 7, b)
        for p0 in range(0, npp[b], chunk_pages):
            p1 = min(npp[b], p0 + chunk_pages)
            n = (p1 - p0) * page_size
            pages = bt_dev[b, p0:p1]
            k_cache[pages] = _keys(factors, n, gk, device).view(p1 - p0, page_size, h_kv, d)
            v_cache[pages] = torch.randn((p1 - p0, page_size, h_kv, d), generator=gv,
                                         device=device, dtype=torch.float32).to(torch.bfloat16)
    if extra_pages:
        used = torch.as_tensor(perm[: sum(npp)], device=device)
        mask = torch.ones(num_pages, dtype=torch.bool, device=device)
        mask[used] = False
        spare = torch.nonzero(mask).flatten()
        g = torch_generator(device, seed, layer, 8)
        k_cache[spare] = torch.randn((len(spare), page_size, h_kv, d), generator=g, device=device).to(torch.bfloat16)
        v_cache[spare] = torch.randn((len(spare), page_size, h_kv, d), generator=g, device=device).to(torch.bfloat16)
    return {
        "k_cache": k_cache,
        "v_cache": v_cache,
        "block_table": torch.as_tensor(bt, device=device),
        "seq_lens": torch.as_tensor(np.asarray(seq_lens, dtype=np.int32), device=device),
        "num_pages": num_pages,
        "page_size": page_size,
    }


def logical_rows(cache: torch.Tensor, block_table: np.ndarray, b: int, positions: np.ndarray,
                 page_size: int) -> torch.Tensor:
    """Rows ``cache[block_table[b, t // page_size], t % page_size]`` for logical positions ``t``
    (plain indexing used by tests to read back what the generator placed)."""
    positions = np.asarray(positions, dtype=np.int64)
    pages = torch.as_tensor(block_table[b, positions // page_size].astype(np.int64), device=cache.device)
    slots = torch.as_tensor(positions % page_size, device=cache.device)
    return cache[pages, slots]
