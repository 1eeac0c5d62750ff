"""Thin PyTorch binding of libjssa.so.

Argument marshalling only: every step of the method runs in the library's CUDA kernels. PyTorch
provides device memory (outputs and workspaces are allocated here with torch) and the current
CUDA stream. There is no CPU path: the functions raise if a tensor is not on a CUDA device or if
the library is missing.
"""

from __future__ import annotations

import ctypes
import math
from typing import Optional, Tuple

import torch

from . import _lib
from ._lib import (FN_COMPUTE_BASIS, FN_DECODE, FN_DECODE_HOST, FN_DENSE_DECODE,
                   FN_INDEXED_ATTEND, FN_MLA_ATTEND, FN_MLA_DECODE, FN_SCORE_TOPK, JSSAError, call,
                   check, load)

__all__ = [
    "gather_kv", "staged_pages", "gather_then_attend", "mla_calibrate_accumulate", "mla_attend",
    "mla_decode",
    "JSSAError", "workspace_size", "Workspace", "calibrate_accumulate", "compute_basis",
    "calibrate", "store", "score_topk", "indexed_attend", "dense_decode", "decode",
    "device_error", "kv_strides", "default_rank", "PagedLayer", "HostPipeline", "Calibration", "save_basis",
    "load_basis", "set_wait_limit",
]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, contiguous: bool = True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (there is no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def default_rank(head_dim: int) -> int:
    """Default subspace rank, head_dim // 4 (JSSA README, section 4: jssa_rank default)."""
    return head_dim // 4


def kv_strides(cache: torch.Tensor) -> Tuple[int, int, int]:
    """(page, slot, head) element strides of a ``[num_pages, page_size, h_kv, d]`` cache view."""
    if cache.dim() != 4 or cache.stride(3) != 1:
        raise ValueError("KV cache must be [num_pages, page_size, h_kv, d] with a contiguous last dim")
    return cache.stride(0), cache.stride(1), cache.stride(2)


def workspace_size(fn: int, batch: int, h_q: int, h_kv: int, d: int, max_pages: int,
                   page_size: int, budget: int) -> int:
    out = ctypes.c_size_t(0)
    call("jssa_workspace_size", fn, batch, h_q, h_kv, d, max_pages, page_size, budget,
         ctypes.byref(out))
    return int(out.value)


class Workspace:
    """A zero-initialised device workspace that grows on demand (one per stream of use)."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = None

    def get(self, nbytes: int) -> Tuple[Optional[int], int]:
        if nbytes == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            call("jssa_workspace_init", self.buf.data_ptr(), self.buf.numel(), _stream(self.device))
        return self.buf.data_ptr(), self.buf.numel()


_default_ws = {}


def _ws(device: torch.device, ws: Optional[Workspace], fn: int) -> Workspace:
    """The caller's workspace, else a default one per (device, stream, entry point): the split-K
    ticket counters of one entry point must not be overwritten by another's scratch."""
    if ws is not None:
        return ws
    key = (device.index, torch.cuda.current_stream(device).cuda_stream, fn)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


# ------------------------------------------------------------------------------------------------
# Calibration
# ------------------------------------------------------------------------------------------------


def calibrate_accumulate(q: torch.Tensor, k: torch.Tensor, gram_q: torch.Tensor,
                         gram_k: torch.Tensor) -> None:
    """Add the second moments of a batch of calibration samples into ``gram_q``/``gram_k``
    (float64 ``[h_kv, d, d]``). ``q``: bf16 ``[n, h_q, d]``; ``k``: bf16 ``[n, h_kv, d]``."""
    _need(q, "q", torch.bfloat16, contiguous=False)
    _need(k, "k", torch.bfloat16, contiguous=False)
    _need(gram_q, "gram_q", torch.float64)
    _need(gram_k, "gram_k", torch.float64)
    n, h_q, d = q.shape
    h_kv = k.shape[1]
    if q.stride(2) != 1 or q.stride(1) != d or k.stride(2) != 1 or k.stride(1) != d:
        raise ValueError("q and k rows must be [heads, d] contiguous")
    call("jssa_calibrate_accumulate", q.data_ptr(), q.stride(0), k.data_ptr(), k.stride(0), n, h_q,
         h_kv, d, gram_q.data_ptr(), gram_k.data_ptr(), _stream(q.device))


def mla_calibrate_accumulate(q: torch.Tensor, kv: torch.Tensor, gram_q: torch.Tensor,
                             gram_k: torch.Tensor) -> None:
    """Add the latent second moments of a batch of multi-head latent attention samples into
    ``gram_q``/``gram_k`` (float64 ``[1, 512, 512]``): the head mean of the absorbed queries'
    latent part (``q`` bf16 ``[n, h_q, 576]``) and the latent rows' latent part (``kv`` bf16
    ``[n, 576]`` or ``[n, 1, 576]``)."""
    _need(q, "q", torch.bfloat16, contiguous=False)
    _need(kv, "kv", torch.bfloat16, contiguous=False)
    _need(gram_q, "gram_q", torch.float64)
    _need(gram_k, "gram_k", torch.float64)
    n, h_q, dq = q.shape
    if dq < 512 or q.stride(2) != 1 or kv.stride(-1) != 1 or kv.shape[-1] < 512 or kv.shape[0] != n:
        raise ValueError("q must be [n, h_q, >= 512] and kv [n, (1,) >= 512] with contiguous rows")
    call("jssa_mla_calibrate_accumulate", q.data_ptr(), q.stride(0), q.stride(1), kv.data_ptr(),
         kv.stride(0), n, h_q, gram_q.data_ptr(), gram_k.data_ptr(), _stream(q.device))


def compute_basis(gram_q: torch.Tensor, gram_k: torch.Tensor, rank: int,
                  with_eigvals: bool = True):
    """``M = TopEig_r(G_Q/tr + G_K/tr)^T`` per KV head: float32 ``[h_kv, r, d]`` (and float64
    eigenvalues ``[h_kv, d]``, descending)."""
    _need(gram_q, "gram_q", torch.float64)
    _need(gram_k, "gram_k", torch.float64)
    h_kv, d, _ = gram_q.shape
    dev = gram_q.device
    basis = torch.empty((h_kv, rank, d), dtype=torch.float32, device=dev)
    eig = torch.empty((h_kv, d), dtype=torch.float64, device=dev) if with_eigvals else None
    nbytes = workspace_size(FN_COMPUTE_BASIS, 0, 1, h_kv, d, 0, 1, 0)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    call("jssa_compute_basis", gram_q.data_ptr(), gram_k.data_ptr(), h_kv, d, rank, basis.data_ptr(),
         _ptr(eig), ws.data_ptr(), nbytes, _stream(dev))
    return basis, eig


def calibrate(q: torch.Tensor, k: torch.Tensor, rank: int, batch: int = 8192):
    """Whole calibration over ``n`` samples, in batches of ``batch`` samples."""
    acc = Calibration(k.shape[1], q.shape[2], q.device)
    for s in range(0, q.shape[0], batch):
        acc.add(q[s:s + batch], k[s:s + batch])
    basis, eig = acc.basis(rank)
    return {"M": basis, "eigvals": eig, "gram_q": acc.gram_q, "gram_k": acc.gram_k}


class Calibration:
    """Running second moments of one layer (float64 ``[h_kv, d, d]`` on the device) and the
    number of samples they hold; ``add`` accumulates a batch, ``basis`` solves for ``M``, and
    ``state``/``from_state`` carry the moments across processes so that a calibration can stop
    and resume (JSSA README, section 2: second moments from calibration sequences, optionally
    saved with the basis)."""

    def __init__(self, h_kv: int, d: int, device=None, gram_q=None, gram_k=None, samples: int = 0):
        dev = torch.device(device or "cuda")
        self.gram_q = (torch.zeros((h_kv, d, d), dtype=torch.float64, device=dev) if gram_q is None
                       else gram_q.to(dev, torch.float64).contiguous())
        self.gram_k = (torch.zeros_like(self.gram_q) if gram_k is None
                       else gram_k.to(dev, torch.float64).contiguous())
        if self.gram_q.shape != (h_kv, d, d) or self.gram_k.shape != (h_kv, d, d):
            raise ValueError("second moments must be [h_kv, d, d]")
        self.samples = int(samples)

    def add(self, q: torch.Tensor, k: torch.Tensor) -> None:
        calibrate_accumulate(q, k, self.gram_q, self.gram_k)
        self.samples += int(q.shape[0])

    def add_latent(self, q: torch.Tensor, kv: torch.Tensor) -> None:
        """A multi-head latent layer's samples (``Calibration(1, 512)``): absorbed queries
        ``[n, h_q, 576]`` and latent rows ``[n, 576]``."""
        mla_calibrate_accumulate(q, kv, self.gram_q, self.gram_k)
        self.samples += int(q.shape[0])

    def basis(self, rank: int, with_eigvals: bool = True):
        return compute_basis(self.gram_q, self.gram_k, rank, with_eigvals)

    def all_reduce(self, group=None) -> None:
        """Sum the moments and the sample counts over the ranks of ``group`` (the default process
        group when None): one all-reduce of ``2 h_kv d^2 + 1`` float64 values (NCCL over NVLink
        between GPUs). The moments are sums over samples, so ranks that each calibrate on their
        own sequences then all hold the moments of every rank's samples, bit-identical, and
        ``basis`` solves for the same M on every rank (JSSA README, section 2: the latent
        calibration runs across the GPUs of a tensor-parallel group; JSSA summary, section 3.2:
        calibration is second-moment accumulation)."""
        import torch.distributed as dist
        n = self.gram_q.numel()
        flat = torch.empty(2 * n + 1, dtype=torch.float64, device=self.gram_q.device)
        flat[:n] = self.gram_q.reshape(-1)
        flat[n:2 * n] = self.gram_k.reshape(-1)
        flat[2 * n] = float(self.samples)
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
        self.gram_q.copy_(flat[:n].view_as(self.gram_q))
        self.gram_k.copy_(flat[n:2 * n].view_as(self.gram_k))
        self.samples = int(round(float(flat[2 * n].item())))

    def state(self) -> dict:
        """Host copies of the moments and the sample count."""
        return {"gram_q": self.gram_q.cpu(), "gram_k": self.gram_k.cpu(), "samples": self.samples}

    @classmethod
    def from_state(cls, state: dict, device=None) -> "Calibration":
        gq = state["gram_q"]
        return cls(gq.shape[0], gq.shape[1], device, gq, state["gram_k"], state.get("samples", 0))


def save_basis(path: str, bases: dict, calibrations: Optional[dict] = None,
               eigvals: Optional[dict] = None, rank: Optional[int] = None) -> None:
    """Write a basis file: ``{'M': {layer: Tensor[h_kv, r, d]}}`` (the layout the pages' runtime
    reads; a latent layer's basis is ``[1, r, kv_lora_rank]``), plus, when given, each layer's
    second moments under ``'grams'`` (``{layer: {'gram_q', 'gram_k', 'samples'}}``, so that the
    calibration can resume) and eigenvalues under ``'eigvals'``. JSSA README, section 2 (the
    output file; ``--save_grams``)."""
    out = {"M": {int(layer): m.detach().to("cpu", torch.float32).contiguous()
                 for layer, m in bases.items()}}
    for layer, m in out["M"].items():
        if m.dim() != 3:
            raise ValueError(f"basis of layer {layer} must be [h_kv, r, d]")
        if rank is not None and m.shape[1] != rank:
            raise ValueError(f"basis of layer {layer} has rank {m.shape[1]}, not {rank}")
    if calibrations:
        out["grams"] = {int(layer): (c.state() if isinstance(c, Calibration) else
                                     {"gram_q": c["gram_q"].detach().cpu(),
                                      "gram_k": c["gram_k"].detach().cpu(),
                                      "samples": int(c.get("samples", 0))})
                        for layer, c in calibrations.items()}
    if eigvals:
        out["eigvals"] = {int(layer): e.detach().to("cpu", torch.float64) for layer, e in eigvals.items()}
    torch.save(out, path)


def load_basis(path: str, device=None, rank: Optional[int] = None) -> dict:
    """Read a basis file written by :func:`save_basis` (or any file with the same ``'M'``
    layout). Returns ``{'M': {layer: float32 Tensor}}`` on ``device`` and, when the file has
    them, ``'grams'`` as :class:`Calibration` objects (resume with ``add``) and ``'eigvals'``.
    A ``rank`` that differs from a stored basis's raises (the runtime's rank must match the
    basis: JSSA README, section 4, ``jssa_rank``)."""
    raw = torch.load(path, map_location="cpu", weights_only=True)
    if "M" not in raw:
        raise ValueError(f"{path}: not a basis file (no 'M')")
    dev = torch.device(device) if device is not None else None
    res = {"M": {}}
    for layer, m in raw["M"].items():
        if m.dim() != 3:
            raise ValueError(f"{path}: basis of layer {layer} is not [h_kv, r, d]")
        if rank is not None and m.shape[1] != rank:
            raise ValueError(f"{path}: basis of layer {layer} has rank {m.shape[1]}, not {rank}")
        m = m.to(torch.float32).contiguous()
        res["M"][int(layer)] = m.to(dev) if dev is not None else m
    if "grams" in raw:
        res["grams"] = {int(layer): Calibration.from_state(st, dev or "cpu") for layer, st in raw["grams"].items()}
    if "eigvals" in raw:
        res["eigvals"] = {int(layer): (e.to(dev) if dev is not None else e) for layer, e in raw["eigvals"].items()}
    return res


# ------------------------------------------------------------------------------------------------
# Decode
# ------------------------------------------------------------------------------------------------


def store(k: torch.Tensor, slot_mapping: torch.Tensor, basis: torch.Tensor,
          score_cache: torch.Tensor) -> None:
    """Write ``e4m3(M_h k)`` of each token ``k[t]`` (bf16 ``[t, h_kv, d]``) at flat slot
    ``slot_mapping[t]`` (int64; negative = skip) of the scoring cache
    (uint8 ``[num_pages, h_kv, page_size, r]``; a bfloat16 cache of that shape holds
    ``bf16(M_h k)`` instead, the scoring-cache ablation). A latent layer (``d`` 576, basis
    ``[1, r, 512]``) has ``r + 64`` code columns (the rotary dimensions pass through)."""
    _need(k, "k", torch.bfloat16, contiguous=False)
    _need(slot_mapping, "slot_mapping", torch.int64)
    _need(basis, "basis", torch.float32)
    bf16 = score_cache.dtype == torch.bfloat16
    _need(score_cache, "score_cache", torch.bfloat16 if bf16 else torch.uint8)
    t, h_kv, d = k.shape
    num_pages, _, page_size, cols = score_cache.shape
    r = basis.shape[1]
    if cols != (r + 64 if d == 576 else r):
        raise ValueError(f"scoring cache has {cols} code columns; rank {r} at d {d} needs "
                         f"{r + 64 if d == 576 else r}")
    if k.stride(2) != 1 or k.stride(1) != d:
        raise ValueError("k rows must be [h_kv, d] contiguous")
    call("jssa_store_bf16" if bf16 else "jssa_store", k.data_ptr(), k.stride(0),
         slot_mapping.data_ptr(), t, h_kv, d, r, basis.data_ptr(), score_cache.data_ptr(),
         num_pages, page_size, _stream(k.device))


def score_topk(q: torch.Tensor, basis: torch.Tensor, score_cache: torch.Tensor,
               block_table: torch.Tensor, seq_lens: torch.Tensor, budget: int,
               idx: Optional[torch.Tensor] = None, count: Optional[torch.Tensor] = None,
               ws: Optional[Workspace] = None):
    """Index sets ``idx`` (int32 ``[batch, h_kv, budget]``, ascending, -1 padded) and ``count``.
    A bfloat16 ``score_cache`` selects the bf16 scoring-cache ablation."""
    bf16 = score_cache.dtype == torch.bfloat16
    for t, n, dt in ((q, "q", torch.bfloat16), (basis, "basis", torch.float32),
                     (score_cache, "score_cache", torch.bfloat16 if bf16 else torch.uint8),
                     (block_table, "block_table", torch.int32), (seq_lens, "seq_lens", torch.int32)):
        _need(t, n, dt)
    batch, h_q, d = q.shape
    h_kv, r, _ = basis.shape
    num_pages, _, page_size, _ = score_cache.shape
    if idx is None:
        idx = torch.empty((batch, h_kv, budget), dtype=torch.int32, device=q.device)
    if count is None:
        count = torch.empty((batch, h_kv), dtype=torch.int32, device=q.device)
    max_pages = block_table.shape[1]
    w = _ws(q.device, ws, FN_SCORE_TOPK)
    p, n = w.get(workspace_size(FN_SCORE_TOPK, batch, h_q, h_kv, d, max_pages, page_size, budget))
    call("jssa_score_topk_bf16" if bf16 else "jssa_score_topk", q.data_ptr(), basis.data_ptr(),
         score_cache.data_ptr(),
         block_table.data_ptr(), max_pages, seq_lens.data_ptr(), batch, h_q, h_kv, d, r,
         num_pages, page_size, budget, idx.data_ptr(), count.data_ptr(), p, n, _stream(q.device))
    return idx, count


def indexed_attend(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   block_table: torch.Tensor, idx: torch.Tensor, count: torch.Tensor,
                   scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                   ws: Optional[Workspace] = None) -> torch.Tensor:
    """Gather-free attention of every query head over its KV head's index set."""
    _need(q, "q", torch.bfloat16)
    _need(k_cache, "k_cache", torch.bfloat16, contiguous=False)
    _need(v_cache, "v_cache", torch.bfloat16, contiguous=False)
    _need(block_table, "block_table", torch.int32)
    _need(idx, "idx", torch.int32)
    _need(count, "count", torch.int32)
    batch, h_q, d = q.shape
    num_pages, page_size, h_kv, _ = k_cache.shape
    strides = kv_strides(k_cache)
    if kv_strides(v_cache) != strides:
        raise ValueError("K and V caches must share one layout")
    budget = idx.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    w = _ws(q.device, ws, FN_INDEXED_ATTEND)
    p, n = w.get(workspace_size(FN_INDEXED_ATTEND, batch, h_q, h_kv, d, block_table.shape[1],
                                page_size, budget))
    call("jssa_indexed_attend", q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), *strides,
         block_table.data_ptr(), block_table.shape[1], idx.data_ptr(), count.data_ptr(), batch, h_q,
         h_kv, d, budget, num_pages, page_size, scale, out.data_ptr(), p, n, _stream(q.device))
    return out


def mla_attend(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor,
               idx: torch.Tensor, count: torch.Tensor, scale: float,
               out: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None) -> torch.Tensor:
    """Multi-head latent attention (absorbed queries ``q`` bf16 ``[batch, h_q, 576]``) over the
    selected rows of the latent cache ``kv_cache`` bf16 ``[num_pages, page_size, 576]``; values
    are the first 512 dimensions of each row. Returns bf16 ``[batch, h_q, 512]``."""
    _need(q, "q", torch.bfloat16)
    _need(kv_cache, "kv_cache", torch.bfloat16, contiguous=False)
    _need(block_table, "block_table", torch.int32)
    _need(idx, "idx", torch.int32)
    _need(count, "count", torch.int32)
    batch, h_q, dk = q.shape
    num_pages, page_size, dkc = kv_cache.shape
    if dk != 576 or dkc != 576 or kv_cache.stride(2) != 1:
        raise ValueError("latent rows must be 576 contiguous bf16")
    budget = idx.shape[2]
    out = torch.empty((batch, h_q, 512), dtype=torch.bfloat16, device=q.device) if out is None else out
    w = _ws(q.device, ws, FN_MLA_ATTEND)
    p, n = w.get(workspace_size(FN_MLA_ATTEND, batch, h_q, 1, 576, block_table.shape[1], page_size,
                                budget))
    call("jssa_mla_attend", q.data_ptr(), kv_cache.data_ptr(), kv_cache.stride(0), kv_cache.stride(1),
         block_table.data_ptr(), block_table.shape[1], idx.data_ptr(), count.data_ptr(), batch, h_q,
         budget, num_pages, page_size, scale, out.data_ptr(), p, n, _stream(q.device))
    return out


def mla_decode(q: torch.Tensor, kv_new: Optional[torch.Tensor], kv_cache: torch.Tensor,
               score_cache: torch.Tensor, basis: torch.Tensor, block_table: torch.Tensor,
               seq_lens: torch.Tensor, budget: int, scale: float,
               out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
               count: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None):
    """One decode step of a multi-head latent attention layer: store the new latent row and its
    scoring code (when ``kv_new`` bf16 ``[batch, 576]`` is given), score + top-B over the latent
    scoring cache, latent attention over the selected rows. Returns ``(out, idx, count)``."""
    _need(q, "q", torch.bfloat16)
    if kv_new is not None:
        _need(kv_new, "kv_new", torch.bfloat16)
    _need(kv_cache, "kv_cache", torch.bfloat16, contiguous=False)
    for t, n, dt in ((basis, "basis", torch.float32), (score_cache, "score_cache", torch.uint8),
                     (block_table, "block_table", torch.int32), (seq_lens, "seq_lens", torch.int32)):
        _need(t, n, dt)
    batch, h_q, dk = q.shape
    num_pages, page_size, dkc = kv_cache.shape
    if dk != 576 or dkc != 576 or kv_cache.stride(2) != 1:
        raise ValueError("latent rows must be 576 contiguous bf16")
    r = basis.shape[1]
    max_pages = block_table.shape[1]
    out = torch.empty((batch, h_q, 512), dtype=torch.bfloat16, device=q.device) if out is None else out
    if idx is None:
        idx = torch.empty((batch, 1, budget), dtype=torch.int32, device=q.device)
    if count is None:
        count = torch.empty((batch, 1), dtype=torch.int32, device=q.device)
    w = _ws(q.device, ws, FN_MLA_DECODE)
    p, n = w.get(workspace_size(FN_MLA_DECODE, batch, h_q, 1, 576, max_pages, page_size, budget))
    call("jssa_mla_decode", q.data_ptr(), _ptr(kv_new), kv_cache.data_ptr(), kv_cache.stride(0),
         kv_cache.stride(1), score_cache.data_ptr(), basis.data_ptr(), block_table.data_ptr(),
         max_pages, seq_lens.data_ptr(), batch, h_q, r, num_pages, page_size, budget, scale,
         idx.data_ptr(), count.data_ptr(), out.data_ptr(), p, n, _stream(q.device))
    return out, idx, count


def gather_kv(k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
              idx: torch.Tensor, count: torch.Tensor, bufs=None):
    """Copies of the selected K and V rows in index order (the gather step of the
    gather-then-attend ablation): ``k, v`` bf16 ``[batch, budget_pad, h_kv, d]`` and
    ``lens`` int32 ``[batch]`` (= count[:, 0]); ``bufs`` = (k, v, lens) to reuse."""
    _need(k_cache, "k_cache", torch.bfloat16, contiguous=False)
    _need(v_cache, "v_cache", torch.bfloat16, contiguous=False)
    _need(block_table, "block_table", torch.int32)
    _need(idx, "idx", torch.int32)
    _need(count, "count", torch.int32)
    num_pages, page_size, h_kv, d = k_cache.shape
    strides = kv_strides(k_cache)
    if kv_strides(v_cache) != strides:
        raise ValueError("K and V caches must share one layout")
    batch, _, budget = idx.shape
    budget_pad = -(-budget // 16) * 16
    if bufs is None:
        k = torch.empty((batch, budget_pad, h_kv, d), dtype=torch.bfloat16, device=k_cache.device)
        bufs = (k, torch.empty_like(k), torch.empty((batch,), dtype=torch.int32, device=k_cache.device))
    k, v, lens = bufs
    if k.shape != (batch, budget_pad, h_kv, d) or v.shape != k.shape or lens.shape != (batch,):
        raise ValueError("staging buffers of the wrong shape")
    _need(k, "k", torch.bfloat16)
    _need(v, "v", torch.bfloat16)
    _need(lens, "lens", torch.int32)
    call("jssa_gather_kv", k_cache.data_ptr(), v_cache.data_ptr(), *strides, block_table.data_ptr(),
         block_table.shape[1], idx.data_ptr(), count.data_ptr(), batch, h_kv, d, budget, num_pages,
         page_size, k.data_ptr(), v.data_ptr(), lens.data_ptr(), _stream(k_cache.device))
    return k, v, lens


def staged_pages(k: torch.Tensor, v: torch.Tensor):
    """The staging buffers of :func:`gather_kv` viewed as a paged cache of 16-token pages, with
    its block table (sequence b on its own consecutive pages)."""
    batch, budget_pad, h_kv, d = k.shape
    pages = budget_pad // 16
    kc = k.view(batch * pages, 16, h_kv, d)
    vc = v.view(batch * pages, 16, h_kv, d)
    bt = torch.arange(batch * pages, dtype=torch.int32, device=k.device).view(batch, pages)
    return kc, vc, bt


def gather_then_attend(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                       block_table: torch.Tensor, idx: torch.Tensor, count: torch.Tensor,
                       scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                       ws: Optional[Workspace] = None, bufs=None) -> torch.Tensor:
    """The gather-then-attend ablation: copy the selected rows into staging buffers, then run
    the dense paged decode over them (same result as :func:`indexed_attend`)."""
    k, v, lens = gather_kv(k_cache, v_cache, block_table, idx, count, bufs)
    kc, vc, bt = staged_pages(k, v)
    return dense_decode(q, kc, vc, bt, lens, scale, -1, out, ws)


def dense_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 block_table: torch.Tensor, seq_lens: torch.Tensor, scale: Optional[float] = None,
                 window: int = -1, out: Optional[torch.Tensor] = None,
                 ws: Optional[Workspace] = None) -> torch.Tensor:
    """Dense paged decode attention over ``[max(0, L - window), L)`` (all when window <= 0)."""
    _need(q, "q", torch.bfloat16)
    _need(k_cache, "k_cache", torch.bfloat16, contiguous=False)
    _need(v_cache, "v_cache", torch.bfloat16, contiguous=False)
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32)
    batch, h_q, d = q.shape
    num_pages, page_size, h_kv, _ = k_cache.shape
    strides = kv_strides(k_cache)
    if kv_strides(v_cache) != strides:
        raise ValueError("K and V caches must share one layout")
    max_pages = block_table.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    w = _ws(q.device, ws, FN_DENSE_DECODE)
    p, n = w.get(workspace_size(FN_DENSE_DECODE, batch, h_q, h_kv, d, max_pages, page_size, window))
    call("jssa_dense_decode", q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), *strides,
         block_table.data_ptr(), max_pages, seq_lens.data_ptr(), batch, h_q, h_kv, d, num_pages,
         page_size, window, scale, out.data_ptr(), p, n, _stream(q.device))
    return out


def decode(q: torch.Tensor, k_new: Optional[torch.Tensor], v_new: Optional[torch.Tensor],
           k_cache: torch.Tensor, v_cache: torch.Tensor, score_cache: torch.Tensor,
           basis: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor, budget: int,
           scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
           idx: Optional[torch.Tensor] = None, count: Optional[torch.Tensor] = None,
           ws: Optional[Workspace] = None):
    """One JSSA decode step for one layer (store new token, score + top-B, indexed attend).
    Returns ``(out, idx, count)``."""
    _need(q, "q", torch.bfloat16)
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None:
        _need(k_new, "k_new", torch.bfloat16)
        _need(v_new, "v_new", torch.bfloat16)
    for t, n, dt in ((basis, "basis", torch.float32), (score_cache, "score_cache", torch.uint8),
                     (block_table, "block_table", torch.int32), (seq_lens, "seq_lens", torch.int32)):
        _need(t, n, dt)
    _need(k_cache, "k_cache", torch.bfloat16, contiguous=False)
    _need(v_cache, "v_cache", torch.bfloat16, contiguous=False)
    batch, h_q, d = q.shape
    num_pages, page_size, h_kv, _ = k_cache.shape
    r = basis.shape[1]
    strides = kv_strides(k_cache)
    if kv_strides(v_cache) != strides:
        raise ValueError("K and V caches must share one layout")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    if idx is None:
        idx = torch.empty((batch, h_kv, budget), dtype=torch.int32, device=q.device)
    if count is None:
        count = torch.empty((batch, h_kv), dtype=torch.int32, device=q.device)
    w = _ws(q.device, ws, FN_DECODE)
    p, n = w.get(workspace_size(FN_DECODE, batch, h_q, h_kv, d, block_table.shape[1], page_size,
                                budget))
    call("jssa_decode", q.data_ptr(), _ptr(k_new), _ptr(v_new), k_cache.data_ptr(),
         v_cache.data_ptr(), *strides, score_cache.data_ptr(), basis.data_ptr(),
         block_table.data_ptr(), block_table.shape[1], seq_lens.data_ptr(), batch, h_q, h_kv, d, r,
         num_pages, page_size, budget, scale, idx.data_ptr(), count.data_ptr(), out.data_ptr(), p, n,
         _stream(q.device))
    return out, idx, count


def set_wait_limit(cycles: int) -> int:
    """Clock-cycle limit of the tensor-core waits in the latent attention's tile loop (a debug
    control; <= 0 restores the default). Returns the previous limit."""
    return int(_lib.load().jssa_set_wait_limit(int(cycles)))


def device_error(clear: bool = True, device=None) -> int:
    """Flags raised by the kernels' bounds checks since the last clear (synchronises)."""
    dev = torch.device(device or "cuda")
    flags = ctypes.c_uint32(0)
    call("jssa_device_error", ctypes.byref(flags), int(clear), _stream(dev))
    return int(flags.value)


class PagedLayer:
    """One attention layer's decode state: paged bf16 K/V caches, the FP8 scoring cache, the
    basis and the per-step buffers, with ``step`` running one JSSA decode step."""

    def __init__(self, k_cache, v_cache, block_table, seq_lens, basis, budget, scale=None):
        self.k_cache, self.v_cache = k_cache, v_cache
        self.block_table, self.seq_lens = block_table, seq_lens
        self.basis = basis
        self.budget = budget
        num_pages, page_size, h_kv, d = k_cache.shape
        self.page_size = page_size
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        r = basis.shape[1]
        self.score_cache = torch.zeros((num_pages, h_kv, page_size, r), dtype=torch.uint8,
                                       device=k_cache.device)
        batch = block_table.shape[0]
        self.idx = torch.empty((batch, h_kv, budget), dtype=torch.int32, device=k_cache.device)
        self.count = torch.empty((batch, h_kv), dtype=torch.int32, device=k_cache.device)
        self.ws = Workspace(k_cache.device)        # decode steps
        self.ws_dense = Workspace(k_cache.device)  # dense baseline

    def prefill_scores(self, chunk_pages: int = 4096) -> None:
        """Store the scoring code of every cached position (all slots of every page)."""
        num_pages, page_size, h_kv, d = self.k_cache.shape
        flat = self.k_cache.view(num_pages * page_size, h_kv, d)
        for p0 in range(0, num_pages, chunk_pages):
            p1 = min(num_pages, p0 + chunk_pages)
            slots = torch.arange(p0 * page_size, p1 * page_size, dtype=torch.int64,
                                 device=flat.device)
            store(flat[p0 * page_size:p1 * page_size], slots, self.basis, self.score_cache)

    def step(self, q, k_new=None, v_new=None, out=None):
        return decode(q, k_new, v_new, self.k_cache, self.v_cache, self.score_cache, self.basis,
                      self.block_table, self.seq_lens, self.budget, self.scale, out, self.idx,
                      self.count, self.ws)

    def dense(self, q, out=None, window=-1):
        return dense_decode(q, self.k_cache, self.v_cache, self.block_table, self.seq_lens,
                            self.scale, window, out, self.ws_dense)


class HostPipeline:
    """Decode steps of a ``PagedLayer`` fed from host memory through ``jssa_decode_host``: each
    ``step`` copies that step's query and new K / V rows (host, pinned for overlap) to device
    staging, runs the decode step and copies the output back to host, with the uploads of a step
    running while the previous step computes and its download while the next one does (two
    staging sets and two copy streams inside the library, ordered by events). Steps run on the
    CUDA stream that is current when the pipeline is built. Calls are asynchronous: a step's
    output is in its host buffer, and its host inputs may be rewritten, after ``synchronize``."""

    def __init__(self, layer: "PagedLayer", q_shape, kv_new_shape):
        dev = layer.k_cache.device
        batch, h_q, d = q_shape
        num_pages, page_size, h_kv, _ = layer.k_cache.shape
        r = layer.basis.shape[1]
        self.device = dev
        self.layer = layer
        self.ws = Workspace(dev)
        ws_p, ws_n = self.ws.get(workspace_size(FN_DECODE_HOST, batch, h_q, h_kv, d,
                                                layer.block_table.shape[1], page_size,
                                                layer.budget))
        self._stream = _stream(dev)
        self._mid = (layer.k_cache.data_ptr(), layer.v_cache.data_ptr(), *kv_strides(layer.k_cache),
                     layer.score_cache.data_ptr(), layer.basis.data_ptr(),
                     layer.block_table.data_ptr(), layer.block_table.shape[1],
                     layer.seq_lens.data_ptr(), batch, h_q, h_kv, d, r, num_pages, page_size,
                     layer.budget, layer.scale, layer.idx.data_ptr(), layer.count.data_ptr())
        self._tail = (ws_p, ws_n, self._stream)
        self._ws_p = ws_p
        self._q_shape, self._kv_shape = tuple(q_shape), tuple(kv_new_shape)
        self._fn = load().jssa_decode_host
        # the library keys its copy streams by workspace address: if an earlier pipeline used this
        # address, its next step orders its copies after the work already on the stream again
        call("jssa_decode_host_join", ws_p, self._stream)

    def _host(self, t, name, shape):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu" or t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a bf16 tensor in host memory")
        if tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous with shape {shape}")

    def step(self, q_host, k_new_host, v_new_host, out_host):
        self._host(q_host, "q_host", self._q_shape)
        self._host(out_host, "out_host", self._q_shape)
        if (k_new_host is None) != (v_new_host is None):
            raise ValueError("k_new_host and v_new_host go together")
        if k_new_host is not None:
            self._host(k_new_host, "k_new_host", self._kv_shape)
            self._host(v_new_host, "v_new_host", self._kv_shape)
        check("jssa_decode_host",
              self._fn(q_host.data_ptr(), _ptr(k_new_host), _ptr(v_new_host), *self._mid,
                       out_host.data_ptr(), *self._tail))

    def join(self):
        """Make the pipeline's stream wait for every copy issued so far (the last output
        included)."""
        call("jssa_decode_host_join", self._ws_p, self._stream)

    def synchronize(self):
        self.join()
        torch.cuda.synchronize(self.device)
