"""Plain fp64 CPU oracle of Joint Subspace Sparse Attention (JSSA) decode and calibration.

Test infrastructure only: the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg use it; the product path never imports, links or calls anything here, and this
module imports nothing from the product package.

Every function restates one step of the method as the pages define it, in float64 NumPy with no
blocking, fusion or reordering. Citations name the page and the section or equation:

* "JSSA summary" = the picx.dev summary of *Joint Subspace Sparse Attention for Efficient
  Long-Context Decoding* (sections "Theoretical Foundation", "3.1 Overview",
  "3.3 Gather-Free Indexed Attention", "3.4 Projected Scoring Cache"; equations (1)-(5)).
* "JSSA README" = the mirror of the official repository README (sections "Highlights",
  "Paper-to-code map", "2. Calibration", "3. Throughput", "4. vLLM configuration reference").

Conventions where the pages are silent (each one is a reading, listed with the others in the
design notes): query head ``i`` belongs to KV head ``i // G``; second moments are uncentred;
eigenvectors are ordered by descending eigenvalue and signed so that each row's largest-magnitude
entry is positive (lowest column on ties); the FP8 cache is a direct saturating round-to-nearest-
even cast with no scale; ties in the top-B selection go to the lower token position; the selected
positions are reported in ascending order and padded with -1.

Inputs are NumPy arrays; bf16 tensors are widened exactly to float64 by the caller.
"""

from __future__ import annotations

import numpy as np

from .bf16 import bf16_decode, bf16_encode
from .fp8 import e4m3_decode, e4m3_encode

# ---------------------------------------------------------------------------------------------
# Calibration: second moments and the joint basis
# ---------------------------------------------------------------------------------------------


def group_mean_query(q: np.ndarray, h_kv: int) -> np.ndarray:
    """Mean of the G query heads that share each KV head.

    JSSA summary, Theoretical Foundation (the text before eq. (1)): selection uses
    ``q_bar = (1/G) sum_g q_g`` over the query heads associated with the KV head; section 3.1,
    step 1. ``q``: ``[..., H_q, d]`` -> ``[..., h_kv, d]``, with query head ``i`` in group
    ``i // G``.
    """
    q = np.asarray(q, dtype=np.float64)
    h_q, d = q.shape[-2:]
    g = h_q // h_kv
    return q.reshape(q.shape[:-2] + (h_kv, g, d)).mean(axis=-2)


def second_moments(qbar: np.ndarray, k: np.ndarray) -> tuple:
    """Uncentred second moments ``G_Qbar = sum_n qbar_n qbar_n^T`` and ``G_K = sum_n k_n k_n^T``
    per KV head.

    JSSA summary, Theoretical Foundation (the matrices in eq. (3)) and section 3.2 ("calibration
    reduces to second-moment accumulation"); JSSA README, section 2. ``qbar``: ``[N, h_kv, d]``,
    ``k``: ``[N, h_kv, d]`` -> two ``[h_kv, d, d]`` arrays.
    """
    qbar = np.asarray(qbar, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    g_q = np.einsum("nhi,nhj->hij", qbar, qbar)
    g_k = np.einsum("nhi,nhj->hij", k, k)
    return g_q, g_k


def unit_trace(g: np.ndarray) -> np.ndarray:
    """``G / tr(G)`` for each head. JSSA summary, Theoretical Foundation (eq. (3): the two second
    moments are unit-trace-normalised independently); JSSA README, paper-to-code map
    (``G_Qm / tr(G_Qm) + G_K / tr(G_K)``)."""
    g = np.asarray(g, dtype=np.float64)
    tr = np.trace(g, axis1=-2, axis2=-1)
    return g / tr[..., None, None]


def sign_rows(m: np.ndarray) -> np.ndarray:
    """Fix each row's sign so its largest-magnitude entry is positive (lowest column on ties)."""
    m = np.array(m, dtype=np.float64, copy=True)
    idx = np.argmax(np.abs(m), axis=-1)  # argmax returns the first (lowest) index on ties
    s = np.sign(np.take_along_axis(m, idx[..., None], axis=-1))
    s[s == 0] = 1.0
    return m * s


def joint_basis(g_q: np.ndarray, g_k: np.ndarray, r: int) -> tuple:
    """``M* = TopEig_r(G~_Qbar + G~_K)^T`` per KV head, and all eigenvalues (descending).

    JSSA summary, Theoretical Foundation, eq. (5): the rows of ``M`` are the eigenvectors of the
    r largest eigenvalues of the sum of the unit-trace second moments; JSSA README, highlights
    and section 2 (one eigendecomposition per layer and KV head). Shapes: ``[h_kv, d, d]`` ->
    ``M [h_kv, r, d]``, ``eigvals [h_kv, d]``.
    """
    a = unit_trace(g_q) + unit_trace(g_k)
    w, u = np.linalg.eigh(a)               # ascending, columns are eigenvectors
    w = w[..., ::-1]
    u = u[..., ::-1]
    m = np.swapaxes(u[..., :r], -1, -2)    # TopEig_r(.) as columns, transposed into rows
    return np.ascontiguousarray(sign_rows(m)), np.ascontiguousarray(w)


def projector(m: np.ndarray) -> np.ndarray:
    """``P = M^T M`` (JSSA summary, Theoretical Foundation)."""
    m = np.asarray(m, dtype=np.float64)
    return np.swapaxes(m, -1, -2) @ m


def l_sel(p: np.ndarray, a_q: np.ndarray, a_k: np.ndarray) -> float:
    """Exact selection objective ``tr((I-P) A_Q (I-P) A_K)``. JSSA summary, eq. (3)."""
    c = np.eye(p.shape[-1]) - p
    return float(np.trace(c @ a_q @ c @ a_k))


def l_marg(p: np.ndarray, a_q: np.ndarray, a_k: np.ndarray) -> float:
    """Marginal objective ``tr((I-P)(A_Q + A_K))``. JSSA summary, eq. (4)."""
    c = np.eye(p.shape[-1]) - p
    return float(np.trace(c @ (a_q + a_k)))


def score_error(qbar: np.ndarray, k: np.ndarray, p: np.ndarray) -> float:
    """``s - s_hat = qbar^T (I - P) k``. JSSA summary, eq. (2)."""
    return float(qbar @ (np.eye(p.shape[-1]) - p) @ k)


# ---------------------------------------------------------------------------------------------
# Decode: store, score, select, attend
# ---------------------------------------------------------------------------------------------


def store_codes(k: np.ndarray, m: np.ndarray) -> np.ndarray:
    """FP8 projected key ``e4m3(M k)`` for each token of one KV head.

    JSSA summary, section 3.4 (``K_proj = K M^T`` kept as an FP8 scoring-only cache); JSSA
    README, section 4 notes (r bytes per token and KV head). ``k``: ``[T, d]``, ``m``:
    ``[r, d]`` -> ``uint8 [T, r]``.
    """
    y = np.asarray(k, dtype=np.float64) @ np.asarray(m, dtype=np.float64).T
    return e4m3_encode(y)


def store_codes_bf16(k: np.ndarray, m: np.ndarray) -> np.ndarray:
    """The scoring-cache ablation: ``bf16(M k)`` (float64 product, one rounding) instead of the
    E4M3 code of :func:`store_codes`. ``k``: ``[T, d]``, ``m``: ``[r, d]`` -> ``uint16 [T, r]``
    bit patterns."""
    y = np.asarray(k, dtype=np.float64) @ np.asarray(m, dtype=np.float64).T
    return bf16_encode(y)


def scores_bf16(codes: np.ndarray, p: np.ndarray) -> np.ndarray:
    """:func:`scores` over a bf16 scoring cache: ``s_t = sum_j bf16(c_tj) p_j``."""
    return bf16_decode(codes) @ np.asarray(p, dtype=np.float64)


def mla_scoring_basis(m_lat: np.ndarray, rope_dims: int = 64) -> np.ndarray:
    """Latent scoring projection of multi-head latent attention: the rank-r basis acts on the
    latent dimensions only and the rotary dimensions pass through unprojected, so a token's
    scoring row is ``[M_lat c ; k_rope]`` (r + rope_dims codes). JSSA README, section 4 notes
    (the MLA basis is [1, r, kv_lora_rank]; the rotary part is kept) and JSSA summary, section 3.4.
    ``m_lat``: ``[r, latent]`` -> ``[r + rope_dims, latent + rope_dims]``."""
    m_lat = np.asarray(m_lat, dtype=np.float64)
    r, lat = m_lat.shape
    out = np.zeros((r + rope_dims, lat + rope_dims))
    out[:r, :lat] = m_lat
    out[r:, lat:] = np.eye(rope_dims)
    return out


def projected_query(qbar: np.ndarray, m: np.ndarray) -> np.ndarray:
    """``p = M q_bar`` (JSSA summary, eq. (1): ``s_hat = q_bar^T P k = (M q_bar) . (M k)``)."""
    return np.asarray(m, dtype=np.float64) @ np.asarray(qbar, dtype=np.float64)


def scores(codes: np.ndarray, p: np.ndarray) -> np.ndarray:
    """Projected score of every cached token, ``s_t = sum_j dec(c_tj) p_j``.

    JSSA summary, eq. (1) with the key side read from the FP8 cache (section 3.4) and section
    3.1 step 2. ``codes``: ``uint8 [L, r]``, ``p``: ``[r]`` -> ``[L]``.
    """
    return e4m3_decode(codes) @ np.asarray(p, dtype=np.float64)


def select_top_b(s: np.ndarray, budget: int) -> np.ndarray:
    """Positions of the ``min(B, L)`` largest scores, ties to the lower position, ascending.

    JSSA summary, section 3.1 step 2 (top-B token positions per KV head); JSSA README, section 4
    (``jssa_budget``: token budget per decode step and KV head).
    """
    s = np.asarray(s, dtype=np.float64)
    t = np.arange(s.shape[0])
    order = np.lexsort((t, -s))            # primary key: score descending; secondary: position
    return np.sort(order[: min(int(budget), s.shape[0])])


def attend(q: np.ndarray, k_sel: np.ndarray, v_sel: np.ndarray, scale: float) -> np.ndarray:
    """Softmax attention of one query head over the given key/value rows.

    JSSA summary, section 3.1 step 3 and section 3.3 (attention from the original full-dim
    query, keys and values at the selected positions). ``q``: ``[d]``; ``k_sel``, ``v_sel``:
    ``[n, d]`` -> ``[d]`` (zeros when ``n == 0``).
    """
    k_sel = np.asarray(k_sel, dtype=np.float64)
    v_sel = np.asarray(v_sel, dtype=np.float64)
    if k_sel.shape[0] == 0:
        return np.zeros(v_sel.shape[-1])
    z = scale * (k_sel @ np.asarray(q, dtype=np.float64))
    w = np.exp(z - z.max())
    w = w / w.sum()
    return w @ v_sel


# ---------------------------------------------------------------------------------------------
# Paged cache addressing and whole decode steps
# ---------------------------------------------------------------------------------------------


def paged_rows(cache: np.ndarray, block_table: np.ndarray, b: int, h: int,
               positions: np.ndarray) -> np.ndarray:
    """Rows of KV head ``h`` at logical positions of sequence ``b`` in a cache laid out
    ``[page, slot, head, ...]``: physical page ``block_table[b, t // page_size]``, slot
    ``t % page_size`` (the standard paged GQA layout, JSSA summary section 3.3)."""
    ps = cache.shape[1]
    positions = np.asarray(positions, dtype=np.int64)
    return cache[block_table[b, positions // ps], positions % ps, h]


def scoring_rows(score_cache: np.ndarray, block_table: np.ndarray, b: int, h: int,
                 length: int) -> np.ndarray:
    """FP8 rows of positions ``0..length-1`` from a scoring cache laid out
    ``[page, head, slot, r]``."""
    ps = score_cache.shape[2]
    t = np.arange(length)
    return score_cache[block_table[b, t // ps], h, t % ps]


def store_step(k_new: np.ndarray, slots: np.ndarray, m: np.ndarray,
               score_cache: np.ndarray) -> None:
    """Write ``e4m3(M_h k)`` for each new token and KV head into the scoring cache in place.

    ``k_new``: ``[T, h_kv, d]``; ``slots``: ``[T]`` flat slot numbers ``page * ps + offset``
    (negative: skip); ``m``: ``[h_kv, r, d]``; ``score_cache``: ``uint8 [pages, h_kv, ps, r]``.
    """
    ps = score_cache.shape[2]
    for t, slot in enumerate(np.asarray(slots, dtype=np.int64)):
        if slot < 0:
            continue
        for h in range(m.shape[0]):
            score_cache[slot // ps, h, slot % ps] = store_codes(k_new[t, h][None], m[h])[0]


def select_step(q: np.ndarray, m: np.ndarray, score_cache: np.ndarray, block_table: np.ndarray,
                seq_lens: np.ndarray, budget: int) -> tuple:
    """Per-(sequence, KV head) index sets for one decode step: group-mean query, projection,
    scores over every cached token, top-B. Returns ``idx int32 [batch, h_kv, budget]`` (ascending,
    -1 padded), ``count int32 [batch, h_kv]`` and the float64 scores per (b, h) as a dict.
    A ``uint16`` scoring cache holds bf16 codes (the ablation), a ``uint8`` one E4M3 codes."""
    score = scores_bf16 if np.asarray(score_cache).dtype == np.uint16 else scores
    batch = q.shape[0]
    h_kv = m.shape[0]
    idx = np.full((batch, h_kv, budget), -1, dtype=np.int32)
    count = np.zeros((batch, h_kv), dtype=np.int32)
    all_scores = {}
    qbar = group_mean_query(q, h_kv)
    for b in range(batch):
        L = int(seq_lens[b])
        for h in range(h_kv):
            s = score(scoring_rows(score_cache, block_table, b, h, L),
                      projected_query(qbar[b, h], m[h]))
            sel = select_top_b(s, budget)
            idx[b, h, : sel.shape[0]] = sel
            count[b, h] = sel.shape[0]
            all_scores[(b, h)] = s
    return idx, count, all_scores


def indexed_attend_step(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                        block_table: np.ndarray, idx: np.ndarray, count: np.ndarray,
                        scale: float) -> np.ndarray:
    """Attention of every query head over its KV head's selected positions, read in place from
    the paged cache (JSSA summary, section 3.3). Returns ``[batch, H_q, d]``."""
    batch, h_q, d = q.shape
    h_kv = idx.shape[1]
    g = h_q // h_kv
    out = np.zeros((batch, h_q, v_cache.shape[-1]))
    for b in range(batch):
        for h in range(h_kv):
            pos = idx[b, h, : count[b, h]].astype(np.int64)
            ks = paged_rows(k_cache, block_table, b, h, pos)
            vs = paged_rows(v_cache, block_table, b, h, pos)
            for j in range(g):
                out[b, h * g + j] = attend(q[b, h * g + j], ks, vs, scale)
    return out


def dense_step(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_table: np.ndarray,
               seq_lens: np.ndarray, scale: float, window: int = -1) -> np.ndarray:
    """Full-KV decode attention over positions ``[max(0, L - window), L)`` (all of them when
    ``window < 0``): the dense baseline (JSSA README, section 3 microbenchmark against full-KV
    decode; section 4 notes: sliding-window layers stay dense)."""
    batch, h_q, d = q.shape
    h_kv = k_cache.shape[2]
    g = h_q // h_kv
    out = np.zeros((batch, h_q, v_cache.shape[-1]))
    for b in range(batch):
        L = int(seq_lens[b])
        lo = 0 if window < 0 else max(0, L - window)
        pos = np.arange(lo, L)
        for h in range(h_kv):
            ks = paged_rows(k_cache, block_table, b, h, pos)
            vs = paged_rows(v_cache, block_table, b, h, pos)
            for j in range(g):
                out[b, h * g + j] = attend(q[b, h * g + j], ks, vs, scale)
    return out


def decode_step(q: np.ndarray, k_new, v_new, k_cache: np.ndarray, v_cache: np.ndarray,
                score_cache: np.ndarray, block_table: np.ndarray, seq_lens: np.ndarray,
                m: np.ndarray, budget: int, scale: float) -> dict:
    """One JSSA decode step on copies of the caches: store the new token (position ``L - 1`` of
    each sequence) when ``k_new``/``v_new`` are given, then select and attend.

    JSSA summary, section 3.1 (steps 1-3); JSSA README, paper-to-code map (store, score + top-B,
    indexed attend). Returns ``out``, ``idx``, ``count``, the per-(b, h) scores and the updated
    caches.
    """
    k_cache = np.array(k_cache, copy=True)
    v_cache = np.array(v_cache, copy=True)
    score_cache = np.array(score_cache, copy=True)
    batch = q.shape[0]
    ps = k_cache.shape[1]
    if k_new is not None:
        slots = np.empty(batch, dtype=np.int64)
        for b in range(batch):
            t = int(seq_lens[b]) - 1
            if t < 0:                      # an empty sequence has no position to store into
                slots[b] = -1
                continue
            page = block_table[b, t // ps]
            k_cache[page, t % ps] = k_new[b]
            v_cache[page, t % ps] = v_new[b]
            slots[b] = int(page) * ps + t % ps
        store_step(k_new, slots, m, score_cache)
    idx, count, s = select_step(q, m, score_cache, block_table, seq_lens, budget)
    out = indexed_attend_step(q, k_cache, v_cache, block_table, idx, count, scale)
    return {"out": out, "idx": idx, "count": count, "scores": s, "k_cache": k_cache,
            "v_cache": v_cache, "score_cache": score_cache}


def calibrate(q: np.ndarray, k: np.ndarray, r: int) -> dict:
    """Whole calibration: group-mean queries, second moments, unit-trace sum, top-r eigenvectors
    (JSSA README, section 2: second moments, then a single eigendecomposition per KV head)."""
    h_kv = k.shape[1]
    qbar = group_mean_query(q, h_kv)
    g_q, g_k = second_moments(qbar, k)
    m, w = joint_basis(g_q, g_k, r)
    return {"gram_q": g_q, "gram_k": g_k, "M": m, "eigvals": w}


def algorithmic_bytes(batch: int, h_kv: int, d: int, seq_len: int, page_size: int, rank: int,
                      budget: int, dense: bool = False) -> int:
    """Bytes one decode step must move for one layer: FP8 scoring rows + selected bf16 K and V
    rows + the page table (queries, outputs and the basis are negligible and not counted).
    Dense: every bf16 K and V row + the page table."""
    pages = -(-seq_len // page_size)
    if dense:
        return batch * (h_kv * seq_len * 2 * d * 2 + 4 * pages)
    return batch * (h_kv * seq_len * rank + h_kv * min(budget, seq_len) * 2 * d * 2 + 4 * pages)
