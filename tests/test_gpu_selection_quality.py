"""Selection quality of the library's own selections (the product path), for the joint basis and
for key-only and query-only bases of the same rank, r in {4, 8, 16, 32}: a data-free analogue of
the pages' basis comparison (JSSA summary, "Ablations", projection rank, Figure 5a; Theoretical
Foundation, eqs. (3)-(5)).

For every (basis, rank) the library stores the FP8 scoring codes of the cached keys (jssa_store)
and selects the top-B per KV head (jssa_score_topk); ranks 4 and 8 run through the r = 16 kernels
with zero rows appended to the basis (their codes are zero, so the scores are those of the smaller
rank). The selections must match the oracle's (same basis, its own codes) within the tie
tolerance; the report then gives, per (basis, rank), the recall of the exact top-B of the
full-dimension group-mean scores and the attention mass the selected positions keep relative to
that exact top-B. The workload is the 128K layer's generator (d 128, 8 KV heads, 4 query heads
each) at 16384 cached positions, B 256, 4 decode queries. Set JSSA_REPORT_DIR to also write the
table as JSON there.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import jssa as O
from oracle.selection_quality import attention_mass, bases
from parity import check_selection, f64
from synth import layer_factors, sample_calibration, sample_decode_queries

pytestmark = pytest.mark.gpu

RANKS = (4, 8, 16, 32)


def test_library_selection_quality():
    import token_level_sparse_fp8_b200 as J
    seed, h_kv, group, d, L, B, nq, ps = 1002, 8, 4, 128, 16384, 256, 4, 16
    dev = torch.device("cuda")
    f = layer_factors(seed, 0, h_kv, d)
    qc, kc = sample_calibration(f, 8192, group, seed, device=dev)
    g_q, g_k = O.second_moments(O.group_mean_query(f64(qc), h_kv), f64(kc))
    del qc, kc
    # the cached keys: a fresh stream of the layer's key distribution, L positions, one sequence
    # per decode query sharing the same pages (identity page table)
    _, keys = sample_calibration(f, L, group, seed, layer=7)
    keys_np = f64(keys)                                      # [L, h_kv, d]
    pages = L // ps
    k_cache = keys.view(pages, ps, h_kv, d).to(dev)
    bt = torch.arange(pages, dtype=torch.int32, device=dev).repeat(nq, 1).contiguous()
    lens = torch.full((nq,), L, dtype=torch.int32, device=dev)
    q = torch.cat([sample_decode_queries(f, 1, group, seed, step=i) for i in range(nq)])
    qn = f64(q)                                              # [nq, h_q, d]
    flat = k_cache.view(pages * ps, h_kv, d)
    slots = torch.arange(pages * ps, dtype=torch.int64, device=dev)
    scale = 1.0 / np.sqrt(d)
    # the exact top-B of the full-dimension group-mean scores and the attention mass
    exact, mass = {}, {}
    for i in range(nq):
        for h in range(h_kv):
            qg = qn[i, h * group:(h + 1) * group]
            k = keys_np[:, h]
            exact[(i, h)] = O.select_top_b(k @ qg.mean(axis=0), B)
            mass[(i, h)] = attention_mass(k, qg, scale)
    report = {}
    for r in RANKS:
        for name, m in bases(g_q, g_k, r).items():
            m32 = np.ascontiguousarray(m, dtype=np.float32)       # [h_kv, r, d]
            r_lib = max(r, 16)
            m_lib = np.zeros((h_kv, r_lib, d), dtype=np.float32)
            m_lib[:, :r] = m32
            sc = torch.zeros((pages, h_kv, ps, r_lib), dtype=torch.uint8, device=dev)
            J.store(flat, slots, torch.from_numpy(m_lib).to(dev), sc)
            idx, count = J.score_topk(q.to(dev), torch.from_numpy(m_lib).to(dev), sc, bt, lens, B)
            gi, gc = idx.cpu().numpy(), count.cpu().numpy()
            # the oracle's selection with the same basis and its own codes
            codes = np.zeros((pages, h_kv, ps, r), dtype=np.uint8)
            for h in range(h_kv):
                codes[:, h] = O.store_codes(keys_np[:, h], m32[h].astype(np.float64)).reshape(pages, ps, r)
            ref_idx, ref_count, s = O.select_step(qn, m32.astype(np.float64), codes,
                                                  bt.cpu().numpy(), np.full(nq, L), B)
            rec, kept = [], []
            for i in range(nq):
                for h in range(h_kv):
                    check_selection(gi[i, h], gc[i, h], ref_idx[i, h], ref_count[i, h], s[(i, h)], B)
                    sel = gi[i, h, :gc[i, h]]
                    rec.append(np.intersect1d(sel, exact[(i, h)]).size / B)
                    kept.append(mass[(i, h)][sel].sum() / mass[(i, h)][exact[(i, h)]].sum())
            report[f"{name}, r {r}"] = {"recall": float(np.mean(rec)), "mass_kept": float(np.mean(kept))}
    print(json.dumps(report, indent=1))
    out_dir = os.environ.get("JSSA_REPORT_DIR")
    if out_dir:
        with open(os.path.join(out_dir, "selection_quality_library.json"), "w") as fh:
            json.dump(report, fh, indent=1)
    # more rank never selects worse on this generator, and r = 32 recovers most of the exact set
    for name in ("joint (JSSA)", "keys only", "queries only"):
        assert report[f"{name}, r 32"]["recall"] >= report[f"{name}, r 4"]["recall"]
    assert report["joint (JSSA), r 32"]["recall"] >= 0.8
