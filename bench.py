"""Decode-attention throughput of JSSA on B200 at 128K context (one layer, Llama-3-8B-shaped).

One step = one ``jssa_decode`` call for the whole batch on one layer: store the new token's K/V
rows and FP8 scoring code, score every cached token, select the top-B per KV head, run the
gather-free indexed attention. Default workload: 32 query / 8 KV heads, d 128, 131072-token
contexts in 16-token pages with a random page permutation, r 32, B 2048, batch 16; synthetic
low-rank keys/queries from the seeded generator; the basis is calibrated on the GPU from 32768
seeded samples per KV head.

The ``e2e`` key times the same steps fed from pinned host buffers through the C ABI
(``jssa_decode_host``: per step the uploads of q, k_new, v_new and the download of the output,
overlapped with the neighbouring steps' kernels).

Prints one JSON line (rank 0). ``--impl reference`` times the float64 CPU oracle instead (the
only reference that exists for this method) on a bounded sample of the same workload.
Multi-GPU (``torchrun``): every rank runs its own batch of sequences (weak scaling, no
collective on the data path); times are the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "JSSA decode-attn steps/s & HBM GB/s at 128K ctx vs dense full-KV, 1×B200"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=["jssa", "reference"], default="jssa")
    ap.add_argument("--workload", choices=["llama128k", "hybrid", "mla"], default="llama128k",
                    help="llama128k: one 128K-context GQA layer (the headline); hybrid: a stack of "
                         "5 sliding-window layers (dense over the last 1024 positions) and 1 global "
                         "JSSA layer, head dim 256, 64K context; mla: one multi-head latent "
                         "attention layer, 128 heads, 576-dim latent rows, 128K context")
    ap.add_argument("--batch", type=int, default=16)
    ap.add_argument("--budget", type=int, default=2048)
    ap.add_argument("--seq-len", type=int, default=131072)
    ap.add_argument("--no-dense", action="store_true", help="skip the dense baseline timing")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-check", action="store_true", help="skip the oracle agreement in the CPU baseline leg")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--mla-batch", type=int, default=16, help="sequences of the mla workload")
    ap.add_argument("--hybrid-batch", type=int, default=8, help="sequences of the hybrid workload")
    ap.add_argument("--jsonl", default=None,
                    help="also append one JSON record per measured configuration (the headline, each "
                         "sweep row, the hybrid stack, the MLA layer) to this file")
    ap.add_argument("--headline-only", action="store_true",
                    help="llama128k: skip the hybrid and mla sub-measurements of the default line")
    return ap.parse_args()


def append_records(path, line):
    """One record per measured configuration of a bench line (time, rate, algorithmic GB/s,
    roofline fraction, the oracle agreement where the line has one), appended to `path`."""
    if not path:
        return
    recs = []
    base = {"impl": line.get("impl", "jssa"), "n_gpus": line.get("n_gpus", 1),
            "metric": line.get("metric"), "time": time.strftime("%Y-%m-%dT%H:%M:%SZ", time.gmtime())}

    def rec(name, d):
        r = dict(base)
        r.update({"configuration": name, "config": d.get("config"), "steps_per_s": d.get("value"),
                  "ms_per_step": d.get("ms_per_step"), "hbm_gbs": d.get("hbm_gbs"),
                  "roofline_frac": (d.get("roofline_step") or {}).get("frac"),
                  "speedup_vs_dense": d.get("speedup_vs_dense")})
        agree = (d.get("cpu_baseline") or {}).get("agreement")
        if agree is not None:
            r["oracle_agreement"] = agree
        return r

    recs.append(rec(line.get("config", {}).get("workload", "headline"), line))
    for name in ("hybrid", "mla"):
        if isinstance(line.get(name), dict):
            recs.append(rec(name, line[name]))
    for row in (line.get("sweep") or {}).get("rows", []):
        r = dict(base)
        r.update({"configuration": f"{row['workload']} batch {row['batch']} B {row['budget']}",
                  "steps_per_s": row["steps_per_s"], "ms_per_step": row["ms_per_step"],
                  "hbm_gbs": row["hbm_gbs"], "roofline_frac": row["frac"],
                  "speedup_vs_dense": row["speedup_vs_dense"]})
        recs.append(r)
    with open(path, "a") as f:
        for r in recs:
            f.write(json.dumps(r) + "\n")


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class RankGroup:
    """One process per GPU (torchrun environment): barriers and the max over ranks of a time.
    Every rank takes the same collective steps in the same order; with one rank nothing is
    initialised. backend: "nccl" on GPUs, "gloo" for the CPU tests of this plumbing."""

    def __init__(self, backend="nccl", device=None, timeout_s=300):
        import torch.distributed as dist
        from datetime import timedelta
        self.rank, self.world, self.local = dist_env()
        self.device = device
        self.dist = dist
        if self.world > 1:
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, x):
        if self.world == 1:
            return x
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.barrier()
            self.dist.destroy_process_group()


def whole_job_rate(world, steps_per_rank, t_max_s):
    """Weak scaling: every rank runs steps_per_rank steps on its own batch; the job's rate is the
    steps all ranks processed over the slowest rank's time."""
    return world * steps_per_rank / t_max_s


# ------------------------------------------------------------------------------------------------
# clocks
# ------------------------------------------------------------------------------------------------


class ClockSampler:
    """SM clock and throttle reasons sampled with NVML from a thread during a timed region."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int, period_s: float = 0.01):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []
        self.thread = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            idx = torch.cuda._get_nvml_device_index(self.cuda_index)
        except Exception:
            idx = self.cuda_index
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        import threading
        try:
            self.nvml, self.h = self._handle()
            self.max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None
            return
        self.stop_flag = threading.Event()

        def run():
            while not self.stop_flag.is_set():
                try:
                    mhz = self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
                    rs = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
                self.stop_flag.wait(self.period)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self) -> dict:
        if self.nvml is None or self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.stop_flag.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        reasons = sorted({name for _, rs in self.samples for bit, name in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


# ------------------------------------------------------------------------------------------------
# workload
# ------------------------------------------------------------------------------------------------


def workload(args, rank):
    from synth import WORKLOADS
    w = WORKLOADS["llama128k"].replace(batch=args.batch, budget=args.budget, seq_len=args.seq_len)
    return w.replace(seed=w.seed + 7919 * rank)


def config_of(w, world):
    """The workload description both arms print (identical for the same arguments)."""
    return {
        "workload": f"llama3-8b-layer-128k: h_q {w.h_q}, h_kv {w.h_kv}, d {w.d}, L {w.seq_len}, "
                    f"page {w.page_size} (permuted), r {w.rank}, B {w.budget}, batch {w.batch} per GPU",
        "global_batch": w.batch * world,
        "seq_len": w.seq_len,
        "budget": w.budget,
        "parallelism": f"dp{world} (independent sequences per GPU)",
        "l2": "inputs larger than L2: the 512 MiB scoring cache is streamed every step; 8 query sets rotate",
    }


def setup_gpu(w, dev):
    import torch
    import token_level_sparse_fp8_b200 as J
    from synth import build_paged_kv, layer_factors, sample_calibration, sample_decode_queries

    f = layer_factors(w.seed, 0, w.h_kv, w.d)
    qc, kc = sample_calibration(f, w.calib_samples, w.group, w.seed, device=dev)
    cal = J.calibrate(qc, kc, w.rank)
    del qc, kc
    kv = build_paged_kv(f, [w.seq_len] * w.batch, w.page_size, w.seed, device=dev)
    layer = J.PagedLayer(kv["k_cache"], kv["v_cache"], kv["block_table"], kv["seq_lens"], cal["M"],
                         w.budget)
    layer.prefill_scores()
    n_q = 8  # distinct query sets, rotated over the steps
    qs = [sample_decode_queries(f, w.batch, w.group, w.seed, step=i, device=dev) for i in range(n_q)]
    # the new token of each step is the last cached position (rewriting it is idempotent)
    t = w.seq_len - 1
    bt = kv["block_table"].long()
    page = bt[:, t // w.page_size]
    k_new = kv["k_cache"][page, t % w.page_size].contiguous()
    v_new = kv["v_cache"][page, t % w.page_size].contiguous()
    torch.cuda.synchronize(dev)
    return {"layer": layer, "qs": qs, "k_new": k_new, "v_new": v_new, "kv": kv, "factors": f,
            "cal": cal}


def timed(fn, steps, warmup, stream, barrier):
    """Device time of `steps` calls of fn (CUDA events on `stream`), after `warmup` calls."""
    import torch
    for i in range(warmup):
        fn(i)
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1) / 1e3


class GraphSteps:
    """`per` consecutive calls fn(first..first+per-1) captured once in a CUDA graph; calling it
    replays the graph. Removes the host launch cost from device timings (the kernels themselves
    are unchanged)."""

    def __init__(self, fn, per, warmup=2, first=0):
        import torch
        for i in range(warmup):
            fn(first + i)
        torch.cuda.synchronize()
        self.per = per
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            for i in range(per):
                fn(first + i)
        torch.cuda.synchronize()

    def __call__(self, i=0):
        self.graph.replay()


def timed_graph(fn, steps, warmup, stream, barrier, per=8):
    """Device time of `steps` calls (rounded up to whole graphs of `per` calls) and the count
    (used for the per-kernel figures, not for the headline steps)."""
    g = GraphSteps(fn, per)
    reps = max(1, -(-steps // per))
    wreps = max(1, -(-warmup // per))
    t = timed(g, reps, wreps, stream, barrier)
    del g
    return t, reps * per


class ExactSteps:
    """Exactly `steps` consecutive calls fn(0..steps-1) per run: a CUDA graph of `per` calls
    replayed steps // per times, then a graph of the steps % per remaining calls (query sets
    rotate with i, so the remainder continues the rotation)."""

    def __init__(self, fn, steps, per=8):
        self.steps = steps
        self.n_main = steps // per
        self.main = GraphSteps(fn, per) if self.n_main else None
        rem = steps % per
        self.rem = GraphSteps(fn, rem, warmup=0, first=self.n_main * per) if rem else None

    def __call__(self):
        for _ in range(self.n_main):
            self.main()
        if self.rem is not None:
            self.rem()


def repeated_runs(run, steps, warmup_fn, warmup, stream, group, sampler=None, min_region_s=0.2,
                  max_repeats=400):
    """Runs of exactly `steps` steps (`run()` issues them), each bracketed by a barrier and a
    device synchronisation on both sides and timed with CUDA events on `stream`, repeated until
    about `min_region_s` of device time so that the clock sampler sees the region; `warmup`
    untimed steps first. Returns the per-run seconds (max over ranks), one entry per run."""
    import torch
    for i in range(warmup):
        warmup_fn(i)
    torch.cuda.synchronize()

    def one():
        group.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        torch.cuda.synchronize()
        group.barrier()
        return group.max_over_ranks(e0.elapsed_time(e1) / 1e3)

    first = one()
    repeats = int(group.max_over_ranks(min(max_repeats, max(1, math.ceil(min_region_s / max(first, 1e-9))))))
    if sampler is not None:
        sampler.start()
    times = [one() for _ in range(repeats)]
    clocks = sampler.stop() if sampler is not None else None
    return times, clocks


def step_stats(times, steps):
    """Per-step milliseconds over the runs: median, p10, p90 (and the run count)."""
    import numpy as np
    per = np.asarray(times) / steps * 1e3
    return {"median": float(np.median(per)), "p10": float(np.percentile(per, 10)),
            "p90": float(np.percentile(per, 90)), "runs": len(times),
            "timed_region_s": float(np.sum(times))}


def algorithmic_bytes(w, dense=False):
    pages = -(-w.seq_len // w.page_size)
    if dense:
        return w.batch * (w.h_kv * w.seq_len * 2 * w.d * 2 + 4 * pages)
    return w.batch * (w.h_kv * w.seq_len * w.rank + w.h_kv * min(w.budget, w.seq_len) * 2 * w.d * 2
                      + 4 * pages)


def recorded_traffic(kernel, w):
    """DRAM bytes per launch from the committed ncu capture of this workload, or None when the
    workload differs or a kernel source changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic_llama128k_b16.json")
    if not (w.batch == 16 and w.seq_len == 131072 and w.budget == 2048 and os.path.exists(path)):
        return None
    rec = json.load(open(path))
    csrc = os.path.join(ROOT, "token_level_sparse_fp8_b200", "csrc")
    for name, digest in rec["sources_sha256_16"].items():
        with open(os.path.join(csrc, name), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != digest:
                return None
    return rec["bytes_per_launch"].get(kernel)


def score_bytes(w):
    pages = -(-w.seq_len // w.page_size)
    return w.batch * (w.h_kv * w.seq_len * w.rank + 4 * pages)


def attend_bytes(w):
    return w.batch * w.h_kv * min(w.budget, w.seq_len) * 2 * w.d * 2


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def bf16_peak():
    """Dense bf16 tensor throughput (TFLOP/s) for a kernel timed alone: the measured burst
    figure, else the pool's earlier measurement."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


# ------------------------------------------------------------------------------------------------
# CPU oracle baseline
# ------------------------------------------------------------------------------------------------


def oracle_pair_inputs(state, w, b, h):
    """Host copies of what the oracle needs for one (sequence, KV head): that sequence's pages of
    the caches (one head) with an identity page table."""
    import numpy as np
    import torch
    from oracle import jssa as O
    layer = state["layer"]
    bt = state["kv"]["block_table"][b].long()
    k = layer.k_cache[bt][:, :, h : h + 1].to(torch.float64).cpu().numpy()
    v = layer.v_cache[bt][:, :, h : h + 1].to(torch.float64).cpu().numpy()
    m = layer.basis[h : h + 1].double().cpu().numpy()
    # the oracle's own store of every position (not the library's scoring cache)
    n_pages, ps = k.shape[0], k.shape[1]
    sc = O.store_codes(k[:, :, 0].reshape(-1, k.shape[-1]), m[0]).reshape(n_pages, 1, ps, -1)
    return k, v, sc, m, np.arange(bt.numel(), dtype=np.int64)[None]


def oracle_step_for_pair(q_b, k, v, sc, m, bt, w):
    """The oracle's select + attend for one (sequence, KV head); q_b is [G, d] of that head."""
    import numpy as np
    from oracle import jssa as O
    lens = np.array([w.seq_len])
    idx, count, s = O.select_step(q_b[None], m, sc, bt, lens, w.budget)
    out = O.indexed_attend_step(q_b[None], k, v, bt, idx, count, 1.0 / math.sqrt(w.d))
    return idx, count, s, out


def pair_agreement(s, sym, budget, go, rout):
    """Oracle agreement of one (sequence, KV head): the index sets may differ only at near-ties,
    the outputs within the parity tolerances."""
    import numpy as np
    kth = np.sort(s)[::-1][min(budget, s.shape[0]) - 1]
    ties_ok = bool(np.all(np.abs(s[sym] - kth) <= 1e-4 * np.abs(s).max()))
    err = np.abs(go - rout)
    rel = float(err.sum() / max(np.abs(rout).sum(), 1e-300))
    return {"swaps": int(sym.size // 2), "ties_ok": ties_ok, "max_abs": float(err.max()),
            "mean_rel": rel, "ok": ties_ok and float(err.max()) <= 1e-2 and rel <= 2e-3}


def cpu_baseline(state, w, seconds, check=True):
    """The oracle, as it stands, on host cores: select + attend for (sequence, KV head) pairs of
    the timed workload, repeated until about `seconds` of CPU time; scaled to one whole step.
    The first oracle result of each pair is also compared with the GPU step's (agreement)."""
    import numpy as np
    import torch
    cores = len(os.sched_getaffinity(0))
    layer = state["layer"]
    q0 = state["qs"][0]
    gout, gidx, gcount = layer.step(q0, state["k_new"], state["v_new"])
    torch.cuda.synchronize()
    q = q0.to(torch.float64).cpu().numpy()
    g = w.group
    pairs = [(0, 0), (w.batch - 1, w.h_kv - 1)]
    inputs = [(q[b, h * g : (h + 1) * g],) + oracle_pair_inputs(state, w, b, h) for b, h in pairs]
    agreement = []
    done, t_total = 0, 0.0
    while t_total < seconds or done < 2:
        qb, k, v, sc, m, bt = inputs[done % len(inputs)]
        t0 = time.perf_counter()
        ridx, rcount, s, rout = oracle_step_for_pair(qb, k, v, sc, m, bt, w)
        t_total += time.perf_counter() - t0
        if check and done < len(pairs):
            b, h = pairs[done]
            gi = gidx[b, h].cpu().numpy()
            sym = np.setxor1d(gi[: int(gcount[b, h])], ridx[0, 0, : rcount[0, 0]])
            go = gout[b, h * g : (h + 1) * g].double().cpu().numpy()
            agreement.append(dict(pair=[b, h], **pair_agreement(s[(0, 0)], sym, w.budget, go, rout[0])))
        done += 1
    per_pair = t_total / done
    pairs_per_step = w.batch * w.h_kv
    steps_per_s = 1.0 / (per_pair * pairs_per_step)
    res = {"value": steps_per_s, "unit": "steps/s", "cores": cores, "kind": "oracle",
           "measured_s_per_pair": per_pair, "extrapolated_pairs_per_step": pairs_per_step,
           "sample": f"{done} oracle calls on 2 (sequence, KV head) pairs of the timed workload "
                     f"(score+top-B+attend over {w.seq_len} tokens, float64 NumPy), {t_total:.1f} s "
                     f"measured; steps/s extrapolated = 1 / (measured time per pair x "
                     f"{pairs_per_step} pairs per step)"}
    if check:
        res["agreement"] = {"ok": all(a["ok"] for a in agreement), "pairs": agreement}
    return res


def cpu_baseline_hybrid(state, w, seconds, local_kv, q0, scale, check=True):
    """The oracle on host cores for the hybrid stack: the global layer's select + attend on
    (sequence, KV head) pairs (as for the single-layer workload) and one sliding-window layer's
    dense attention on a (sequence, KV head) pair; one stack step = pairs x (global + local
    layers x window)."""
    import numpy as np
    import torch
    import token_level_sparse_fp8_b200 as J
    from oracle import jssa as O
    glob = cpu_baseline(state, w, seconds / 2, check)
    t_glob = 1.0 / (glob["value"] * w.batch * w.h_kv)
    gout = J.dense_decode(q0, local_kv["k_cache"], local_kv["v_cache"], local_kv["block_table"],
                          local_kv["seq_lens"], scale, w.window)
    torch.cuda.synchronize()
    b, h, g = 0, 0, w.group
    bt = local_kv["block_table"][b].long()
    k = local_kv["k_cache"][bt][:, :, h : h + 1].double().cpu().numpy()
    v = local_kv["v_cache"][bt][:, :, h : h + 1].double().cpu().numpy()
    ident = np.arange(bt.numel(), dtype=np.int64)[None]
    qb = q0[b : b + 1, h * g : (h + 1) * g].double().cpu().numpy()
    lens = np.array([int(local_kv["seq_lens"][b])])
    done, t_total, rout = 0, 0.0, None
    while t_total < seconds / 2 or done < 2:
        t0 = time.perf_counter()
        rout = O.dense_step(qb, k, v, ident, lens, scale, w.window)
        t_total += time.perf_counter() - t0
        done += 1
    t_local = t_total / done
    per_step = w.batch * w.h_kv * (t_glob + (w.layers - 1) * t_local)
    res = {"value": 1.0 / per_step, "unit": "steps/s", "cores": glob["cores"], "kind": "oracle",
           "sample": f"global layer: {glob['sample']}; sliding-window layer: {done} oracle dense "
                     f"calls over {w.window} positions of one (sequence, KV head), {t_total:.1f} s; "
                     f"steps/s = 1 / ({w.batch * w.h_kv} pairs x (global + {w.layers - 1} x local))"}
    if check:
        go = gout[b, h * g : (h + 1) * g].double().cpu().numpy()
        err = np.abs(go - rout[0])
        rel = float(err.sum() / max(np.abs(rout[0]).sum(), 1e-300))
        local = {"pair": [b, h], "max_abs": float(err.max()), "mean_rel": rel,
                 "ok": float(err.max()) <= 1e-2 and rel <= 2e-3}
        res["agreement"] = {"ok": glob["agreement"]["ok"] and local["ok"],
                            "global": glob["agreement"]["pairs"], "sliding_window": local}
    return res


def cpu_baseline_mla(q, latent, bt, lens, m_lat, sc, idx, count, out, budget, scale, step,
                     seconds, check=True):
    """The oracle on host cores for the MLA step on one sequence (select over the latent scoring
    cache + latent attention over the selected rows), repeated for about `seconds`; the first
    result is also compared with the GPU step's (selection within the tie tolerance, output within
    the output tolerances on the GPU's own index set)."""
    import numpy as np
    import torch
    from oracle import jssa as O
    cores = len(os.sched_getaffinity(0))
    step(0)
    torch.cuda.synchronize()
    batch = q.shape[0]
    b = 0
    L = int(lens[b])
    pages = bt[b].long()
    kv = latent[pages].double().cpu().numpy()[:, :, None]          # [pages, ps, 1, 576]
    ident = np.arange(pages.numel(), dtype=np.int64)[None]
    qn = q[b:b + 1].double().cpu().numpy()
    mn = O.mla_scoring_basis(m_lat[0].double().cpu().numpy())  # the oracle's block basis [128, 576]
    # the oracle's own store of every position (not the library's scoring cache)
    n_pages, ps = kv.shape[0], kv.shape[1]
    codes = O.store_codes(kv.reshape(-1, 576), mn).reshape(n_pages, 1, ps, -1)
    mn = mn[None]
    done, t_total = 0, 0.0
    while t_total < seconds or done < 1:
        t0 = time.perf_counter()
        ridx, rcount, s = O.select_step(qn, mn, codes, ident, np.array([L]), budget)
        O.indexed_attend_step(qn, kv, kv[..., :512], ident, ridx, rcount, scale)
        t_total += time.perf_counter() - t0
        done += 1
    res = {"value": 1.0 / (t_total / done * batch), "unit": "steps/s", "cores": cores,
           "kind": "oracle",
           "sample": f"{done} oracle calls (select over {L} latent scoring rows + latent attention "
                     f"over the top {budget}) on one sequence of the timed workload, float64 NumPy, "
                     f"{t_total:.1f} s; steps/s = 1 / (time per sequence x {batch} sequences)"}
    if check:
        gi = idx[b, 0].cpu().numpy()
        sym = np.setxor1d(gi[: int(count[b, 0])], ridx[0, 0, : rcount[0, 0]])
        gout = O.indexed_attend_step(qn, kv, kv[..., :512], ident, idx[b:b + 1].cpu().numpy(),
                                     count[b:b + 1].cpu().numpy(), scale)
        res["agreement"] = pair_agreement(s[(0, 0)], sym, budget, out[b].double().cpu().numpy(),
                                          gout[0])
    return res


# ------------------------------------------------------------------------------------------------
# arms
# ------------------------------------------------------------------------------------------------


def run_reference(args):
    """CPU oracle arm: rank 0 only. Each step is a bounded sample of the workload, the oracle's
    score + top-B + attend for one (sequence, KV head) pair of it; `ms_per_step` is the measured
    time of that sample, and `value` extrapolates it to whole steps (pairs per step stated)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import numpy as np
    from oracle import jssa as O
    from synth import build_paged_kv, layer_factors, sample_decode_queries
    w = workload(args, 0)
    cores = len(os.sched_getaffinity(0))
    f = layer_factors(w.seed, 0, w.h_kv, w.d)
    # one sequence of the workload, built on the host; the oracle scores one KV head per call
    kv = build_paged_kv(f, [w.seq_len], w.page_size, w.seed, chunk_pages=1024)
    q = sample_decode_queries(f, 1, w.group, w.seed).double().numpy()
    rng = np.random.default_rng(0)
    m = np.linalg.qr(rng.standard_normal((w.d, w.rank)))[0].T[None]  # an orthonormal basis
    h = 0
    k = kv["k_cache"][:, :, h : h + 1].double().numpy()
    v = kv["v_cache"][:, :, h : h + 1].double().numpy()
    sc = np.zeros((k.shape[0], 1, w.page_size, w.rank), dtype=np.uint8)
    sc[:, 0] = O.store_codes(k[:, :, 0].reshape(-1, w.d), m[0]).reshape(k.shape[0], w.page_size, w.rank)
    bt = kv["block_table"].numpy().astype(np.int64)
    qb = q[0, 0 : w.group]
    pairs_per_step = w.batch * w.h_kv
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle_step_for_pair(qb, k, v, sc, m, bt, w)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    per_pair = statistics.median(times)
    value = 1.0 / (per_pair * pairs_per_step)
    sample = (f"each step: the oracle's score+top-B+attend (float64 NumPy) for one (sequence, KV "
              f"head) pair of the workload, {w.seq_len} tokens, timed; value extrapolates the "
              f"median measured time per pair to {pairs_per_step} pairs per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_pair * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "step_is": "one (sequence, KV head) pair per timed step (a bounded sample of one step)",
        "measured_ms_per_pair": {"median": per_pair * 1e3, "p10": float(np.percentile(times, 10)) * 1e3,
                                 "p90": float(np.percentile(times, 90)) * 1e3},
        "extrapolated_pairs_per_step": pairs_per_step,
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "impl_detail": f"float64 NumPy oracle on {cores} host cores",
    }
    print(json.dumps(line), flush=True)
    append_records(args.jsonl, line)


def run_jssa(args):
    import numpy as np
    import torch
    import token_level_sparse_fp8_b200 as J

    rank, world, local = dist_env()
    assert torch.cuda.is_available(), "bench needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    group = RankGroup("nccl", dev)
    barrier, max_over_ranks = group.barrier, group.max_over_ranks

    w = workload(args, rank)
    J._lib.load()
    state = setup_gpu(w, dev)
    layer = state["layer"]
    qs, k_new, v_new = state["qs"], state["k_new"], state["v_new"]
    stream = torch.cuda.current_stream(dev)
    out = torch.empty_like(qs[0])
    nq = len(qs)

    def step(i):
        layer.step(qs[i % nq], k_new, v_new, out)

    # exactly args.steps steps per run, replayed from CUDA graphs (as in the pages' decode
    # protocol); runs repeat until the timed region spans about 0.2 s
    step(0)  # sizes the workspace before capture
    runs = ExactSteps(step, args.steps, nq)
    times, clocks = repeated_runs(runs, args.steps, step, args.warmup, stream, group,
                                  ClockSampler(local))
    del runs
    st = step_stats(times, args.steps)
    launches_per_step = 4  # prep, scan, select, attention

    # per-kernel device times (same configuration, each kernel launched alone)
    idx, count = layer.idx, layer.count

    ws_score, ws_attend = J.Workspace(dev), J.Workspace(dev)

    def score_only(i):
        J.score_topk(qs[i % nq], layer.basis, layer.score_cache, layer.block_table, layer.seq_lens,
                     w.budget, idx, count, ws_score)

    t_score, n_score = timed_graph(score_only, args.steps, args.warmup, stream, barrier, nq)
    t_score = max_over_ranks(t_score) / n_score

    # the attention alone, on the index set of each rotating query set (so its K/V rows change
    # from launch to launch as in the step, instead of repeating one set out of L2)
    sets = []
    for i in range(nq):
        ii, cc = torch.empty_like(idx), torch.empty_like(count)
        J.score_topk(qs[i], layer.basis, layer.score_cache, layer.block_table, layer.seq_lens,
                     w.budget, ii, cc, ws_score)
        sets.append((ii, cc))

    def attend_only(i):
        ii, cc = sets[i % nq]
        J.indexed_attend(qs[i % nq], layer.k_cache, layer.v_cache, layer.block_table, ii, cc,
                         layer.scale, out, ws_attend)

    t_attend, n_attend = timed_graph(attend_only, args.steps, args.warmup, stream, barrier, nq)
    t_attend = max_over_ranks(t_attend) / n_attend

    # the scoring-cache ablation: the same scores from a bf16 cache (twice the bytes)
    t_score_bf16 = None
    if w.rank == 32 and w.d == 128:
        num_pages, page_size = layer.k_cache.shape[0], layer.k_cache.shape[1]
        sc16 = torch.empty((num_pages, w.h_kv, page_size, w.rank), dtype=torch.bfloat16, device=dev)
        flat = layer.k_cache.view(num_pages * page_size, w.h_kv, w.d)
        for p0 in range(0, num_pages, 4096):
            p1 = min(num_pages, p0 + 4096)
            slots = torch.arange(p0 * page_size, p1 * page_size, dtype=torch.int64, device=dev)
            J.store(flat[p0 * page_size:p1 * page_size], slots, layer.basis, sc16)
        idx16, count16 = torch.empty_like(idx), torch.empty_like(count)

        def score_bf16(i):
            J.score_topk(qs[i % nq], layer.basis, sc16, layer.block_table, layer.seq_lens, w.budget,
                         idx16, count16, ws_score)

        t_score_bf16, n16 = timed_graph(score_bf16, args.steps, args.warmup, stream, barrier, nq)
        t_score_bf16 = max_over_ranks(t_score_bf16) / n16
        del sc16

    # the ablation: gather the same index sets into staging buffers, then dense attention there
    ws_gta = J.Workspace(dev)
    bufs = J.gather_kv(layer.k_cache, layer.v_cache, layer.block_table, sets[0][0], sets[0][1])

    def gather_then_attend(i):
        ii, cc = sets[i % nq]
        J.gather_then_attend(qs[i % nq], layer.k_cache, layer.v_cache, layer.block_table, ii, cc,
                             layer.scale, out, ws_gta, bufs)

    gather_then_attend(0)  # sizes the workspace before capture
    t_gta, n_gta = timed_graph(gather_then_attend, args.steps, args.warmup, stream, barrier, nq)
    t_gta = max_over_ranks(t_gta) / n_gta

    t_dense = None
    if not args.no_dense:
        layer.dense(qs[0], out)  # sizes the shared workspace before capture
        t_dense, n_dense = timed_graph(lambda i: layer.dense(qs[i % nq], out), max(8, args.steps // 4),
                                       8, stream, barrier, nq)
        t_dense = max_over_ranks(t_dense) / n_dense

    # end to end through the public API with host buffers: H2D of the step's inputs, D2H of out
    q_host = [q.cpu().pin_memory() for q in qs]
    kn_host, vn_host = k_new.cpu().pin_memory(), v_new.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    # the library's host-buffer decode (jssa_decode_host): a step's uploads run under the previous
    # step's kernels and its download under the next step's; the run ends after the last download
    pipe = J.HostPipeline(layer, qs[0].shape, k_new.shape)

    def e2e_step(i):
        pipe.step(q_host[i % nq], kn_host, vn_host, out_host)

    def e2e_run():
        for i in range(args.steps):
            e2e_step(i)
        pipe.join()

    e2e_times, _ = repeated_runs(e2e_run, args.steps, e2e_step, args.warmup, stream, group)
    t_e2e = statistics.median(e2e_times)
    h2d = qs[0].numel() * 2 + k_new.numel() * 2 + v_new.numel() * 2
    d2h = out.numel() * 2

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(state, w, args.cpu_seconds, check=not args.no_check)

    peak, peak_kind = peaks()
    ms_step = st["median"]
    steps_per_s = world / (ms_step / 1e3)
    bytes_step = algorithmic_bytes(w)
    score_launch_s = t_score
    achieved = score_bytes(w) / score_launch_s / 1e9
    line = {
        "metric": METRIC,
        "value": steps_per_s,
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "ms_per_step_stats": st,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 K/V, e4m3 scoring cache, fp32 math",
        "data": "synthetic",
        "config": config_of(w, world),
        "hbm_gbs": bytes_step / (ms_step / 1e3) / 1e9,
        "roofline_step": {"bound": "hbm", "achieved": bytes_step / (ms_step / 1e3) / 1e9, "peak": peak,
                          "unit": "GB/s", "frac": bytes_step / (ms_step / 1e3) / 1e9 / peak,
                          "traffic": None, "bytes_per_step": bytes_step, "peak_kind": peak_kind},
        "roofline": {"bound": "hbm", "kernel": "score_topk", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak,
                     "traffic": recorded_traffic("score_topk", w),
                     "bytes_per_launch": score_bytes(w), "ms_per_launch": score_launch_s * 1e3,
                     "peak_kind": peak_kind},
        "kernels_ms": {"score_topk": score_launch_s * 1e3, "indexed_attend": t_attend * 1e3,
                       "attend_gbs": attend_bytes(w) / t_attend / 1e9},
        "clocks": clocks,
        "e2e": {"value": whole_job_rate(world, args.steps, t_e2e), "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "timing": f"median of {len(e2e_times)} runs of exactly {args.steps} steps through the "
                          f"C ABI's host-buffer decode (HostPipeline -> jssa_decode_host; per step: pinned-host "
                          f"H2D of q, k_new, v_new and D2H of the output, overlapped with the "
                          f"neighbouring steps' kernels)"},
        "gpu_launches": launches_per_step * args.steps,
        "timing": (f"each run: exactly {args.steps} steps replayed from CUDA graphs (8 consecutive "
                   f"steps per graph, then the remainder), CUDA events on the launching stream, "
                   f"barrier + synchronise on both sides; {st['runs']} runs, median per step "
                   f"(p10 / p90 in ms_per_step_stats)"),
    }
    if t_dense is not None:
        dense_bytes = algorithmic_bytes(w, dense=True)
        line["dense"] = {"steps_per_s": world / t_dense, "ms_per_step": t_dense * 1e3,
                         "hbm_gbs": dense_bytes / t_dense / 1e9, "frac": dense_bytes / t_dense / 1e9 / peak}
        line["speedup_vs_dense"] = t_dense / (ms_step / 1e3)
    if t_score_bf16 is not None:
        bytes16 = score_bytes(w) + w.batch * w.h_kv * w.seq_len * w.rank  # codes twice as wide
        line["ablation_bf16_cache"] = {
            "score_topk_ms_fp8": score_launch_s * 1e3, "score_topk_ms_bf16": t_score_bf16 * 1e3,
            "bf16_over_fp8_time": t_score_bf16 / score_launch_s,
            "bytes_fp8": score_bytes(w), "bytes_bf16": bytes16,
            "bf16_gbs": bytes16 / t_score_bf16 / 1e9,
        }
    line["ablation_gather"] = {
        "gather_free_attend_ms": t_attend * 1e3,
        "gather_then_attend_ms": t_gta * 1e3,
        "gather_free_over_gather": t_gta / t_attend,
    }
    if t_dense is not None:
        line["ablation_gather"]["attend_speedup_vs_dense"] = {
            "gather_free": t_dense / t_attend, "gather_then_attend": t_dense / t_gta}
    if cpu is not None:
        line["cpu_baseline"] = cpu
    # the other two workloads of the method (hybrid local/global stack, MLA layer), measured in the
    # same run as sub-objects; the headline keys above describe the 128K layer only
    del state, layer, qs, k_new, v_new, out, sets, bufs, ws_score, ws_attend, ws_gta
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if not args.headline_only:
        for name, fn in (("hybrid", measure_hybrid), ("mla", measure_mla), ("sweep", measure_sweep)):
            sub = fn(args, group, dev, local, rank, world, with_cpu=False)
            line[name] = {k: v for k, v in sub.items()
                          if k not in ("n_gpus", "higher_is_better", "vs_baseline", "data", "warmup")}
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
    group.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
        append_records(args.jsonl, line)


def measure_sweep(args, group, dev, local, rank, world, with_cpu=False):
    """The decode step at the other sizes of the metric's configurations: the 128K layer at
    batch 1, 4, 8 and 32 (B 2048) and at batch 16 with B 1024 and 4096, and the 32K layer (batch
    8, B 2048). Each row: runs of exactly 32 steps from CUDA graphs repeated over about 0.1 s
    (median), the dense kernel over the same caches, the roofline fraction of the measured copy
    bandwidth."""
    import torch
    import token_level_sparse_fp8_b200 as J
    from synth import WORKLOADS

    peak, peak_kind = peaks()
    rows = []
    cases = [("llama128k", 1, 2048), ("llama128k", 4, 2048), ("llama128k", 8, 2048),
             ("llama128k", 32, 2048), ("llama128k", 16, 1024), ("llama128k", 16, 4096),
             ("llama32k", 8, 2048)]
    stream = torch.cuda.current_stream(dev)
    for name, batch, budget in cases:
        w = WORKLOADS[name].replace(batch=batch, budget=budget)
        w = w.replace(seed=w.seed + 7919 * rank)
        state = setup_gpu(w, dev)
        layer, qs, k_new, v_new = state["layer"], state["qs"], state["k_new"], state["v_new"]
        out = torch.empty_like(qs[0])
        nq = len(qs)

        def step(i):
            layer.step(qs[i % nq], k_new, v_new, out)

        step(0)
        runs = ExactSteps(step, 32, nq)
        times, _ = repeated_runs(runs, 32, step, 4, stream, group, min_region_s=0.1)
        del runs
        ms = step_stats(times, 32)["median"]
        t_dense, n_dense = timed_graph(lambda i: layer.dense(qs[i % nq], out), 8, 3, stream,
                                       group.barrier, nq)
        t_dense = group.max_over_ranks(t_dense) / n_dense
        gbs = algorithmic_bytes(w) / (ms / 1e3) / 1e9
        rows.append({"workload": name, "seq_len": w.seq_len, "batch": batch, "budget": budget,
                     "ms_per_step": ms, "steps_per_s": world / (ms / 1e3), "hbm_gbs": gbs,
                     "frac": gbs / peak, "dense_ms_per_step": t_dense * 1e3,
                     "speedup_vs_dense": t_dense / (ms / 1e3)})
        del state, layer, qs, k_new, v_new, out
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return {"rows": rows, "peak": peak, "peak_kind": peak_kind,
            "timing": "per row: runs of exactly 32 steps replayed from CUDA graphs, CUDA events, "
                      "repeated over about 0.1 s, median per step; dense: 8-step graphs",
            "config": {"workload": "llama3-8b layer (32/8 heads, d 128, 16-token permuted pages, "
                                   "r 32) at 128K and 32K context, the listed batch and budget"}}


def hybrid_bytes(w, dense=False):
    """Algorithmic bytes of one stack step: the global layer (JSSA, or dense over the whole
    context) plus the local layers' K/V rows of the window."""
    pages = -(-w.seq_len // w.page_size)
    local = (w.layers - 1) * w.batch * w.h_kv * w.window * 2 * w.d * 2
    if dense:
        glob = w.batch * (w.h_kv * w.seq_len * 2 * w.d * 2 + 4 * pages)
    else:
        glob = w.batch * (w.h_kv * w.seq_len * w.rank + w.h_kv * min(w.budget, w.seq_len) * 2 * w.d * 2
                          + 4 * pages)
    return glob + local


def run_workload(args, measure):
    """One workload alone (``--workload hybrid`` / ``mla``): its own JSON line."""
    import torch
    rank, world, local = dist_env()
    assert torch.cuda.is_available(), "bench needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    group = RankGroup("nccl", dev)
    line = measure(args, group, dev, local, rank, world, with_cpu=True)
    group.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
        append_records(args.jsonl, line)


def measure_hybrid(args, group, dev, local, rank, world, with_cpu=True):
    """One stack step of a hybrid model: (layers - 1) sliding-window layers, each dense paged
    decode over the last `window` positions of its own KV cache, and one global layer, a full JSSA
    decode step (store + score + top-B + indexed attend) over the whole context."""
    import torch
    import token_level_sparse_fp8_b200 as J
    from synth import WORKLOADS, build_paged_kv, layer_factors

    barrier, max_over_ranks = group.barrier, group.max_over_ranks
    w = WORKLOADS["hybrid"].replace(batch=args.hybrid_batch)
    w = w.replace(seed=w.seed + 7919 * rank)
    J._lib.load()
    state = setup_gpu(w, dev)
    layer = state["layer"]
    qs, k_new, v_new = state["qs"], state["k_new"], state["v_new"]
    nq = len(qs)
    locals_ = []
    for li in range(1, w.layers):
        f = layer_factors(w.seed, li, w.h_kv, w.d)
        kv = build_paged_kv(f, [w.window] * w.batch, w.page_size, w.seed, layer=li, device=dev)
        locals_.append(kv)
    scale = 1.0 / math.sqrt(w.d)
    out = torch.empty_like(qs[0])
    outs = [torch.empty_like(qs[0]) for _ in locals_]
    stream = torch.cuda.current_stream(dev)
    ws_local = J.Workspace(dev)

    def local_layers(i):
        for kv, o in zip(locals_, outs):
            J.dense_decode(qs[i % nq], kv["k_cache"], kv["v_cache"], kv["block_table"],
                           kv["seq_lens"], scale, w.window, o, ws_local)

    def step(i):
        local_layers(i)
        layer.step(qs[i % nq], k_new, v_new, out)

    def dense_step(i):
        local_layers(i)
        layer.dense(qs[i % nq], out)

    step(0)
    dense_step(0)  # sizes the workspaces before capture
    torch.cuda.synchronize()
    runs = ExactSteps(step, args.steps, nq)
    times, clocks = repeated_runs(runs, args.steps, step, args.warmup, stream, group,
                                  ClockSampler(local))
    del runs
    st = step_stats(times, args.steps)
    t_dense = None
    if not args.no_dense:
        t_dense, n_dense = timed_graph(dense_step, max(8, args.steps // 4), 8, stream, barrier, nq)
        t_dense = max_over_ranks(t_dense) / n_dense
    cpu = None
    if with_cpu and rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_hybrid(state, w, args.cpu_seconds, locals_[0], qs[0], scale,
                                  check=not args.no_check)
    peak, peak_kind = peaks()
    ms_step = st["median"]
    bytes_step = hybrid_bytes(w)
    achieved = bytes_step / (ms_step / 1e3) / 1e9
    line = {
        "metric": "hybrid local/global stack decode steps/s (5 sliding-window + 1 global JSSA layer), 1xB200",
        "value": world / (ms_step / 1e3),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "ms_per_step_stats": st,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 K/V, e4m3 scoring cache, fp32 math",
        "data": "synthetic",
        "config": {
            "workload": f"hybrid stack: {w.layers - 1} sliding-window layers (dense over the last "
                        f"{w.window} positions) + 1 global JSSA layer; h_q {w.h_q}, h_kv {w.h_kv}, "
                        f"d {w.d}, L {w.seq_len}, page {w.page_size} (permuted), r {w.rank}, "
                        f"B {w.budget}, batch {w.batch} per GPU",
            "global_batch": w.batch * world,
            "seq_len": w.seq_len,
            "budget": w.budget,
            "parallelism": f"dp{world} (independent sequences per GPU)",
            "l2": "inputs larger than L2: the global layer's 256 MiB scoring cache is streamed every step",
        },
        "hbm_gbs": achieved,
        "roofline_step": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                          "frac": achieved / peak, "traffic": None, "bytes_per_step": bytes_step,
                          "peak_kind": peak_kind},
        "clocks": clocks,
        "gpu_launches": (w.layers - 1 + 4) * args.steps,  # a dense kernel per local layer + 4
        "timing": (f"each run: exactly {args.steps} stack steps replayed from CUDA graphs, CUDA "
                   f"events; {st['runs']} runs, median per step"),
    }
    if t_dense is not None:
        dense_bytes = hybrid_bytes(w, dense=True)
        line["dense"] = {"steps_per_s": world / t_dense, "ms_per_step": t_dense * 1e3,
                         "hbm_gbs": dense_bytes / t_dense / 1e9, "frac": dense_bytes / t_dense / 1e9 / peak}
        line["speedup_vs_dense"] = t_dense / (ms_step / 1e3)
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def mla_bytes(batch, seq_len, budget, page_size, dense=False):
    """Algorithmic bytes of one MLA decode step: 128-byte scoring rows + the selected 1152-byte
    latent rows + page table (dense: every latent row)."""
    pages = -(-seq_len // page_size)
    if dense:
        return batch * (seq_len * 1152 + 4 * pages)
    return batch * (seq_len * 128 + min(budget, seq_len) * 1152 + 4 * pages)


def measure_mla(args, group, dev, local, rank, world, with_cpu=True):
    """One decode step of a multi-head latent attention layer (128 query heads, one latent head of
    512 + 64 dims, 64-token pages): store of the new token's scoring row, score + top-B on the
    latent scoring cache, absorbed latent attention over the selected rows."""
    import torch
    import token_level_sparse_fp8_b200 as J
    from synth import build_paged_kv, layer_factors, sample_calibration, sample_decode_queries

    barrier, max_over_ranks = group.barrier, group.max_over_ranks
    batch, h_q, L, ps, B, r_lat = args.mla_batch, 128, args.seq_len, 64, args.budget, 64
    seed = 1004 + 7919 * rank
    J._lib.load()
    f = layer_factors(seed, 0, 1, 576)
    # latent basis [1, 64, 512]: the library's second moments of the head-mean latent queries and
    # of the latent rows, then its Jacobi solver at d 512
    qc, kc = sample_calibration(f, 4096, h_q, seed, device=dev)
    cal = J.Calibration(1, 512, dev)
    cal.add_latent(qc, kc[:, 0])
    m_lat, _ = cal.basis(r_lat)
    del qc, kc, cal
    kv = build_paged_kv(f, [L] * batch, ps, seed, device=dev)
    latent = kv["k_cache"].view(kv["k_cache"].shape[0], ps, 576)
    del kv["v_cache"]
    bt, lens = kv["block_table"], kv["seq_lens"]
    num_pages = latent.shape[0]
    sc = torch.zeros((num_pages, 1, ps, 128), dtype=torch.uint8, device=dev)
    flat = latent.view(num_pages * ps, 1, 576)
    for p0 in range(0, num_pages, 4096):
        p1 = min(num_pages, p0 + 4096)
        slots = torch.arange(p0 * ps, p1 * ps, dtype=torch.int64, device=dev)
        J.store(flat[p0 * ps:p1 * ps], slots, m_lat, sc)
    nq = 8
    qs = [sample_decode_queries(f, batch, h_q, seed, step=i, device=dev) for i in range(nq)]
    # the new token of each step is the last cached position (rewriting its code is idempotent)
    t = L - 1
    new_slots = (bt[:, t // ps].long() * ps + t % ps).contiguous()
    k_new = flat[new_slots].contiguous()
    idx = torch.empty((batch, 1, B), dtype=torch.int32, device=dev)
    count = torch.empty((batch, 1), dtype=torch.int32, device=dev)
    out = torch.empty((batch, h_q, 512), dtype=torch.bfloat16, device=dev)
    ws_s, ws_a = J.Workspace(dev), J.Workspace(dev)
    scale = 1.0 / math.sqrt(576.0)
    stream = torch.cuda.current_stream(dev)

    kv_new = k_new.view(batch, 576)
    ws_d = J.Workspace(dev)

    def step(i):
        # one call: the new latent row and its scoring code, score + top-B, latent attention
        J.mla_decode(qs[i % nq], kv_new, latent, sc, m_lat, bt, lens, B, scale, out, idx, count,
                     ws_d)

    step(0)  # sizes the workspaces before capture
    torch.cuda.synchronize()
    runs = ExactSteps(step, args.steps, nq)
    times, clocks = repeated_runs(runs, args.steps, step, args.warmup, stream, group,
                                  ClockSampler(local))
    del runs
    st = step_stats(times, args.steps)

    def attend_only(i):
        J.mla_attend(qs[i % nq], latent, bt, idx, count, scale, out, ws_a)

    t_att, n_att = timed_graph(attend_only, args.steps, args.warmup, stream, barrier, nq)
    t_att = max_over_ranks(t_att) / n_att

    def score_only(i):
        J.score_topk(qs[i % nq], m_lat, sc, bt, lens, B, idx, count, ws_s)

    t_sc, n_sc = timed_graph(score_only, args.steps, args.warmup, stream, barrier, nq)
    t_sc = max_over_ranks(t_sc) / n_sc
    t_dense = None
    if not args.no_dense:
        idx_full = torch.arange(L, dtype=torch.int32, device=dev).repeat(batch, 1).view(batch, 1, L)
        count_full = torch.full((batch, 1), L, dtype=torch.int32, device=dev)
        ws_full = J.Workspace(dev)

        def dense(i):
            J.mla_attend(qs[i % nq], latent, bt, idx_full, count_full, scale, out, ws_full)

        dense(0)
        t_dense, n_dense = timed_graph(dense, max(8, args.steps // 8), 8, stream, barrier, nq)
        t_dense = max_over_ranks(t_dense) / n_dense
    cpu = None
    if with_cpu and rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_mla(qs[0], latent, bt, lens, m_lat, sc, idx, count, out, B, scale, step,
                               args.cpu_seconds, check=not args.no_check)
    peak, peak_kind = peaks()
    ms_step = st["median"]
    bytes_step = mla_bytes(batch, L, B, ps)
    achieved = bytes_step / (ms_step / 1e3) / 1e9
    flops_att = 2.0 * batch * h_q * min(B, L) * (576 + 512)
    line = {
        "metric": "MLA decode steps/s (128 heads, 576-dim latent rows) at 128K ctx, 1xB200",
        "value": world / (ms_step / 1e3),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "ms_per_step_stats": st,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 latent rows, e4m3 scoring cache, fp32 math",
        "data": "synthetic",
        "config": {
            "workload": f"MLA layer: h_q {h_q}, latent 512 + rotary 64 (1152 B per token), scoring "
                        f"64 latent + 64 rotary FP8 codes (128 B per token), L {L}, page {ps} "
                        f"(permuted), B {B}, batch {batch} per GPU",
            "global_batch": batch * world,
            "seq_len": L,
            "budget": B,
            "parallelism": f"dp{world} (independent sequences per GPU)",
            "l2": "inputs larger than L2: the 256 MiB scoring cache is streamed every step",
        },
        "hbm_gbs": achieved,
        "roofline_step": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                          "frac": achieved / peak, "traffic": None, "bytes_per_step": bytes_step,
                          "peak_kind": peak_kind},
        "mla_attend": {"ms": t_att * 1e3, "tflops_algorithmic": flops_att / t_att / 1e12,
                       "hbm_gbs": batch * min(B, L) * 1152 / t_att / 1e9},
        "score_topk": {"ms": t_sc * 1e3, "hbm_gbs": batch * (L * 128 + 4 * (-(-L // ps))) / t_sc / 1e9},
        # the two calls of the step, each against its own bound: score + top-B streams the
        # scoring cache (HBM), the latent attention is a bf16 contraction on tcgen05
        "roofline": {"bound": "hbm", "kernel": "score_topk",
                     "achieved": batch * (L * 128 + 4 * (-(-L // ps))) / t_sc / 1e9, "peak": peak,
                     "unit": "GB/s", "frac": batch * (L * 128 + 4 * (-(-L // ps))) / t_sc / 1e9 / peak,
                     "traffic": None, "peak_kind": peak_kind},
        "roofline_attend": {"bound": "tensor", "kernel": "mla_attend",
                            "achieved": flops_att / t_att / 1e12, "peak": bf16_peak()[0],
                            "unit": "TFLOP/s", "frac": flops_att / t_att / 1e12 / bf16_peak()[0],
                            "traffic": None, "peak_kind": bf16_peak()[1]},
        "clocks": clocks,
        "gpu_launches": 4 * args.steps,  # prep (with the store), scan, select, latent attention
        "timing": (f"each run: exactly {args.steps} steps replayed from CUDA graphs, CUDA events; "
                   f"{st['runs']} runs, median per step"),
    }
    if t_dense is not None:
        dense_bytes = mla_bytes(batch, L, B, ps, dense=True)
        line["dense"] = {"steps_per_s": world / t_dense, "ms_per_step": t_dense * 1e3,
                         "hbm_gbs": dense_bytes / t_dense / 1e9, "frac": dense_bytes / t_dense / 1e9 / peak,
                         "kind": "the same latent attention kernel over every position"}
        line["speedup_vs_dense"] = t_dense / (ms_step / 1e3)
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "hybrid":
        run_workload(args, measure_hybrid)
    elif args.workload == "mla":
        run_workload(args, measure_mla)
    else:
        run_jssa(args)


if __name__ == "__main__":
    main()
