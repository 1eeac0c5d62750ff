"""The multi-rank plumbing of bench.py (one process per GPU under torchrun), exercised on CPU with
the gloo backend and two ranks: the barrier, the max over ranks of a time, distinct per-rank
workload seeds, the weak-scaling aggregate, and a clean shutdown. Also the JSON-lines record and
the line of the reference arm (the float64 oracle on host cores), which runs without a GPU."""

import multiprocessing as mp
import json
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        batch, budget, seq_len = 16, 2048, 131072

    group = bench.RankGroup("gloo", timeout_s=60)
    group.barrier()
    t_max = group.max_over_ranks(1.5 + rank)  # ranks report different times
    seed = bench.workload(Args, group.rank).seed
    rate = bench.whole_job_rate(group.world, 800, t_max)
    group.close()
    out.put((rank, group.world, t_max, seed, rate))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, t0, s0, v0), (r1, w1, t1, s1, v1) = res
    assert (r0, r1) == (0, 1) and w0 == w1 == 2
    assert t0 == t1 == 2.5              # max over ranks, seen by every rank
    assert s0 != s1                     # each rank draws its own sequences
    assert v0 == v1 == 2 * 800 / 2.5    # steps of all ranks over the slowest rank's time


def test_single_rank_has_no_process_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench
    g = bench.RankGroup("gloo")
    assert g.world == 1 and g.max_over_ranks(3.0) == 3.0
    g.barrier()
    g.close()


def test_jsonl_records_one_per_configuration(tmp_path):
    # --jsonl: the headline, each sweep row and each sub-workload become one record each
    import bench
    line = {"metric": "m", "value": 6900.0, "ms_per_step": 0.145, "hbm_gbs": 4630.0,
            "roofline_step": {"frac": 0.71}, "speedup_vs_dense": 9.2,
            "config": {"workload": "llama3-8b-layer-128k"},
            "cpu_baseline": {"agreement": {"pairs": 2, "selections_equal": True}},
            "mla": {"value": 7100.0, "ms_per_step": 0.14, "roofline_step": {"frac": 0.33},
                    "config": {"workload": "MLA layer"}},
            "sweep": {"rows": [{"workload": "llama128k", "batch": b, "budget": 2048,
                                "steps_per_s": 1.0, "ms_per_step": 1.0, "hbm_gbs": 1.0,
                                "frac": 0.1, "speedup_vs_dense": 2.0} for b in (1, 4)]}}
    path = tmp_path / "runs.jsonl"
    bench.append_records(str(path), line)
    bench.append_records(str(path), line)  # appended, not overwritten
    recs = [json.loads(x) for x in path.read_text().splitlines()]
    assert len(recs) == 8
    names = [r["configuration"] for r in recs[:4]]
    assert names == ["llama3-8b-layer-128k", "mla", "llama128k batch 1 B 2048",
                     "llama128k batch 4 B 2048"]
    assert recs[0]["roofline_frac"] == 0.71 and recs[0]["oracle_agreement"]["selections_equal"]
    assert recs[2]["steps_per_s"] == 1.0 and recs[2]["impl"] == "jssa"
    bench.append_records(None, line)  # no path: nothing written


def test_reference_arm_line():
    # `bench.py --impl reference` (the float64 oracle on host cores) prints one JSON line with the
    # GPU arm's metric, unit and config, exactly the requested steps, and its own CPU baseline and
    # end-to-end keys (no host-device copies)
    import subprocess
    sys.path.insert(0, ROOT)
    import bench
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "steps/s"
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1 and d["higher_is_better"]

    class Args:
        batch, budget, seq_len = 16, 2048, 131072

    assert d["config"] == bench.config_of(bench.workload(Args, 0), 1)
    assert d["value"] > 0 and abs(d["ms_per_step"] - d["measured_ms_per_pair"]["median"]) < 1e-9
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
