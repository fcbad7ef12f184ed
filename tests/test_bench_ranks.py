"""The multi-rank logic of bench.py, on CPU ranks with the gloo backend.

Under torchrun every rank decodes its own batch (sequences are independent,
so the data path has no collective), the time is the max over ranks and the
whole-job rate counts every rank's tokens.  These tests run that host logic
in two gloo processes; the GPU part of a rank is the same code as at N = 1.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, result_dir: str) -> None:
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    try:
        # the slowest rank sets the time
        t = bench.max_over_ranks(dist, 1.5 + rank, "cpu")
        # each rank draws its own batch of the same shapes
        base = workloads.small("ranks", B=2, H=4, L=300, g=8, w=40, d_c=64, d_r=16, dtype="f32", seed=0)
        wl = bench.rank_workload(base, rank)
        x = workloads.generate(wl)
        digest = float(np.abs(x.c_kv).sum())
        digests = [None] * WORLD
        dist.all_gather_object(digests, (wl.seed, digest, wl.B, wl.L))
        dist.barrier()
        with open(os.path.join(result_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"t": t, "digests": digests}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_per_rank_batches(tmp_path):
    mp.spawn(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]
    for r in res:
        assert r["t"] == 2.5                      # max of 1.5 and 2.5 on every rank
        seeds = [d[0] for d in r["digests"]]
        assert seeds == list(range(WORLD))        # seed = rank
        assert r["digests"][0][1] != r["digests"][1][1]   # different batches
        assert {(d[2], d[3]) for d in r["digests"]} == {(2, 300)}   # same shapes
    assert res[0]["digests"] == res[1]["digests"]


def test_max_over_ranks_without_process_group():
    assert bench.max_over_ranks(None, 3.25, "cpu") == 3.25


def test_whole_job_rate_counts_every_rank():
    wl = workloads.WORKLOADS["v2lite"]
    one = bench.whole_job_rate(1, wl, 10, 1e-3)
    assert one == pytest.approx(wl.B * wl.L * 10 / 1e-3)
    # weak scaling: N ranks with the same per-rank time give N times the rate
    assert bench.whole_job_rate(4, wl, 10, 1e-3) == pytest.approx(4 * one)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_the_contract_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LCA_REFERENCE_BUDGET_S="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["config"]["workload"].startswith("v2:")
    assert d["n_gpus"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_gpus_flag_starts_that_many_ranks():
    """`bench.py --gpus 2` without torchrun launches two local ranks itself
    (here the CPU stand-in arm over gloo); both join and rank 0 reports the
    world size it saw."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "ranks", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and sorted(d["ranks"]) == [0, 1] and d["t_max"] == 2.0
