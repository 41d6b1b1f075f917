"""Multi-process plumbing of bench.py on CPU (gloo, two ranks).

The hot path shards into independent (batch, kv head) units, so the ranks run
replicas with no data-path collective; what they share is the barrier around the
timed region and the maximum of their times. Both are checked here without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world)})
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup(None, timeout_s=60.0)
    try:
        bench.barrier(w)
        # Rank r "took" 1.5 (r + 1) ms: every rank must report the slowest.
        slowest = bench.max_over_ranks(w, 1.5 * (r + 1))
        seed = bench.replica_seed(r)
        bench.barrier(w)
        with open(os.path.join(out_dir, f"rank{r}.txt"), "w") as f:
            f.write(f"{w} {r} {slowest} {seed} {torch.distributed.get_backend()}\n")
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the gloo path; GPU runs use NCCL")
def test_two_rank_barrier_max_and_replica_seeds(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    rows = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    for r, (w, rank, slowest, seed, backend) in enumerate(rows):
        assert int(w) == world and int(rank) == r
        assert float(slowest) == 1.5 * world          # max over ranks, seen by every rank
        assert backend == "gloo"
    assert len({row[3] for row in rows}) == world       # independent caches per rank


def _bench(args, env_extra=None, timeout=300):
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          env=env, timeout=timeout, cwd=ROOT)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the gloo path; GPU runs use NCCL")
def test_bench_gpus_2_spawns_two_ranks_and_reports_them():
    import json
    r = _bench(["--impl", "reference", "--gpus", "2", "--config", "1", "--steps", "1", "--warmup", "0",
                "--cpu-budget", "0.2"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout                   # rank 0 alone prints
    res = json.loads(lines[0])
    assert res["n_gpus"] == 2 and res["impl"] == "reference"
    assert res["config"]["config_id"] == 1 and res["value"] > 0


def test_bench_rejects_gpus_that_differ_from_the_launcher():
    r = _bench(["--impl", "reference", "--gpus", "1", "--config", "1", "--steps", "1", "--warmup", "0"],
               env_extra={"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode != 0
    assert "WORLD_SIZE=2" in r.stderr


@pytest.mark.parametrize("config", [2, 3, 4, 5])
def test_reference_arm_of_every_config_runs_on_the_host(config):
    import json
    r = _bench(["--impl", "reference", "--config", str(config), "--steps", "1", "--warmup", "0", "--cpu-budget", "0.3"])
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
    assert res["impl"] == "reference" and res["config"]["config_id"] == config
    assert res["value"] > 0 and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["value"] == res["value"]


def test_bench_roofline_and_traffic_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.packed_bytes(128, 3, True) == 72 and bench.packed_bytes(128, 3, False) == 52
    assert bench.packed_bytes(64, 3, True) == 40 and bench.packed_bytes(200, 3, True) == 111
    peaks = {"hbm_gbs": 1000.0, "hbm_src": "measured"}
    r = bench.hbm_roofline("k", 2e9, 1e-3, peaks, "unit")          # 2 GB in 1 ms = 2000 GB/s
    assert abs(r["achieved"] - 2000.0) < 1e-9 and abs(r["frac"] - 2.0) < 1e-12 and r["traffic"] is None
    # a traffic entry counts only while the kernel sources hash to its sha
    key = next(iter(bench.TRAFFIC))
    e = bench.TRAFFIC[key]
    current = bench._sources_sha(e["sources"]) == e["sha"]
    t = bench.traffic_for(key, 10)
    assert (t == e["bytes_per_unit"] * 10) if current else (t is None)
    saved = dict(e)
    try:
        e["sha"] = "0" * 16
        assert bench.traffic_for(key, 10) is None
    finally:
        e.update(saved)
