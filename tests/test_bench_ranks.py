"""The multi-rank path of bench.py on the CPU: two gloo ranks run the same rank
bookkeeping the benchmark runs over NCCL (one process per GPU, every rank its
own instance of the workload, the slowest rank's step time, the whole-job
aggregate, rank 0 alone printing), and the reference arm's non-zero ranks exit
without work."""

from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, outdir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    ranks = bench.Ranks("gloo")
    assert (ranks.rank, ranks.world) == (rank, world)
    ranks.barrier()
    ms_local = 10.0 + 5.0 * rank           # rank 1 is the slow one
    ms = ranks.max(ms_local, "cpu")
    work = 3.0e12                          # flops of one rank's own instance
    value = bench.job_rate(ranks.world, work, ms) / 1e12
    seed = bench.rank_seed(5, rank)
    rec = {"rank": rank, "ms": ms, "value": value, "seed": seed}
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump(rec, f)
    ranks.close()


def test_two_gloo_ranks_take_the_slowest_step_and_aggregate(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    recs = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert all(r["ms"] == 15.0 for r in recs)                  # max over ranks, seen by every rank
    assert recs[0]["value"] == pytest.approx(2 * 3.0e12 / 15e-3 / 1e12)  # all ranks' work / slowest time
    assert recs[0]["seed"] != recs[1]["seed"]                    # each rank its own problem


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line(tmp_path):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "bf16_257x8x128", "--steps", "1", "--warmup", "0"], env=env,
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
