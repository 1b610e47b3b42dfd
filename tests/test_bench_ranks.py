"""The multi-rank plumbing of bench.py on CPU: world_size-2 `gloo` ranks run the same Ranks
class the GPU bench runs over NCCL.  Checks the barrier, the max over ranks of a timing,
that each rank draws its own batch (weak scaling: independent problems, no data-path
collective), the whole-job rate, the reference arm on a non-zero rank, and that a rank that
never joins ends the others with an error instead of a hang.
"""
import json
import os
import socket
import subprocess
import sys
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))


def _worker(rank, world, port, out_dir):
    _env(rank, world, port)
    sys.path.insert(0, ROOT)
    import bench
    from ssd_inputs import make_prefill
    r = bench.Ranks("gloo", device=torch.device("cpu"), timeout_s=60)
    r.barrier()
    # rank r "took" 1.5 + r ms; every rank must see the slowest
    slowest = r.max(1.5 + rank)
    r.barrier()
    case = make_prefill(1, 64, 2, 64, 16, 1, 64, "bf16", seed=bench.rank_seed(r.rank))
    res = {"rank": r.rank, "world": r.world, "max": slowest,
           "x_sum": float(np.asarray(case.x, np.float64).sum()), "seed": bench.rank_seed(r.rank)}
    r.close()
    with open(os.path.join(out_dir, "%d.json" % rank), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks_barrier_max_and_independent_batches(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / ("%d.json" % r))) for r in range(world)]
    assert [d["rank"] for d in res] == [0, 1] and all(d["world"] == 2 for d in res)
    assert all(d["max"] == 2.5 for d in res)              # max over ranks, seen by all
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["x_sum"] != res[1]["x_sum"]             # each rank its own sequences


def test_job_rate_counts_every_rank_over_the_slowest():
    import bench
    # 2 ranks x 32768 tokens, slowest rank 0.5 ms -> 131072 k tokens/s
    assert bench.job_rate(32768, 2, 0.5) == pytest.approx(2 * 32768 / 0.5e-3)
    assert bench.job_rate(10, 1, 1.0) == pytest.approx(1e4)


def test_single_process_ranks_need_no_process_group(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    r = bench.Ranks("gloo", device=torch.device("cpu"))
    assert (r.world, r.rank, r.dist) == (1, 0, None)
    r.barrier()
    assert r.max(3.25) == 3.25
    r.close()


def test_reference_arm_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert p.returncode == 0 and p.stdout.strip() == ""


_LONE_RANK = r"""
import os, sys, torch
sys.path.insert(0, %r)
import bench
bench.Ranks("gloo", device=torch.device("cpu"), timeout_s=3)
"""


def test_missing_rank_ends_with_an_error_not_a_hang():
    """Rank 1 of 2 never starts: rank 0's process-group set-up must fail within its timeout."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(_free_port()))
    t0 = time.time()
    p = subprocess.run([sys.executable, "-c", _LONE_RANK % ROOT], env=env, capture_output=True, text=True,
                       timeout=120)
    assert p.returncode != 0
    assert time.time() - t0 < 100
