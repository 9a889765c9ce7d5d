"""The multi-rank bench path on CPU: world_size-2 gloo ranks run the bench's own
seed sharding and cross-rank reduction (time = max over ranks, work = sum), and the
reference arm does no work on ranks other than 0."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seeds = bench.rank_seeds(rank, (0, 1, 2))
        # rank r: elapsed 100+10r ms, e2e 200-10r ms; work 1e12*(r+1), 2e12*(r+1), 3e12
        times, work = bench.reduce_over_ranks([100.0 + 10 * rank, 200.0 - 10 * rank],
                                              [1e12 * (rank + 1), 2e12 * (rank + 1), 3e12],
                                              torch.device("cpu"), world)
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        out[rank] = (times, work, gathered)
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_sharding():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        times, work, gathered = res[r]
        assert times == [110.0, 200.0]                  # max over ranks
        assert work == [3e12, 6e12, 6e12]               # sum over ranks
        flat = [s for g in gathered for s in g]
        assert len(set(flat)) == len(flat) == 6         # every rank solves different problems
    assert bench.job_value(3e12, 110.0) == pytest.approx(3e12 / 0.110 / 1e12)


def test_single_rank_reduction_is_identity():
    import torch
    times, work = bench.reduce_over_ranks([5.0, 7.0], [1.0, 2.0, 3.0], torch.device("cpu"), 1)
    assert times == [5.0, 7.0] and work == [1.0, 2.0, 3.0]
    assert bench.rank_seeds(0, (0, 1, 2)) == [0, 1, 2]


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_rank0_prints_contract_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "small_bf16", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    for k in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "config",
              "cpu_baseline", "e2e"):
        assert k in line
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
