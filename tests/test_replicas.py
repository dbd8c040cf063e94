"""Multi-process host logic of the replica form (CPU, gloo, world size 2).

bench.py --gpus N runs N independent replicas; all they share is the barrier
around the timed region, the maximum of the elapsed times over ranks and the
whole-job throughput. These tests run that logic as two gloo ranks on CPU,
including a rank that leaves before the collective.
"""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

from trainable_block_sparse_cube_b200 import replicas


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})


def _worker(rank, world, port, out_dir):
    _env(rank, world, port)
    rep = replicas.from_env("gloo", timeout_s=30)
    rep.barrier()
    t_max = rep.max_over_ranks(1.5 + rank)  # rank r took 1.5 + r seconds
    res = {"world": rep.world, "reporter": rep.is_reporter, "t_max": t_max,
           "throughput": rep.job_throughput(10.0, t_max)}
    rep.barrier()
    rep.close()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)


def _leaver(rank, world, port, out_dir):
    _env(rank, world, port)
    rep = replicas.from_env("gloo", timeout_s=5)
    if rank == 1:
        return  # leaves between steps, before the collective, without closing
    try:
        rep.max_over_ranks(1.0)
        outcome = "no error"
    except Exception as e:  # the peer is gone: the collective must fail, not hang
        outcome = "error: " + type(e).__name__
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"outcome": outcome}, f)


def test_single_process_needs_no_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    rep = replicas.from_env("gloo")
    assert rep.world == 1 and rep.backend is None and rep.is_reporter
    assert rep.max_over_ranks(3.25) == 3.25
    assert rep.job_throughput(10.0, 2.0) == 5.0
    rep.barrier()
    rep.close()


def test_two_ranks_max_time_and_job_throughput(tmp_path):
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, start_method="spawn")
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(2)]
    for i, x in enumerate(r):
        assert x["world"] == 2
        assert x["reporter"] == (i == 0)       # rank 0 alone prints the JSON line
        assert x["t_max"] == 2.5               # the slower rank's time, seen by both
        assert x["throughput"] == 2 * 10.0 / 2.5  # both ranks' work over the max time


@pytest.mark.timeout(120)
def test_a_rank_that_leaves_fails_the_next_collective(tmp_path):
    mp.start_processes(_leaver, args=(2, _free_port(), str(tmp_path)), nprocs=2, start_method="spawn")
    r0 = json.load(open(tmp_path / "r0.json"))
    assert r0["outcome"].startswith("error")
