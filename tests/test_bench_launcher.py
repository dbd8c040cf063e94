"""CPU checks of bench.py's replica launcher (no GPU work).

With --gpus N and no rank environment, bench.py starts the N replica
processes itself; with the rank environment of torch.distributed.run it
runs one rank. --dry-run replaces the GPU step by a small CPU step so the
launch, the barrier, the max over ranks and the single report line can be
checked here, with the gloo backend.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None, timeout=240):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    env.update(env_extra or {})
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       timeout=timeout, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    return [json.loads(l) for l in p.stdout.splitlines() if l.startswith("{")]


def test_gpus_2_spawns_two_ranks_one_line():
    lines = _run(["--gpus", "2", "--dry-run", "--steps", "5", "--warmup", "3"])
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["scaling"] == "weak"
    assert lines[0]["value"] > 0 and lines[0]["config"]["parallelism"] == "replicas x2"


def test_single_process_default():
    lines = _run(["--dry-run", "--steps", "3", "--warmup", "3"])
    assert len(lines) == 1 and lines[0]["n_gpus"] == 1


def test_mismatched_world_size_is_an_error():
    env = dict(os.environ)
    env.update(WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run"],
                       capture_output=True, text=True, timeout=120, env=env, cwd=ROOT)
    assert p.returncode != 0 and "does not match" in p.stderr
