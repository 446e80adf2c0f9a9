"""bench.py's multi-rank launch path on the CPU (gloo): `--gpus N` without a
torch.distributed environment starts N ranks itself, every rank sums its
weight gradients with the others through the bench's all-reduce, and rank 0
prints one JSON line with n_gpus = N; a --gpus that disagrees with
WORLD_SIZE is an error."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def _env(**kw):
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                                                           "MASTER_PORT")}
    env.update(kw)
    return env


def test_gpus_2_launches_two_ranks():
    r = subprocess.run([sys.executable, BENCH, "--gpus", "2", "--dist-check", "--steps", "3"], capture_output=True,
                       text=True, timeout=600, env=_env(), cwd=ROOT)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout  # rank 0 alone prints
    line = lines[0]
    assert line["n_gpus"] == 2 and line["allreduce_sum_ok"] is True, line


def test_gpus_disagreeing_with_world_size_is_an_error():
    r = subprocess.run([sys.executable, BENCH, "--gpus", "2", "--dist-check"], capture_output=True, text=True,
                       timeout=120, env=_env(WORLD_SIZE="3", RANK="0", LOCAL_RANK="0"), cwd=ROOT)
    assert r.returncode == 2 and "WORLD_SIZE" in r.stderr, r.stdout + r.stderr
