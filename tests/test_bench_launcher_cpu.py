"""bench.py --gpus N starts N ranks itself (CPU, gloo).

Runs the rank launcher through a stand-in step (tests/bench_rank_stub.py) with
--gpus 2 from a plain process: the launcher must start two ranks under
torch.distributed.run, and exactly one JSON line must come back, from rank 0,
with n_gpus 2 and the slower rank's time (the maximum over ranks).  A world
size that disagrees with --gpus is refused.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STUB = os.path.join(ROOT, "tests", "bench_rank_stub.py")


def _env(**extra):
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env.update(extra)
    return env


def test_gpus_two_starts_two_ranks_and_reports_the_max():
    r = subprocess.run([sys.executable, STUB, "--gpus", "2", "--steps", "3", "--warmup", "3"], cwd=ROOT,
                       capture_output=True, text=True, env=_env(), timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["n_gpus"] == 2
    # rank 0 sleeps 20 ms per step, rank 1 40 ms: the reported time is rank 1's
    assert line["ms_per_step"] >= 40.0
    assert line["rank_ms_per_step"] < line["ms_per_step"]


def test_one_gpu_runs_in_process():
    r = subprocess.run([sys.executable, STUB, "--gpus", "1"], cwd=ROOT, capture_output=True, text=True,
                       env=_env(), timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 1


def test_world_size_must_match_gpus():
    r = subprocess.run([sys.executable, STUB, "--gpus", "4"], cwd=ROOT, capture_output=True, text=True,
                       env=_env(WORLD_SIZE="2", RANK="0", LOCAL_RANK="0"), timeout=120)
    assert r.returncode != 0
    assert "WORLD_SIZE=2 but --gpus 4" in r.stderr
