"""bench.py's launcher on the CPU: `--gpus 2` without torchrun starts two
ranks (one process per GPU under torchrun) that find each other, agree on the
rank list and take the max over ranks; a world size that disagrees with
--gpus is an error.  Run with the gloo backend (--check-launch), no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def _env():
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT", "LOCAL_WORLD_SIZE"):
        env.pop(k, None)
    return env


def test_gpus_2_starts_two_ranks():
    r = subprocess.run([sys.executable, BENCH, "--gpus", "2", "--check-launch"], capture_output=True, text=True,
                       timeout=300, env=_env())
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2
    assert d["ranks"] == [0, 1]
    assert d["max_over_ranks"] == 2.0  # rank r reports 1 + r: the max is rank 1's


def test_gpus_1_stays_one_process():
    r = subprocess.run([sys.executable, BENCH, "--check-launch"], capture_output=True, text=True, timeout=300,
                       env=_env())
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([x for x in r.stdout.splitlines() if x.startswith("{")][0])
    assert d["n_gpus"] == 1 and d["ranks"] == [0]


def test_world_size_disagreeing_with_gpus_is_an_error():
    env = _env()
    env.update(WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, BENCH, "--gpus", "2", "--check-launch"], capture_output=True, text=True,
                       timeout=120, env=env)
    assert r.returncode != 0
    assert "--gpus 2" in r.stderr
