"""bench.py's multi-process plumbing on the CPU, through the command the driver runs: `--gpus 2`
without a launcher starts two ranks under torch.distributed.run (gloo here, no GPU), rank 0 prints
one JSON line whose time is the slowest rank's and whose throughput counts both ranks' work; a
WORLD_SIZE that disagrees with --gpus is an error."""
import json
import os
import subprocess
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parent.parent


def _env(**kw):
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                             "MASTER_PORT")}
    env.update(kw)
    return env


def test_gpus_2_spawns_two_ranks_and_reports_the_job():
    r = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--gpus", "2", "--steps", "3", "--warmup", "3",
                        "--plumbing-check"], capture_output=True, text=True, timeout=300, env=_env(), cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["steps"] == 3
    assert d["total_tokens"] == 2 * 3 * 8
    # whole-job throughput: both ranks' work over the slowest rank's time
    assert abs(d["value"] - d["total_tokens"] / (d["ms_per_step"] * d["steps"] / 1e3)) <= 1e-6 * d["value"]
    assert d["ms_per_step"] * d["steps"] >= d["rank_ms"] - 1e-9


def test_world_size_must_match_gpus():
    r = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--gpus", "2", "--steps", "3", "--warmup", "3",
                        "--plumbing-check"], capture_output=True, text=True, timeout=120,
                       env=_env(WORLD_SIZE="1", RANK="0", LOCAL_RANK="0"), cwd=ROOT)
    assert r.returncode != 0
    assert "WORLD_SIZE" in (r.stderr + r.stdout)
