"""bench.py's reference arm on the host: the JSON line the benchmark contract
asks for (keys, types, the oracle as the baseline), and silence on the ranks
other than 0 under a multi-process launch.  The native arm needs a GPU and
is exercised by the GPU runs."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, args=()):
    env = dict(os.environ)
    env.update(extra_env or {})
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3",
           "--ref-budget", "2", *args]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_the_contract_line():
    res = _run()
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "unit", "dtype", "data", "scaling"):
        assert isinstance(d[key], str) and d[key]
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["vs_baseline"] is None
    assert "h3_5s" in d["config"]["workload"]
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == d["value"] and cpu["cores"] >= 1
    assert cpu["unit"] == d["unit"] and cpu["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_gpus_n_starts_n_ranks_and_only_rank_0_prints():
    """--gpus 2 with no torchrun environment starts two ranks itself (never one
    process silently); the ranks count themselves over gloo, so n_gpus is the
    number that ran, and only rank 0 prints a line."""
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
           "--ref-budget", "1", "--gpus", "2"]
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    assert json.loads(lines[0])["n_gpus"] == 2


def test_gpus_must_agree_with_the_launcher():
    res = _run({"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}, args=("--gpus", "4"))
    assert res.returncode != 0
