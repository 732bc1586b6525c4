"""bench.py's reference arm on CPU: one JSON line with the contract's keys
(the oracle timed on the host cores on a bounded sample of the workload),
and ranks other than 0 exit without work."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, gpus=1):
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env.update(extra_env or {})
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny",
                           "--steps", "2", "--warmup", "3", "--gpus", str(gpus)], cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_one_contract_line():
    p = _run()
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in j, k
    assert j["value"] > 0 and j["unit"] == "tokens/s" and j["higher_is_better"] is True
    assert j["steps"] == 2 and j["warmup"] == 3
    assert j["config"]["workload"] == "tiny"
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"]
    assert cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    p = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, gpus=2)
    assert p.returncode == 0, p.stderr[-2000:]
    assert not [ln for ln in p.stdout.splitlines() if ln.startswith("{")]


def test_gpus_n_starts_n_ranks():
    """`bench.py --gpus 2` run as one plain process starts two ranks itself
    (torch.distributed.run on 127.0.0.1); each sees WORLD_SIZE 2, rank 0
    prints the one line with n_gpus 2 and the other rank exits quietly."""
    p = _run(gpus=2)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_world_size_must_match_gpus():
    p = _run({"RANK": "0", "WORLD_SIZE": "3", "LOCAL_RANK": "0"}, gpus=2)
    assert p.returncode != 0
    assert "WORLD_SIZE=3" in p.stderr
