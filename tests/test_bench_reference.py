"""bench.py's reference arm (the fp64 oracle on the host cores): the JSON line the driver
reads, on CPU.  Rank 0 prints one line; other ranks exit 0 without work."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return [l for l in out.stdout.splitlines() if l.startswith("{")]


def test_reference_arm_prints_the_contract_line():
    lines = _run(["--workload", "tiny_f32", "--steps", "2", "--warmup", "1"])
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "samples/s"
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in d["e2e"]
    for k in ("value", "unit", "cores", "kind", "sample"):
        assert k in d["cpu_baseline"]
    assert d["config"]["workload"] == "tiny_f32"


def test_reference_arm_other_ranks_do_no_work():
    assert _run(["--workload", "tiny_f32", "--steps", "1", "--warmup", "1"],
                {"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_our_arm_refuses_a_gpu_count_it_was_not_launched_with():
    """--gpus N without N ranks would time one GPU and report it as N: it stops first,
    before any device work (this runs on a machine without a GPU)."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1",
                          "--warmup", "3"], cwd=ROOT,
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode != 0
    assert "needs 2 ranks" in out.stderr
