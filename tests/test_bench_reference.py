"""bench.py's reference arm (the fp64 oracle on host cores) on CPU: rank 0 prints one JSON
line with the contract's keys; any other rank of a multi-rank launch exits 0 silently."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny-fp32",
                           "--steps", "1", "--warmup", "0"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_rank0_prints_one_line():
    r = _run(0)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == os.cpu_count()
    # the line says what it timed: a bounded sample of layers, extrapolated to a step
    assert d["extrapolated"] is True and d["cpu_baseline"]["extrapolated"] is True
    assert d["timed_layers"] == d["cpu_baseline"]["timed_layers"] == 1
    assert d["measured_wall_s"] > 0 and d["cpu_baseline"]["threads"] >= 1


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(1)
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
