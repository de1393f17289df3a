"""bench.py's own arm on the GPU: one JSON line carrying every key the benchmark contract
reads -- throughput and timing, the end-to-end figure with its copied bytes, the number of
library kernel launches, the roofline object of the dominant kernel, the clocks sampled during
the timed region, and the per-kernel breakdown.  Run on the 192x336 unit (bf16, 28 layers),
whose solve takes ~13 ms, so the whole check stays around a minute."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_carries_the_contract(cuda_device):
    r = subprocess.run([sys.executable, "bench.py", "--workload", "v0.1-192x336", "--steps", "2",
                        "--warmup", "3", "--no-cpu-baseline"],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout[-3000:]
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "e2e", "gpu_launches", "roofline",
              "clocks", "kernel_ms_per_unit"):
        assert k in d, k
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["dtype"] == "bf16"
    assert "workload" in d["config"]
    # end to end: the same metric through host copies, with the bytes it moved
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    # the library's own kernels ran: 28 layers x 4 Euler steps x (at least QKV, attention,
    # O, up, down) per timed unit
    assert d["gpu_launches"] >= 2 * 28 * 4 * 5
    rf = d["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s"
    assert rf["peak"] > 0 and rf["achieved"] > 0 and 0.0 < rf["frac"] < 1.5
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-9
    assert isinstance(d["clocks"], dict)
    ks = d["kernel_ms_per_unit"]
    for k in ("attention", "gemm_qkv", "gemm_o", "gemm_up", "gemm_down", "append"):
        assert ks[k] > 0, k
