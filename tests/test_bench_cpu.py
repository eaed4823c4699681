"""CPU tests of bench.py's contract pieces that need no GPU: the reference arm (the fp64
oracle on the host cores) prints one JSON line with the fields the driver reads, and the
algorithmic work models match their closed forms at the benchmark shape."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.timeout(600)
def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--cpu-tokens", "64"], cwd=ROOT, capture_output=True,
                       text=True, timeout=540)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "bf16_h32_t8192_d128"


def test_work_models():
    sys.path.insert(0, ROOT)
    import bench
    # 2C(3dk + 2dv) + 6 dk dv + C^2/3 at C = 64, d = 128
    assert bench.prefill_flops_per_token_head(128, 128) == pytest.approx(181589.33, rel=1e-6)
    # 2 (7 dk dv + 7 C dk + 5 C dv + 7 C^2 / 3)
    assert bench.backward_flops_per_token_head(128, 128) == pytest.approx(445098.67, rel=1e-6)
    # bf16: q, k, g, v, beta read and out written
    assert bench.prefill_bytes_per_token_head(128, 128) == 2 * (3 * 128 + 128 + 1) + 2 * 128
    assert bench.fp32_alu_peak_tflops() == pytest.approx(74.4, abs=0.05)
