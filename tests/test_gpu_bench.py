"""bench.py's CUDA arm on small workloads: it runs end to end (device step, e2e with host
buffers and the bitwise output check, rooflines, clocks) and prints one line with every key
of the bench contract."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"}


@pytest.mark.parametrize("workload,extra", [("small-mixed-g4-s1000", "xattn_roofline"),
                                            ("small-xattn-g7-s1000", "xattn_roofline"),
                                            ("small-stack3-s1000", "probe_roofline")])
def test_bench_line_on_a_small_workload(workload, extra):
    res = subprocess.run([sys.executable, "bench.py", "--workload", workload, "--steps", "2", "--warmup", "3",
                          "--no-cpu-baseline"], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert KEYS <= set(line), KEYS - set(line)
    assert line["value"] > 0 and line["n_gpus"] == 1 and line["config"]["workload"] == workload
    assert line["roofline"]["frac"] > 0 and line["e2e"]["value"] > 0 and line["gpu_launches"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["e2e"]["d2h_bytes_per_step"] > 0
    if workload == "small-xattn-g7-s1000":
        assert line[extra]["frac"] > 0
    if workload == "small-stack3-s1000":
        assert line[extra]["bytes"] > 0 and line["config"]["layers"] == 3
