"""bench.py's reference arm (the CPU oracle, the one leg that runs without a GPU): the JSON
line it prints carries every key of the bench contract, and under torchrun only rank 0 prints."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def _check(line, workload):
    assert KEYS <= set(line), KEYS - set(line)
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["config"]["workload"] == workload and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert cb.get("cpu_model") is not None or not os.path.exists("/proc/cpuinfo")
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # The same config object as the CUDA arm prints (the driver compares the two).
    sys.path.insert(0, ROOT)
    import bench
    import workloads as wl
    w = wl.WORKLOADS[workload]
    cfg = line["config"]
    if w.layers > 1:
        ref = bench.stack_config(w, cfg["full_kv_heads"], cfg["omega_msr"], cfg["omega_esr"], line["n_gpus"])
    else:
        ref = bench.workload_config(w, cfg["omega_msr"], cfg["omega_esr"], cfg["forced_sparse_kv_heads"],
                                    line["n_gpus"])
    assert cfg == ref


@pytest.mark.parametrize("workload", ["small-mixed-g4-s1000", "small-xattn-g7-s1000", "small-stack3-s1000"])
def test_reference_arm_line(workload):
    """One line with every contract key; ms_per_step is the sample's own measured time (work
    that ran), and the config is the CUDA arm's."""
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", workload, "--steps", "1",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = _lines(res.stdout)
    assert len(lines) == 1
    _check(lines[0], workload)
    assert 0 < lines[0]["ms_per_step"] and "ms_per_step_is" in lines[0]


def test_reference_arm_forced_heads():
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "small-mixed-g4-s1000",
                          "--omega-sparse", "1", "--steps", "1", "--warmup", "3"], cwd=ROOT, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    line = _lines(res.stdout)[0]
    _check(line, "small-mixed-g4-s1000")
    assert line["config"]["forced_sparse_kv_heads"] == 1


def test_reference_arm_under_torchrun_prints_once():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    res = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                          "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
                          "--gpus", "2", "--workload", "small-mixed-g4-s1000", "--steps", "1", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = _lines(res.stdout)
    assert len(lines) == 1
    _check(lines[0], "small-mixed-g4-s1000")
    assert lines[0]["n_gpus"] == 2


def test_config_states_how_l2_reuse_is_avoided():
    """Timed steps need inputs larger than L2 (126 MB) or a flush: every bench workload's inputs
    exceed L2, and a parity-size case says that it fits instead of claiming otherwise."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as wl
    for name in ("llama3-8b-s32k-streaming", "qwen-g7-s64k-blocksparse", "llama3-8b-b4-s16k-mixed",
                 "llama3-8b-s128k-sweep", "llama3-8b-s32k-xassa"):
        assert bench.l2_note(wl.WORKLOADS[name]).startswith("inputs larger than L2"), name
    small = bench.l2_note(wl.WORKLOADS["small-mixed-g4-s1000"])
    assert small.startswith("inputs fit in L2") and "not a bench line" in small
