"""bench.py on a machine without a GPU: the module loads and the reference arm (the oracle on the
host cores) prints one well-formed JSON line for the decode and the prefill workloads."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_bench_module_defines_its_helpers():
    sys.path.insert(0, ROOT)
    import bench
    for name in ("ClockSampler", "_sha", "_peaks", "_tc_peaks", "_graphed", "run_ours", "run_prefill",
                 "run_reference", "cpu_baseline_sample", "cpu_prefill_sample", "block_filter_leg",
                 "cpu_block_filter_sample", "paged_leg"):
        assert hasattr(bench, name), name
    assert bench._sha(bench.TRAFFIC["file"])


@pytest.mark.parametrize("workload", ["2", "3"])
def test_reference_arm_prints_a_json_line(workload):
    line = _run("--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "0")
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_block_filter_cpu_sample():
    """The oracle leg of the block-filter measurement on a small decode workload."""
    sys.path.insert(0, ROOT)
    import bench
    from long_context_sparse_mean_b200 import workloads as W
    wl = W.small(2, L=4096, n_seq=2, T=2)
    dt, thr = bench.cpu_block_filter_sample(wl, [0], 4)
    assert dt > 0 and thr >= 1


def test_block_filter_flag_parses():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"], capture_output=True, text=True,
                         timeout=120, cwd=ROOT)
    assert out.returncode == 0 and "--block-filter" in out.stdout and "--paged" in out.stdout
