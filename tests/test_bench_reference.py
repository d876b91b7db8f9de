"""The reference arm of bench.py (the float64 oracle timed on the host cores) runs
without a GPU and prints one JSON line with the bench contract's keys, for the
default workload, the n=5120 inverse and the W2A16 GEMM."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*extra):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "3", *extra], capture_output=True, text=True, cwd=ROOT, env=env, timeout=600)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, proc.stdout
    return json.loads(lines[0])


def _check_contract(d, metric_prefix, unit):
    assert d["impl"] == "reference"
    assert d["metric"].startswith(metric_prefix)
    assert d["unit"] == unit and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


@pytest.mark.timeout(900)
def test_reference_arm_default_workload():
    d = _run()
    _check_contract(d, "butterfly fwd+quant rows/s", "rows/s")
    assert d["config"]["rows_per_gpu"] == 2048 and d["config"]["n"] == 4096


@pytest.mark.timeout(900)
def test_reference_arm_w2a16():
    d = _run("--workload", "w2a16")
    _check_contract(d, "W2A16 GEMM TFLOP/s", "TFLOP/s")


@pytest.mark.timeout(900)
def test_reference_arm_inverse():
    d = _run("--workload", "inv5120")
    _check_contract(d, "butterfly fwd+quant rows/s", "rows/s")
    assert d["config"]["n"] == 5120 and "inverse" in d["config"]["workload"]


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_gpu_local_cpus_sets_and_restores_affinity(monkeypatch):
    """The e2e legs allocate pinned buffers on the CPUs NVML reports as local to the GPU
    (a fake NVML here: the first allowed CPU) and restore the affinity afterwards."""
    import types
    bench = _bench_module()
    before = os.sched_getaffinity(0)
    if len(before) < 2:
        pytest.skip("needs two allowed CPUs")
    first = min(before)
    fake = types.SimpleNamespace(
        nvmlInit=lambda: None, nvmlShutdown=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda uuid: "handle",
        nvmlDeviceGetCpuAffinity=lambda h, n: [(1 << (first % 64)) if i == first // 64 else 0 for i in range(n)])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(bench, "gpu_id_for", lambda dev: "GPU-fake")
    with bench.GpuLocalCpus(0) as loc:
        assert os.sched_getaffinity(0) == {first} and loc.cpus == 1
    assert os.sched_getaffinity(0) == before


def test_gpu_local_cpus_without_nvml_changes_nothing(monkeypatch):
    bench = _bench_module()
    before = os.sched_getaffinity(0)
    monkeypatch.setitem(sys.modules, "pynvml", None)  # import fails
    with bench.GpuLocalCpus(0) as loc:
        assert os.sched_getaffinity(0) == before and loc.cpus is None
    assert os.sched_getaffinity(0) == before
