"""The bench's JSON contract on the host: the reference arm (the fp64 oracle
timed on the host cores) prints one line with every key the driver reads,
and the measured arm refuses to run without a GPU instead of falling back to
anything else."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=timeout, cwd=ROOT)


def test_reference_arm_prints_the_contract_line():
    r = run_bench("--impl", "reference", "--config", "tiny_f32", "--steps", "2", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 3 and d["vs_baseline"] is None
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_refused():
    r = run_bench("--impl", "reference", "--config", "tiny_f32", "--steps", "1", "--warmup", "1")
    assert r.returncode != 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_measured_arm_fails_loudly_without_a_gpu():
    r = run_bench("--config", "tiny_f32", "--steps", "1", "--warmup", "3", "--no-cpu-baseline")
    assert r.returncode != 0
    assert not [l for l in r.stdout.splitlines() if l.strip().startswith("{")]


def test_clock_sampler_follows_the_ranks_visible_gpu(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3,5,GPU-0f1e2d")
    assert [bench.visible_gpu(r) for r in range(3)] == ["3", "5", "GPU-0f1e2d"]
    assert bench.visible_gpu(4) == "4"
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.visible_gpu(2) == "2"
