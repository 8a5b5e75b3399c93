"""Host-side checks of the benchmark's contract (no GPU): the reference arm's
JSON line carries every key of the contract, both arms describe the workload
with the same config keys, and the stored DRAM traffic is used only while the
kernel sources still hash to the captured ones."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_moe_routed_router_b200 import synth  # noqa: E402

CONTRACT = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def test_reference_arm_line_has_the_contract_keys():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--cfg", "1", "--M", "1",
           "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT,
                       env=dict(os.environ, OMP_NUM_THREADS="1"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert CONTRACT <= set(d), CONTRACT - set(d)
    assert d["impl"] == "reference" and d["higher_is_better"] is True and d["unit"] == "tokens/s"
    assert d["metric"] == bench.METRIC
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # the same workload keys as our arm reports for this config
    assert d["config"] == bench.workload_config(synth.CONFIGS[1], 1, 1, 1)


def test_workload_config_names_the_workload():
    shape = synth.CONFIGS[5]
    c = bench.workload_config(shape, shape.num_layers, 16, 1)
    assert c["workload"].startswith(shape.name) and "24 layers" in c["workload"] and "M=16" in c["workload"]
    assert (c["hidden"], c["moe_inter"], c["experts"], c["top_k"], c["M"], c["layers"]) == (2880, 2880, 32, 4, 16, 24)


def test_stored_traffic_is_used_only_for_the_captured_sources(monkeypatch, tmp_path):
    rec = {"dram_bytes_per_launch": 1020, "algorithmic_bytes_per_launch": 1000, "sources_sha256": "a" * 64}
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    monkeypatch.setattr(bench, "kernel_sources_sha256", lambda: "a" * 64)
    assert bench.measured_traffic(2000) == pytest.approx(2040)       # scaled by the launch's algorithmic bytes
    monkeypatch.setattr(bench, "kernel_sources_sha256", lambda: "b" * 64)
    assert bench.measured_traffic(2000) is None                        # the kernel changed since the capture
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.measured_traffic(2000) is None


def test_source_hash_covers_the_kernel_sources():
    h = bench.kernel_sources_sha256()
    assert len(h) == 64 and int(h, 16) >= 0
    names = sorted(n for n in os.listdir(bench.KERNEL_SOURCES) if n.endswith((".cu", ".cuh")))
    assert {"expert.cuh", "route.cuh", "common.cuh", "ts_moe.cu"} <= set(names)
