"""bench.py's host-side contract, on the CPU: the reference arm's JSON line (it times the oracle,
so it needs no GPU), its silence on ranks other than 0, and the rule that a recorded DRAM
traffic figure is reported only while the kernel's source is the one it was measured on."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_reference(extra_env=None):
    env = dict(os.environ, **(extra_env or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run_reference()
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "stage1"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_is_quiet_on_other_ranks():
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_recorded_traffic_follows_the_kernel_source(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        table = json.load(f)
    for kernel, per_workload in table.items():
        assert kernel in bench.KERNEL_SOURCES, kernel
        for workload, rec in per_workload.items():
            assert rec["bytes_per_launch"] == rec["dram_read"] + rec["dram_write"]
            if rec["source_sha256"] == bench.source_sha(bench.KERNEL_SOURCES[kernel]):
                assert bench.recorded_traffic(kernel, workload) == rec["bytes_per_launch"]
    assert bench.recorded_traffic("attend_gather_umma", "no_such_workload") is None
    # a kernel source that no longer matches its record reports no traffic
    monkeypatch.setattr(bench, "source_sha", lambda rel: "0" * 64)
    for kernel, per_workload in table.items():
        for workload in per_workload:
            assert bench.recorded_traffic(kernel, workload) is None
