"""bench.py's JSON contract, checked on CPU through the reference arm (the
oracle on a bounded sample): one JSON line with the keys the driver reads."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT,
                         env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tok/s"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_clock_summary_keeps_the_timed_region_only():
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    # (time, SM MHz, max MHz, reason bits): idle samples outside the window
    c.nvml = [(0.0, 345, 1965, 0), (1.0, 1965, 1965, 0), (1.1, 1965, 1965, 0x4), (1.2, 1950, 1965, 0),
              (5.0, 300, 1965, 0x8)]
    c.mark(0.9, 1.3)
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["source"].startswith("nvml")
    # without NVML samples in the window: the nvidia-smi lines
    c2 = bench.ClockSampler(0)
    c2.lines = ["0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Active",
                "0, 1900, 1965, 710.0, 0x4, Not Active, Not Active, Not Active, Active"]
    s2 = c2.summary()
    assert s2["samples"] == 2 and s2["reasons"] == ["sw_power_cap"] and s2["source"] == "nvidia-smi"


def test_oracle_baseline_uses_every_host_core_and_one():
    sys.path.insert(0, ROOT)
    import bench
    import tqsynth
    shape = tqsynth.StackShape("tiny", 2, 512, 512, 512, 1024)
    d = bench.oracle_baseline(shape, 1, budget_s=0.3)
    assert d["kind"] == "oracle" and d["unit"] == "tok/s"
    assert d["cores"] == bench.host_cores() >= 1
    assert d["value"] > 0 and d["single_thread_value"] > 0
    assert "phase seeds" in d["sample"]


def test_ncu_traffic_only_for_the_kernel_it_was_taken_on(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    prof = tmp_path / "profiles"
    prof.mkdir()
    (tmp_path / "decode_matmul_b200").symlink_to(os.path.join(ROOT, "decode_matmul_b200"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"workload": "qwen3-4b-shaped", "dram_bytes_per_layer": 1000.0, "source_sha256": bench.kernel_source_hash()}
    (prof / "stack1_kernel_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("qwen3-4b-shaped", 36, 1) == 36000.0
    assert bench.ncu_traffic("qwen3-4b-shaped", 36, 2) is None
    assert bench.ncu_traffic("27b-class", 64, 1) is None
    rec["source_sha256"] = "0" * 64
    (prof / "stack1_kernel_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("qwen3-4b-shaped", 36, 1) is None
