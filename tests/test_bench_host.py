"""Host-side pieces of bench.py that need no GPU: the tie between a committed ncu summary and
the kernel source it was taken on, the clock summary's parsing of nvidia-smi lines, and the
reference arm's JSON line (the fp64 oracle on the host cores)."""
import hashlib
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_profile_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    h = hashlib.sha256(src.read_bytes()).hexdigest()
    (prof / "k.md").write_text(f"kernel_source_sha256: {h}\n\nprep_dram_bytes_per_launch: 123456\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("k.md", "kernel.cu", key="prep_dram_bytes_per_launch") == 123456.0
    assert bench.profile_traffic("k.md", "kernel.cu", key="chain_dram_bytes_per_launch") is None
    assert bench.profile_traffic("missing.md", "kernel.cu") is None
    src.write_text("// kernel v2\n")  # the kernel changed after the capture: no traffic claimed
    assert bench.profile_traffic("k.md", "kernel.cu", key="prep_dram_bytes_per_launch") is None


def test_clock_summary_parses_samples_and_reasons():
    c = bench.ClockSampler("GPU-x")
    c.lines = [
        "0, 1965, 1965, 700.1, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.0, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 800.0, Not Active, Not Active, Not Active, Not Active",
        "garbage",
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    c.lines = []
    assert c.summary()["samples"] == 0


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` times the fp64 oracle on the host (no GPU) and prints the
    contract's line with impl, cpu_baseline and e2e."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--ref-tokens", "16"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["host_cpus"] >= d["cpu_baseline"]["cores"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["gpu_launches"] == 0
