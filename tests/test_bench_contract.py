"""bench.py's host side on the CPU: the JSON line contract, the roofline traffic file, clock summaries.

The reference arm (the CPU oracle on sampled query rows) runs here as a subprocess, the way the driver runs
it. The GPU arm's line has the same keys plus the measured extras and is exercised on a B200.
"""
import hashlib
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

CONTRACT = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "config", "gpu_launches", "e2e")


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "1"], capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in CONTRACT:
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["warmup"] >= 3                       # at least three untimed warm-up steps
    assert d["steps"] == 2 and d["n_gpus"] == 1 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["unit"] == "query-tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_profiled_traffic_is_dropped_once_the_kernel_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# comment\n"
        f"attend:prefill 12345 k.cu {digest} x.md\n"
        "index:prefill 777 k.cu 0000000000000000 y.md\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic() == {"attend:prefill": 12345}
    src.write_text("kernel v2\n")
    assert bench.profiled_traffic() == {}


def test_committed_traffic_file_parses():
    t = bench.profiled_traffic()
    assert isinstance(t, dict)
    for k, v in t.items():
        assert ":" in k and v > 0


def test_clock_summary_reports_median_max_and_reasons():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.samples = [(1965.0, 1965.0, []), (1900.0, 1965.0, ["sw_power_cap"]), (1950.0, 1965.0, [])]
    cs.source = "nvml"
    cs.bus = "00000000:00:00.0"
    s = cs.summary()
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3


def test_roofline_entry_fractions():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1250.0, "source": "measured"}
    r = bench.roofline_entry("tensor", 1.5e12, 2e-3, peaks)
    assert r["bound"] == "tensor" and abs(r["achieved"] - 750.0) < 1e-6 and abs(r["frac"] - 0.5) < 1e-9
    assert r["peak_sustained"] == 1250.0 and abs(r["frac_sustained"] - 0.6) < 1e-9
    r = bench.roofline_entry("hbm", 3e9, 1e-3, peaks, traffic=123)
    assert r["unit"] == "GB/s" and abs(r["frac"] - 0.5) < 1e-9 and r["traffic"] == 123


def test_every_profile_summary_gives_its_ncu_command():
    """Each ncu summary names the command that made it, with the clocks left alone, and runs committed files."""
    import glob
    summaries = glob.glob(os.path.join(ROOT, "profiles", "*.md"))
    assert summaries
    for path in summaries:
        text = open(path).read()
        cmds = [ln for ln in text.splitlines() if ln.strip().startswith("ncu ")]
        assert cmds, f"{path}: no ncu command"
        for c in cmds:
            assert "--clock-control none" in c, f"{path}: {c}"
        assert "_work/" not in text, f"{path} refers to working files"
