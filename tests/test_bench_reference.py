"""bench.py's reference arm (the CPU oracle) on the host: one JSON line with
the contract's keys, the oracle's own sample described, no GPU needed."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "3", "--workload", "w8_gemv_1024"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2 and d["warmup"] >= 3
    assert d["config"]["workload"] == "w8_gemv_1024"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_profile_traffic_needs_every_listed_source_current(tmp_path, monkeypatch):
    """The roofline's traffic comes from a committed ncu summary only while
    every source file the summary lists (the kernel's own file among them)
    still has the sha256 recorded there."""
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    csrc = tmp_path / "weight_only_quantized_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cu").write_text("kernel\n")
    (csrc / "h.cuh").write_text("header\n")

    def summary(files):
        body = ["# k", "", "- traffic_bytes_per_launch M=16: 1234", ""]
        for f in files:
            sha = hashlib.sha256((csrc / f).read_bytes()).hexdigest()
            body += [f"- source_sha256: {sha}", f"- source: `weight_only_quantized_02_b200/csrc/{f}`"]
        (tmp_path / "profiles" / "k.md").write_text("\n".join(body) + "\n")

    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    summary(["k.cu", "h.cuh"])
    assert bench.profile_traffic("k.cu", "k.md", 16) == 1234.0
    assert bench.profile_traffic("k.cu", "k.md", 1) is None  # no figure for this M
    assert bench.profile_traffic("other.cu", "k.md", 16) is None  # the kernel's file is not covered
    (csrc / "h.cuh").write_text("header, changed\n")
    assert bench.profile_traffic("k.cu", "k.md", 16) is None  # a listed header changed since the capture
    summary(["h.cuh"])
    assert bench.profile_traffic("k.cu", "k.md", 16) is None  # the kernel's own file unlisted
