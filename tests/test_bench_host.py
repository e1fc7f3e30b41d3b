"""Host helpers of bench.py that need no GPU.

The clock sampler is driven by a stand-in `nvidia-smi` on PATH that prints a
sample every 50 ms: a timed region much shorter than the sampling interval
must still come back with samples and the throttle reasons they report.
"""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FAKE = """#!{py}
import time
while True:
    print("0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Active", flush=True)
    time.sleep(0.05)
"""


def test_clock_sampler_brackets_a_short_region(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(FAKE.format(py=sys.executable))
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.005)   # the timed region
    r = c.stop()
    assert r is not None and r["samples"] >= 2
    assert r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))   # nothing to run
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    c.start()
    assert c.stop() is None


def test_traffic_is_read_only_for_the_profiled_source(tmp_path, monkeypatch):
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    prof = tmp_path / "profiles" / "markov_gemm_qwen3_4b.txt"
    prof.write_text(f"# summary\nsource_sha256_16: {sha}\ndram_bytes_per_launch: 80091904\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profile(str(src)) == 80091904.0
    src.write_text("// kernel v2\n")          # the kernel changed since the capture
    assert bench.traffic_from_profile(str(src)) is None
    prof.unlink()
    assert bench.traffic_from_profile(str(src)) is None
