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
import datetime, time
while True:
    ts = datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    print("0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Active, " + ts,
          flush=True)
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
    t0 = time.time()
    time.sleep(0.005)   # the timed region
    r = c.stop((t0, time.time()))
    assert r is not None and r["samples"] >= 2
    assert r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    # shorter than the sampling interval: the samples around it stand in
    assert r["window"] in ("bracketing", "region")


def test_clock_summary_keeps_only_the_region():
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    base = datetime.datetime(2026, 1, 1, 12, 0, 0)
    line = lambda s, mhz, cap: (f"0, {mhz}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, "
                                f"{cap}, " + (base + datetime.timedelta(seconds=s)).strftime(
                                    "%Y/%m/%d %H:%M:%S.%f")[:-3])
    lines = [line(0.0, 1200, "Active"), line(0.5, 1965, "Not Active"), line(0.6, 1965, "Not Active"),
             line(1.5, 1100, "Active")]
    t = lambda s: (base + datetime.timedelta(seconds=s)).timestamp()
    r = bench.summarise_clocks(lines, (t(0.4), t(0.7)))
    # the throttled samples outside the region do not count
    assert r["window"] == "region" and r["samples_in_region"] == 2
    assert r["sm_mhz"] == 1965.0 and r["reasons"] == []
    r = bench.summarise_clocks(lines, (t(0.7), t(0.8)))   # no sample inside
    assert r["window"] == "bracketing" and r["samples_in_region"] == 0
    assert r["sm_mhz"] == (1965.0 + 1100.0) / 2 and r["reasons"] == ["sw_power_cap"]


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
    name = "markov_gemm_qwen3_4b.txt"
    assert bench.traffic_from_profile(str(src), name) == 80091904.0
    src.write_text("// kernel v2\n")          # the kernel changed since the capture
    assert bench.traffic_from_profile(str(src), name) is None
    prof.unlink()
    assert bench.traffic_from_profile(str(src), name) is None
    # each kernel source has its own summary
    assert bench.PROFILE_OF["pbuild.cu"] == "pbuild_qwen3_4b.txt"


def test_build_roofline_counts_bm_once_and_reports_the_stream():
    """The roofline charges the Markov factor once per build; the stream
    object counts one pass over it per wave."""
    sys.path.insert(0, ROOT)
    import bench
    kern = {"pbuild": {"avg_us": 100.0}}
    V, r = 1000, 64
    roof = bench.build_roofline(kern, V=V, r=r, B=2, Bk=5, inner=9, lbytes=2, waves=4)
    assert roof["algorithmic_bytes_per_launch"] == V * r * 2 + 2 * 5 * V * 2 + 9 * r * 2
    assert roof["stream"]["bytes_per_launch"] == 4 * V * r * 2
    assert abs(roof["stream"]["achieved_gbs"] - 4 * V * r * 2 / 100e-6 / 1e9) < 0.1
    assert "stream" not in bench.build_roofline({"markov_gemm": {"avg_us": 10.0}}, V=V, r=r,
                                                B=2, Bk=5, inner=9, lbytes=2, waves=4)


def test_round_roofline_sums_the_three_calls():
    """Round roofline: build + verify + accept bytes (and flops where they
    bind) at the peak; the headline shape gives ~99 MB per round."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    V, r = 151936, 256
    build_bytes = V * r * 2 + 7 * V * 2 + 27 * r * 2
    rr = bench.round_roofline(1000.0, 1, build_bytes=build_bytes, build_flops=2.0 * 27 * V * r,
                              prefix_lens=np.array([2048]), n_nodes=np.array([32]), inner=27,
                              V=V, Hq=32, Hkv=8, d=128, tbytes=2, temp=0.0)
    kv = (2048 + 33) * 8 * 128 * 2 * 2
    qo = 33 * 32 * 128 * 2 * 2
    assert rr["bytes_per_round"] == build_bytes + kv + qo + 33 * V * 2
    pk, _ = bench.peaks()
    t = rr["bytes_per_round"] / (pk["hbm_gbs"] * 1e9)
    assert abs(rr["rounds_per_s_at_roofline"] - 1.0 / t) / (1.0 / t) < 1e-3
    assert abs(rr["frac"] - 1000.0 * t) < 1e-3
    # at T > 0 the build also writes its fp32 q rows; two GPUs double the job rate
    r2 = bench.round_roofline(2000.0, 2, build_bytes=build_bytes, build_flops=0.0,
                              prefix_lens=np.array([2048]), n_nodes=np.array([32]), inner=27,
                              V=V, Hq=32, Hkv=8, d=128, tbytes=2, temp=0.6)
    assert r2["bytes_per_round"] == rr["bytes_per_round"] + 27 * V * 4
    assert r2["frac"] > rr["frac"]
