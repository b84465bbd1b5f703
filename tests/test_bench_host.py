"""Host-side pieces of bench.py that the reported numbers rest on, checked on the CPU.

- The roofline bound follows each configuration's arithmetic intensity against
  the ridge of the peaks in use: tensor for 4096^3, 8192^3 and the first two
  ragged shapes, HBM for the small-M shapes and (8191, 129, 8193).
- The fraction is the achieved rate over the peak, from the algorithmic flops
  or bytes and the kernel time.
- Without MEASURED_PEAKS.json the recipe's fallback peaks are used, and say so.
- A committed profile's DRAM traffic is used only for its own path and
  workload, and only while the kernel sources hash to the recorded value.
"""
import json
import os

import pytest

import bench
from tiled_dense_gemm_fp16_b200 import inputs

PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


@pytest.mark.parametrize("M,N,K,bound", [
    (4096, 4096, 4096, "tensor"), (8192, 8192, 8192, "tensor"),
    (3001, 5003, 1021, "tensor"), (777, 12289, 4095, "tensor"),
    (1, 8192, 8192, "hbm"), (16, 8192, 8192, "hbm"), (64, 8192, 8192, "hbm"),
    (8191, 129, 8193, "hbm"), (256, 256, 256, "hbm"),
])
def test_roofline_bound_follows_arithmetic_intensity(M, N, K, bound):
    rec = bench.roofline_for(M, N, K, 1.0, PEAKS, "fallback")
    assert rec["bound"] == bound
    intensity = 2 * M * N * K / (2 * (M * K + K * N + M * N))
    assert rec["intensity_flop_per_byte"] == pytest.approx(intensity)
    assert rec["ridge_flop_per_byte"] == pytest.approx(1590e12 / 6650e9)


def test_roofline_fraction_is_achieved_over_peak():
    # 8192^3 in 0.7 ms: 1.0995e12 flop / 7e-4 s = 1570.8 TFLOP/s.
    rec = bench.roofline_for(8192, 8192, 8192, 0.7, PEAKS, "fallback")
    assert rec["achieved"] == pytest.approx(2 * 8192 ** 3 / 0.7e-3 / 1e12)
    assert rec["frac"] == pytest.approx(rec["achieved"] / 1590.0)
    assert rec["unit"] == "TFLOP/s" and "fallback" in rec["peak_source"]
    # M = 16 in 25 us: 2(MK + KN + MN) bytes over the time, against the copy bandwidth.
    rec = bench.roofline_for(16, 8192, 8192, 0.025, PEAKS, "fallback")
    nbytes = 2 * (16 * 8192 + 8192 * 8192 + 16 * 8192)
    assert nbytes == inputs.min_bytes(16, 8192, 8192)
    assert rec["achieved"] == pytest.approx(nbytes / 25e-6 / 1e9)
    assert rec["unit"] == "GB/s" and rec["frac"] == pytest.approx(rec["achieved"] / 6650.0)
    # The sustained record takes the sustained tensor peak.
    rec = bench.roofline_for(8192, 8192, 8192, 0.8, PEAKS, "fallback", sustained=True)
    assert rec["peak"] == 1400.0 and "sustained" in rec["peak_source"]


def test_fallback_peaks_without_the_measured_file(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback"
    assert peaks["bf16_tflops"] == pytest.approx(1590.0) and peaks["hbm_gbs"] == pytest.approx(6650.0)
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1656.9, "hbm_gbs": 6431.7}))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["bf16_tflops"] == pytest.approx(1656.9)


def test_committed_traffic_is_keyed_by_path_workload_and_source_hash(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    sha = bench.kernel_source_sha("skinny")
    body = f"kernel_source_sha: {sha}\ntraffic_workload: skinny:16\ntraffic_bytes_per_launch: 138044672\n"
    (tmp_path / "gemm_relu_skinny_skinny_m16.md").write_text(body)
    assert bench.committed_traffic("skinny", "skinny:16") == 138044672.0
    assert bench.committed_traffic("skinny", "skinny:64") is None          # no summary for that workload
    assert bench.committed_traffic("tc_pair512", "skinny:16") is None      # another path
    (tmp_path / "gemm_relu_skinny_skinny_m16.md").write_text(body.replace(sha, "0" * 16))
    assert bench.committed_traffic("skinny", "skinny:16") is None          # kernel changed since the capture
    (tmp_path / "gemm_relu_skinny_skinny_m16.md").write_text(body.replace("skinny:16\n", "skinny:1\n"))
    assert bench.committed_traffic("skinny", "skinny:16") is None          # figures of another workload


def test_committed_profiles_name_their_workload_and_hash():
    """Every committed summary that bench.py reads carries the three machine-read keys."""
    found = 0
    for name in sorted(os.listdir(bench.PROFILES)):
        if not name.startswith("gemm_relu_") or not name.endswith(".md"):
            continue
        text = open(os.path.join(bench.PROFILES, name)).read()
        if "traffic_bytes_per_launch" not in text:
            continue
        found += 1
        for key in ("kernel_source_sha:", "traffic_workload:", "traffic_bytes_per_launch:"):
            assert key in text, (name, key)
    assert found >= 10
