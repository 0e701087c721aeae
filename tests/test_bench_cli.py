"""bench.py's command line on CPU: bad flag combinations stop before any device work."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("args,needle", [
    (["--workload", "hf_repro_n64", "--tail", "64"], "--tail must be in (0, N)"),   # N = 64
    (["--tail", "2048"], "--tail must be in (0, N)"),       # the default workload has N = 2048
    (["--tail", "-3"], "--tail must be in (0, N)"),
    (["--warmup", "2"], "--warmup must be >= 3"),
    (["--workload", "no_such_workload"], "invalid choice"),
    (["--segment-len", "100"], "--segment-len must be"),
])
def test_bench_rejects_bad_flags(args, needle):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 2
    assert needle in r.stderr


def test_tensor_peak_follows_the_power_cap():
    """A tensor-bound kernel is held to the sustained bf16 figure only when the clock record
    of its timed region shows sw_power_cap active; otherwise (no reason, other reasons, no
    NVML, no sustained figure) to the burst one."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1665.9, "bf16_tflops_sustained": 1414.4, "hbm_gbs": 6544.0}
    assert bench.tensor_peak(peaks, {"reasons": ["sw_power_cap"]})[0] == 1414.4
    assert bench.tensor_peak(peaks, {"reasons": ["sw_power_cap", "sync_boost"]})[0] == 1414.4
    assert bench.tensor_peak(peaks, {"reasons": []}) == (1665.9, "burst")
    assert bench.tensor_peak(peaks, {"reasons": ["sync_boost"]})[0] == 1665.9
    assert bench.tensor_peak(peaks, {"reasons": None})[0] == 1665.9
    assert bench.tensor_peak(peaks, None)[0] == 1665.9
    no_sustained = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}
    assert bench.tensor_peak(no_sustained, {"reasons": ["sw_power_cap"]})[0] == 1590.0


def test_captured_traffic_is_dropped_once_the_kernel_changes():
    """The bench line's roofline.traffic comes from an ncu capture recorded with a digest of
    the kernel's sources: a matching digest gives the bytes, a changed one (the kernel was
    edited after the capture) or a missing entry gives None."""
    sys.path.insert(0, ROOT)
    import bench
    key = ("test_workload", "segment_tc")
    try:
        bench.NCU_TRAFFIC_BYTES[key] = (123456, bench.kernel_digest("segment_tc"))
        assert bench.captured_traffic(*key)[0] == 123456
        bench.NCU_TRAFFIC_BYTES[key] = (123456, "0" * 16)
        byts, note = bench.captured_traffic(*key)
        assert byts is None and note.startswith("stale")
    finally:
        bench.NCU_TRAFFIC_BYTES.pop(key, None)
    assert bench.captured_traffic(*key)[0] is None
    assert bench.kernel_digest("no_such_kernel") is None
