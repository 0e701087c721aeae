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
