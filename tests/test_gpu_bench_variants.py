"""bench.py's variant methods run end to end and print one well-formed JSON
line (the default method is exercised by the benchmark itself)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("extra", [["--method", "decode", "--decode-shape", "2,8,4096,128"],
                                   ["--method", "index"],
                                   ["--p-levels", "255"],
                                   ["--q-path", "fused"]],
                         ids=["decode", "index", "pcodes", "fused_q"])
def test_bench_variant_line(extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
           "--no-e2e", "--no-repeats", "--no-configs", *extra]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["value"] > 0 and line["steps"] == 3 and line["gpu_launches"] > 0
    assert line["roofline"]["frac"] > 0
