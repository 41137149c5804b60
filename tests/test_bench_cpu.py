"""bench.py's host-side pieces, without a GPU: the peak table, the ncu traffic lookup
and the reference arm (the CPU oracle) end to end, with its JSON line."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_peaks_and_traffic():
    pk = bench._peaks()
    assert pk["hbm"] > 1000 and pk["bf16"] > 100 and pk["source"] in ("measured", "fallback")
    for kernel in bench.KERNEL_DEVICE_SOURCES:
        t = bench._traffic(kernel)
        assert t is None or t > 0


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == bench.UNIT
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
