"""The CPU oracle against its pins (closed forms, exact rationals, brute force,
invariants) and against the hand-derived golden cases.  No GPU."""
import os
import subprocess
import sys

import numpy as np
import pytest

import pins
from synth import bf16_bits_to_f32, f64_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    return rows


def test_golden_block_cases(orc):
    rows = _golden_rows("block_quant_cases.txt")
    assert len(rows) >= 10
    for r in rows:
        absmax, x, scale, code_x, code_a = float(r[0]), float(r[1]), float(r[2]), int(r[3]), int(r[4])
        blk = np.zeros((128, 128))
        blk[0, 0] = absmax
        blk[5, 9] = x
        bits = f64_to_bf16_bits(blk)
        assert bf16_bits_to_f32(bits)[5, 9] == x and bf16_bits_to_f32(bits)[0, 0] == absmax
        q, s = orc.block_quantize(bits)
        assert s[0, 0] == np.float32(scale), r
        assert q[5, 9] == code_x, r
        assert q[0, 0] == code_a, r


def test_thread_count_does_not_change_bits(orc, tmp_path):
    """OpenMP splits only independent outputs: one thread gives the same bits."""
    code = r'''
import sys, hashlib, numpy as np
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import oracle
from synth import workload
o = oracle.default()
w = workload("linear_256"); lin = w.linears[0]
xq, xs = o.block_quantize(w.x(256, 256)); wq, ws = o.block_quantize(w.w(lin))
y = o.w8a8_linear(xq, xs, wq, ws, w.bias(lin))
g = w.gamma(256); yn, r = o.rmsnorm(w.x(256, 256), g, 1e-6)
h = hashlib.sha256(xq.tobytes() + xs.tobytes() + y.tobytes() + yn.tobytes() + r.tobytes())
print(o.num_threads(), h.hexdigest())
'''
    root = os.path.dirname(GOLDEN.rstrip("/")).rsplit("/", 1)[0]
    outs = []
    for nt in ("1", "4"):
        env = dict(os.environ, OMP_NUM_THREADS=nt)
        p = subprocess.run([sys.executable, "-c", code, root], env=env, capture_output=True,
                           text=True, check=True)
        outs.append(p.stdout.split())
    assert outs[0][0] == "1" and outs[1][0] == "4"
    assert outs[0][1] == outs[1][1]
