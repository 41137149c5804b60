"""The near-tie sweep's inputs (tests/norm_sweep.py) do what the GPU test relies on, checked
with the oracle on the CPU: rstd is exactly 1.0, the normalised values equal the inputs,
each sweep block holds every BF16 value of [A/512, A] of both signs and has absmax A."""
import numpy as np
import pytest

from norm_sweep import ABSMAXES, sweep_block, unit_rms_rows
from synth import bf16_bits_to_f32


@pytest.mark.parametrize("eps", [0.0, 1e-6])
def test_unit_rms_rows(orc, eps):
    K = 4096
    x = unit_rms_rows(K, eps)
    y, rstd = orc.rmsnorm(x, np.full(K, 0x3F80, np.uint16), eps)
    assert np.all(rstd == 1.0)
    np.testing.assert_array_equal(y, x)
    z = np.zeros((1, K), np.uint16)
    y2, rstd2 = orc.mod_rmsnorm(x, None, z, z, x.shape[0], eps)
    assert np.all(rstd2 == 1.0)
    np.testing.assert_array_equal(y2, x)


def test_sweep_blocks_cover_every_value():
    for A in ABSMAXES:
        blk = sweep_block(A)
        v = bf16_bits_to_f32(blk).astype(np.float64)
        assert np.abs(v).max() == A
        lo = int(np.array([A / 512], np.float32).view(np.uint32)[0] >> 16)
        hi = int(np.array([A], np.float32).view(np.uint32)[0] >> 16)
        want = set(range(lo, hi + 1)) | {b | 0x8000 for b in range(lo, hi + 1)}
        assert set(np.unique(blk).tolist()) == want
