"""The INT8 path at its largest reduction length and just past it.  K = 65536 is 512 K
blocks, which fills the GEMM's per-tile scale tables exactly; K = 65664 fails the guard
(K <= 65536) and must take the BF16 GEMM on the retained weight."""
import numpy as np
import pytest

import block_wise_w8a8_b200 as w8
from gpu_util import assert_close_bf16, dev_bf16, host_bits
from synth import f64_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def _bits(shape, seed, scale=1.0):
    return f64_to_bf16_bits(np.random.default_rng(seed).standard_normal(shape) * scale)


def test_int8_path_at_the_largest_k(orc):
    M, K, N = 128, 65536, 256
    x, w, b = _bits((M, K), 71), _bits((N, K), 72, K ** -0.5), _bits((N,), 73, 0.1)
    wt = w8.W8A8Weight(dev_bf16(w))
    y, path = w8.linear(dev_bf16(x), wt, dev_bf16(b), return_path=True)
    assert path == w8.PATH_INT8
    xq, xs = orc.block_quantize(x)
    wq, ws = orc.block_quantize(w)
    assert np.array_equal(host_bits(wt.wq).view(np.int8), wq)
    assert_close_bf16(host_bits(y), orc.w8a8_linear(xq, xs, wq, ws, b), orc, "K = 65536")


def test_guard_takes_bf16_past_the_largest_k(orc):
    M, K, N = 128, 65536 + 128, 128
    x, w = _bits((M, K), 74), _bits((N, K), 75, K ** -0.5)
    wt = w8.W8A8Weight(dev_bf16(w))
    y, path = w8.linear(dev_bf16(x), wt, None, return_path=True)
    assert path == w8.PATH_BF16
    assert_close_bf16(host_bits(y), orc.bf16_linear(x, w, None), orc, "K = 65664")
