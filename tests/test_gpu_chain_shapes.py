"""The M = 32768 block chain's own GEMM shapes on the INT8 path: the concatenated QKV
projection (K = 4096 -> N = 12288) and the MLP down projection (K = 16384 -> N = 4096),
with the chain's weights and 1024 rows of N(0, 1) activations: activation and weight
codes and scales and a slice of the INT32 block sums bit for bit, outputs on a row slice
and on sampled points within tolerance, all against the oracle on its own codes."""
import numpy as np
import pytest

import block_wise_w8a8_b200 as w8
from gpu_util import assert_close_bf16, assert_codes_equal, dev_bf16, host_bits
from synth import workload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


@pytest.mark.parametrize("which", ["qkv", "down"])
def test_chain_projection_shape(orc, which):
    wl = workload("hires_chain_32768")
    lin = next(l for l in wl.linears if l["name"] == which)
    M, K, N = 1024, lin["K"], lin["N"]
    x, w = wl.x(M, K), wl.w(lin)
    wt = w8.W8A8Weight(dev_bf16(w))
    y, path = w8.linear(dev_bf16(x), wt, None, return_path=True)
    assert path == w8.PATH_INT8
    yb = host_bits(y)
    xq, xs = orc.block_quantize(x)
    wq, ws = orc.block_quantize(w)
    assert_codes_equal(wt.wq, wt.ws, wq, ws, "weight")
    gq, gs = w8.quantize_act(dev_bf16(x))
    assert_codes_equal(gq, gs, xq, xs, "activations")
    # INT32 block sums of a 128-row x 256-column corner, at the full K
    sums = w8.debug_block_sums(gq[:128].contiguous(), wt.wq[:256].contiguous())
    np.testing.assert_array_equal(sums.cpu().numpy(), orc.block_sums(xq[:128], wq[:256]))
    assert_close_bf16(yb[896:], orc.w8a8_linear(xq, xs, wq, ws, None, m0=896, rows=128), orc, "rows")
    r = np.random.default_rng(11)
    ms, ns = r.integers(0, M, 2048), r.integers(0, N, 2048)
    assert_close_bf16(yb[ms, ns], orc.w8a8_linear_at(xq, xs, wq, ws, None, ms, ns), orc, "sampled")
