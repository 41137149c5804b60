"""The gated residual update fused into the block-wise W8A8 GEMM's epilogue (TurboT2VA
paper, fused-operator paragraph), on the GPU through the C ABI, against the oracle:
out = bf16(fl(r + fl(gate[m / T, n] * v))) with v the FP32 linear output.

The oracle quantizes x and w itself and runs the linear and the gated update on its own
codes; the GPU's codes and scales must equal the oracle's bit for bit (so both sides
multiply the same integers), and the outputs are compared with the tolerance of the
linear layer (1e-2 + 1e-2 |ref|).  The gate and residual arithmetic itself is checked
exactly through special cases (gate 0 gives the residual, gate 1 on a zero residual gives
the plain linear's bits) and in-place use (out aliasing the residual)."""
import numpy as np
import pytest
import torch

import block_wise_w8a8_b200 as w8
from gpu_util import assert_close_bf16, assert_codes_equal, bf16_to_f32, dev_bf16, host_bits
from synth import f64_to_bf16_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def _case(M, K, N, T, seed, with_bias=True):
    r = np.random.default_rng(seed)
    x = f64_to_bf16_bits(np.clip(r.standard_t(3, (M, K)), -64, 64))
    w = f64_to_bf16_bits(r.standard_normal((N, K)) * 0.05)
    b = f64_to_bf16_bits(r.standard_normal(N) * 0.1) if with_bias else None
    res = f64_to_bf16_bits(r.standard_normal((M, N)))
    g = f64_to_bf16_bits(r.standard_normal((M // T, N)) * 0.5)
    return x, w, b, res, g


@pytest.mark.parametrize("M,K,N,T,with_bias", [(128, 128, 128, 128, True),
                                               (256, 384, 256, 128, False),
                                               (384, 1024, 640, 384, True),
                                               (256, 256, 384, 1, True),      # per-row gate
                                               (640, 512, 256, 64, False)])   # T below a block
def test_gated_small(orc, M, K, N, T, with_bias):
    x, w, b, res, g = _case(M, K, N, T, M + K + N + T, with_bias)
    wt = w8.W8A8Weight(dev_bf16(w))
    xq, xs = w8.quantize_act(dev_bf16(x))
    out = w8.linear_prequant_gated(xq, xs, wt, dev_bf16(res), dev_bf16(g),
                                   None if b is None else dev_bf16(b))
    xq_ref, xs_ref = orc.block_quantize(x)
    wq_ref, ws_ref = orc.block_quantize(w)
    assert_codes_equal(xq, xs, xq_ref, xs_ref, "x")
    assert_codes_equal(wt.wq, wt.ws, wq_ref, ws_ref, "w")
    v = orc.w8a8_linear(xq_ref, xs_ref, wq_ref, ws_ref, b)
    ref = orc.gated_residual(v, res, g, T, M)
    assert_close_bf16(host_bits(out), bf16_to_f32(ref), orc, f"gated {M}x{K}x{N} T={T}")
    # in place: the residual buffer itself receives the update, same bits
    rd = dev_bf16(res)
    w8.linear_prequant_gated(xq, xs, wt, rd, dev_bf16(g), None if b is None else dev_bf16(b), out=rd)
    np.testing.assert_array_equal(host_bits(rd), host_bits(out))


def test_gated_special_cases(orc):
    M, K, N = 256, 512, 384
    x, w, b, res, _ = _case(M, K, N, M, 3)
    wt = w8.W8A8Weight(dev_bf16(w))
    xq, xs = w8.quantize_act(dev_bf16(x))
    bd = dev_bf16(b)
    plain = host_bits(w8.linear_prequant(xq, xs, wt, bd))
    ones = dev_bf16(f64_to_bf16_bits(np.ones((1, N))))
    zeros_r = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    # gate 1, residual 0: fl(0 + fl(1 * v)) = v, so the plain linear's bits
    np.testing.assert_array_equal(host_bits(w8.linear_prequant_gated(xq, xs, wt, zeros_r, ones, bd)),
                                  plain)
    # gate 0: the residual (up to the sign of zero)
    zg = torch.zeros((2, N), dtype=torch.bfloat16, device="cuda")
    got = host_bits(w8.linear_prequant_gated(xq, xs, wt, dev_bf16(res), zg, bd))
    np.testing.assert_array_equal(got & 0x7FFF, res & 0x7FFF)


def test_gated_hires_out_projection_sampled(orc):
    """The M = 32768 chain's out projection (K = N = 4096) as a gated residual update,
    one sample (T = M): 4096 sampled outputs against the oracle."""
    wl = workload("hires_chain_32768")
    lin = [l for l in wl.linears if l["name"] == "out"][0]
    M, K, N = lin["M"], lin["K"], lin["N"]
    x = wl.x(M, K)
    w = wl.w(lin)
    res = wl.residual(M, N)
    g = wl.gate(1, N)
    wt = w8.W8A8Weight(dev_bf16(w))
    xq, xs = w8.quantize_act(dev_bf16(x))
    out = host_bits(w8.linear_prequant_gated(xq, xs, wt, dev_bf16(res), dev_bf16(g)))
    # all 32768 x 4096 activation codes and the whole weight, against the oracle's own
    xq_ref, xs_ref = orc.block_quantize(x)
    wq_ref, ws_ref = orc.block_quantize(w)
    assert_codes_equal(xq, xs, xq_ref, xs_ref, "x")
    assert_codes_equal(wt.wq, wt.ws, wq_ref, ws_ref, "w")
    r = np.random.default_rng(11)
    ms, ns = r.integers(0, M, 4096), r.integers(0, N, 4096)
    v = orc.w8a8_linear_at(xq_ref, xs_ref, wq_ref, ws_ref, None, ms, ns)
    ref = orc.gated_residual(v, res[ms, ns], g, M, M, ms, ns)
    assert_close_bf16(out[ms, ns], bf16_to_f32(ref), orc, "gated out projection (sampled)")
    # and one whole 128-row strip
    rows = slice(128 * 200, 128 * 201)
    v = orc.w8a8_linear(xq_ref, xs_ref, wq_ref, ws_ref, None, m0=128 * 200, rows=128)
    ref = orc.gated_residual(v, res[rows], g, M, M, np.repeat(np.arange(128 * 200, 128 * 201), N),
                             np.tile(np.arange(N), 128))
    assert_close_bf16(out[rows].reshape(-1), bf16_to_f32(ref).reshape(-1), orc,
                      "gated out projection (strip 200)")


def test_gated_errors():
    L = w8.lib()
    st = w8._stream(torch.device("cuda"))
    xq = torch.zeros((256, 256), dtype=torch.int8, device="cuda")
    xs = torch.ones((2, 2), dtype=torch.float32, device="cuda")
    wt = w8.W8A8Weight(torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda"))
    r = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((2, 256), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((256, 256), dtype=torch.bfloat16, device="cuda")
    f = L.w8a8_linear_prequant_gated
    P = lambda t: t.data_ptr()
    assert f(P(xq), P(xs), 256, 256, wt.record(), None, P(r), P(g), 128, P(y), st) == 0
    assert f(P(xq), P(xs), 256, 256, wt.record(), None, P(r), P(g), 0, P(y), st) == 1
    assert f(P(xq), P(xs), 256, 256, wt.record(), None, P(r), P(g), 96, P(y), st) == 2
    assert f(P(xq), P(xs), 256, 256, wt.record(), None, P(r) + 2, P(g), 128, P(y), st) == 4
    host = torch.zeros((2, 256), dtype=torch.bfloat16)
    assert f(P(xq), P(xs), 256, 256, wt.record(), None, P(r), P(host), 128, P(y), st) == 3
    assert f(P(xq), P(xs), 256, 256, wt.record(), None, None, P(g), 128, P(y), st) == 1
    torch.cuda.synchronize()
