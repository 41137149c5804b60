"""The per-row / per-output-channel post-scale W8A8 operator (TurboT2VA paper, W8A8
operator paragraph) on the GPU, through the C ABI, against the oracle.

Codes and scales must be bit-exact.  The oracle quantizes x and w itself and its linear
runs on its own codes.  The kernel's epilogue performs the oracle's FP32 operations in
the oracle's order (the INT32 sum rounded to FP32, the scale product, the product, the
bias, one rounding each, no fused multiply-add), so its BF16 outputs must equal the
oracle's FP32 outputs rounded to BF16 bit for bit; the tolerance bar of the block-wise
path (1e-2 + 1e-2 |ref|) is checked as well."""
import numpy as np
import pytest
import torch

import block_wise_w8a8_b200 as w8
from gpu_util import assert_close_bf16, assert_codes_equal, dev_bf16, host_bits
from synth import f64_to_bf16_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def _rows(shape, seed):
    """Heavy-tailed rows over very different magnitudes, plus an all-zero row, a row
    below the 1e-4 floor and rows with exact half-integer quotients."""
    r = np.random.default_rng(seed)
    x = r.standard_t(3, shape) * np.exp(r.uniform(-6, 6, (shape[0], 1)))
    x[0] = 0.0
    if shape[0] > 1:
        x[1] = r.uniform(-1, 1, shape[1]) * 3e-5
    if shape[0] > 3:
        x[2] = np.round(r.uniform(-126, 125, shape[1])) + 0.5      # s = 1: x / s = k + 1/2
        x[2, 0] = 127.0
    return f64_to_bf16_bits(x)


@pytest.mark.parametrize("rows,K", [(1, 8), (2, 24), (37, 1000), (256, 4096), (130, 16384)])
def test_rowwise_quantize_bit_exact(orc, rows, K):
    x = _rows((rows, K), rows + K)
    q, s = w8.rowwise_quantize(dev_bf16(x))
    q_ref, s_ref = orc.row_quantize(x)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)


def _check_linear(orc, x, w, b, what):
    xq, xs = w8.rowwise_quantize(dev_bf16(x))
    wq, ws = w8.rowwise_quantize(dev_bf16(w))
    y = w8.rowwise_linear_prequant(xq, xs, wq, ws, None if b is None else dev_bf16(b))
    xq_ref, xs_ref = orc.row_quantize(x)
    wq_ref, ws_ref = orc.row_quantize(w)
    assert_codes_equal(xq, xs, xq_ref, xs_ref, f"{what} x")
    assert_codes_equal(wq, ws, wq_ref, ws_ref, f"{what} w")
    ref = orc.row_linear(xq_ref, xs_ref, wq_ref, ws_ref, b)
    yb = host_bits(y)
    np.testing.assert_array_equal(yb, orc.f32_to_bf16(ref), err_msg=what)
    assert_close_bf16(yb, ref, orc, what)


@pytest.mark.parametrize("M,K,N,bias", [(128, 128, 128, True), (256, 384, 640, False),
                                        (384, 1024, 256, True), (128, 2048, 384, True)])
def test_rowwise_linear_small(orc, M, K, N, bias):
    r = np.random.default_rng(M * 3 + K + N)
    x = _rows((M, K), M + K)
    w = f64_to_bf16_bits(r.standard_normal((N, K)) * 0.05)
    b = f64_to_bf16_bits(r.standard_normal(N) * 0.1) if bias else None
    _check_linear(orc, x, w, b, f"{M}x{K}x{N}")


def test_rowwise_int32_sum_rounding(orc):
    """INT32 sums 2^24 + 1 (rounds to 2^24) with unit scales, padded to a 128 multiple."""
    K, M, N = 1152, 128, 128
    x = np.zeros((M, K))
    w = np.zeros((N, K))
    x[:, :1041] = 127
    x[:, 1041] = 9
    w[:, :1040] = 127
    w[:, 1040] = 24
    w[:, 1041] = 1
    xq, xs = w8.rowwise_quantize(dev_bf16(f64_to_bf16_bits(x)))
    wq, ws = w8.rowwise_quantize(dev_bf16(f64_to_bf16_bits(w)))
    y = w8.rowwise_linear_prequant(xq, xs, wq, ws)
    assert torch.all(y.float() == 2.0 ** 24)


def test_rowwise_linear_attn_proj_4096(orc):
    """The 4096^3 workload: codes and scales of all 4096 activation rows and all weight
    rows, outputs on a 128-row strip and at 4096 sampled points, against the oracle on its
    own codes."""
    wl = workload("attn_proj_4096")
    lin = wl.linears[0]
    xb = wl.x(4096, 4096)
    wb = wl.w(lin)
    xq, xs = w8.rowwise_quantize(dev_bf16(xb))
    wq, ws = w8.rowwise_quantize(dev_bf16(wb))
    q_ref, s_ref = orc.row_quantize(xb)
    assert_codes_equal(xq, xs, q_ref, s_ref, "x")
    wq_ref, ws_ref = orc.row_quantize(wb)
    assert_codes_equal(wq, ws, wq_ref, ws_ref, "w")
    y = host_bits(w8.rowwise_linear_prequant(xq, xs, wq, ws))
    r = np.random.default_rng(7)
    ms, ns = r.integers(0, 4096, 4096), r.integers(0, 4096, 4096)
    ref = orc.row_linear_at(q_ref, s_ref, wq_ref, ws_ref, None, ms, ns)
    np.testing.assert_array_equal(y[ms, ns], orc.f32_to_bf16(ref))
    ref = orc.row_linear(q_ref, s_ref, wq_ref, ws_ref, None, m0=1920, rows=128)
    np.testing.assert_array_equal(y[1920:2048], orc.f32_to_bf16(ref))


def test_rowwise_errors():
    L = w8.lib()
    st = w8._stream(torch.device("cuda"))
    x = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((256, 256), dtype=torch.int8, device="cuda")
    s = torch.empty((256,), dtype=torch.float32, device="cuda")
    assert L.w8a8_rowwise_quantize(x.data_ptr(), 256, 252, q.data_ptr(), s.data_ptr(), st) == 2
    assert L.w8a8_rowwise_quantize(x.data_ptr() + 2, 128, 128, q.data_ptr(), s.data_ptr(), st) == 4
    host = torch.zeros((256, 256), dtype=torch.bfloat16)
    assert L.w8a8_rowwise_quantize(host.data_ptr(), 256, 256, q.data_ptr(), s.data_ptr(), st) == 3
    y = torch.empty((256, 256), dtype=torch.bfloat16, device="cuda")
    assert L.w8a8_rowwise_linear(q.data_ptr(), s.data_ptr(), 256, 200, q.data_ptr(), s.data_ptr(),
                                 256, None, y.data_ptr(), st) == 2
    assert L.w8a8_rowwise_linear(q.data_ptr(), s.data_ptr(), 256, 256, q.data_ptr(), s.data_ptr(),
                                 256, None, y.data_ptr() + 2, st) == 4
