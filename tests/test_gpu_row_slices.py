"""Row slices: every step of the path treats 128-row blocks of the activation on their own,
so calling the library on a 128-aligned slice of the rows gives exactly the rows of the
call on the whole input.  A caller that streams its batch through in row chunks (as the
M = 32768 chain's end-to-end benchmark leg does, overlapping its host copies with the
compute) relies on that.

Checked bit for bit: the block quantizer's codes and scales, the linear's BF16 output
(INT8 path and BF16 fallback), and the RMSNorm + quantizer within one of its two forms.
Across the two forms (a slice below 192 rows per SM takes the one-grid form, the whole
input above it the two-grid form) rstd may differ by one FP32 ulp on rare rows; the
codes and scales must agree on every 128-row strip whose rstd all agree."""
import numpy as np
import pytest
import torch

import block_wise_w8a8_b200 as w8
from gpu_util import dev_bf16
from synth import f64_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def _bits(shape, seed, scale=1.0):
    r = np.random.default_rng(seed)
    return f64_to_bf16_bits(r.standard_t(3, shape).clip(-64, 64) * scale)


def _eq(a, b):
    return torch.equal(a.contiguous().view(torch.int16) if a.dtype == torch.bfloat16 else a,
                       b.contiguous().view(torch.int16) if b.dtype == torch.bfloat16 else b)


SLICES = [(0, 128), (128, 512), (512, 1408), (1408, 1536)]


def test_quantize_act_row_slices():
    x = dev_bf16(_bits((1536, 1024), 1))
    q, s = w8.quantize_act(x)
    for r0, r1 in SLICES:
        qs, ss = w8.quantize_act(x[r0:r1])
        assert torch.equal(qs, q[r0:r1])
        assert torch.equal(ss.view(torch.int32), s[r0 // 128:r1 // 128].view(torch.int32))


@pytest.mark.parametrize("K,N,with_bias", [(1024, 768, True), (2048, 384, False)])
def test_linear_row_slices(K, N, with_bias):
    x = dev_bf16(_bits((1536, K), K))
    wt = w8.W8A8Weight(dev_bf16(_bits((N, K), N, 0.05)))
    b = dev_bf16(_bits((N,), 7, 0.1)) if with_bias else None
    y, path = w8.linear(x, wt, b, return_path=True)
    assert path == w8.PATH_INT8
    for r0, r1 in SLICES:
        ys, ps = w8.linear(x[r0:r1], wt, b, return_path=True)
        assert ps == w8.PATH_INT8
        assert _eq(ys, y[r0:r1]), (r0, r1)


def test_bf16_fallback_row_slices():
    """K = 2000 takes the BF16 GEMM for the whole input and for every slice."""
    x = dev_bf16(_bits((640, 2000), 3))
    wt = w8.W8A8Weight(dev_bf16(_bits((512, 2000), 4, 0.05)))
    y, path = w8.linear(x, wt, None, return_path=True)
    assert path == w8.PATH_BF16
    for r0, r1 in [(0, 128), (128, 640)]:
        ys, ps = w8.linear(x[r0:r1], wt, None, return_path=True)
        assert ps == w8.PATH_BF16
        assert _eq(ys, y[r0:r1])


def test_rmsnorm_row_slices_one_form():
    x = dev_bf16(_bits((1536, 4096), 5))
    g = dev_bf16(f64_to_bf16_bits(np.random.default_rng(6).uniform(0.5, 1.5, 4096)))
    q, s, r = w8.rmsnorm_quantize_act(x, g, 1e-6)
    for r0, r1 in SLICES:
        qs, ss, rs = w8.rmsnorm_quantize_act(x[r0:r1], g, 1e-6)
        assert torch.equal(rs.view(torch.int32), r[r0:r1].view(torch.int32))
        assert torch.equal(qs, q[r0:r1])
        assert torch.equal(ss.view(torch.int32), s[r0 // 128:r1 // 128].view(torch.int32))


def test_rmsnorm_across_the_two_forms():
    """The whole input in the two-grid form against 4096-row chunks in the one-grid form."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    M = -(-192 * sms // 4096) * 4096
    K = 1024
    x = dev_bf16(_bits((M, K), 8))
    g = dev_bf16(f64_to_bf16_bits(np.random.default_rng(9).uniform(0.5, 1.5, K)))
    q, s, r = w8.rmsnorm_quantize_act(x, g, 1e-6)
    r_bits = r.view(torch.int32)
    diff_rows = 0
    for r0 in range(0, M, 4096):
        r1 = r0 + 4096
        qs, ss, rs = w8.rmsnorm_quantize_act(x[r0:r1], g, 1e-6)
        d = (rs.view(torch.int32) - r_bits[r0:r1]).abs()
        assert int(d.max()) <= 1
        diff_rows += int((d != 0).sum())
        same = (d != 0).view(-1, 128).any(dim=1).logical_not()      # strips with equal rstd
        qv, qf = qs.view(-1, 128, K), q[r0:r1].view(-1, 128, K)
        assert torch.equal(qv[same], qf[same])
        sv, sf = ss.view(torch.int32), s[r0 // 128:r1 // 128].view(torch.int32)
        assert torch.equal(sv[same], sf[same])
    assert diff_rows <= max(1, M // 100000)
