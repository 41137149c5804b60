"""The M = 32768 high-resolution block chain end to end on the GPU through the C ABI,
against the oracle's own chain (TurboDiffusion article, inference items 3-5: the fused
RMSNorm feeds the INT8 linears; TurboT2VA paper, W8A8 operator and guard paragraphs).

GPU: w8a8_rmsnorm_quantize_act on x, then the QKV / out / MLP-up GEMMs
(w8a8_linear_prequant) on its codes, w8a8_quantize_act on the MLP-up BF16 output, then the
MLP-down GEMM on those codes.

Oracle: RMSNorm and block quantization of x, the linears on its own codes, BF16 rounding
of the MLP-up output, its block quantization, the MLP-down linear.

Checked: the fused norm's rstd, codes and scales for all 32768 rows, bit for bit; the
weight codes; QKV / out / up outputs on three whole 128-row strips and 4096 sampled points
each, within 1e-2 + 1e-2 |ref|; the down projection's input codes and scales (all
32768 x 16384), bit for bit against the oracle's quantization of the GPU's own MLP-up
output bits (the only exact reference: that output is itself toleranced); the down output
at 4096 sampled points against the oracle's down linear on those codes; and the down
output on the three strips against the oracle's chain from x."""
import numpy as np
import pytest

import block_wise_w8a8_b200 as w8
from gpu_util import assert_close_bf16, assert_codes_equal, bf16_to_f32, dev_bf16, host_bits
from synth import workload

pytestmark = pytest.mark.gpu

STRIPS = (0, 137, 255)


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def test_hires_chain_end_to_end(orc):
    wl = workload("hires_chain_32768")
    lins = {lin["name"]: lin for lin in wl.linears}
    M, K = lins["qkv"]["M"], lins["qkv"]["K"]
    eps = wl.extra["eps"]
    x = wl.x(M, K)
    g = wl.gamma(K)
    # ---- fused RMSNorm + act-quant
    xq, xs, rstd = w8.rmsnorm_quantize_act(dev_bf16(x), dev_bf16(g), eps)
    y_ref, r_ref = orc.rmsnorm(x, g, eps)
    q_ref, s_ref = orc.block_quantize(y_ref)
    np.testing.assert_array_equal(rstd.cpu().numpy().view(np.uint32), r_ref.view(np.uint32))
    assert_codes_equal(xq, xs, q_ref, s_ref, "fused norm")
    del y_ref
    r = np.random.default_rng(44)
    outs, refs = {}, {}
    # ---- QKV, out, MLP-up on the norm's codes
    for name in ("qkv", "out", "up"):
        lin = lins[name]
        w = wl.w(lin)
        wt = w8.W8A8Weight(dev_bf16(w))
        wq_ref, ws_ref = orc.block_quantize(w)
        assert_codes_equal(wt.wq, wt.ws, wq_ref, ws_ref, f"{name} weight")
        y = w8.linear_prequant(xq, xs, wt)
        yb = host_bits(y)
        N = lin["N"]
        for mb in STRIPS:
            ref = orc.w8a8_linear(q_ref, s_ref, wq_ref, ws_ref, None, m0=128 * mb, rows=128)
            assert_close_bf16(yb[128 * mb:128 * (mb + 1)], ref, orc, f"{name} strip {mb}")
            if name == "up":
                refs[mb] = ref
        ms, ns = r.integers(0, M, 4096), r.integers(0, N, 4096)
        ref = orc.w8a8_linear_at(q_ref, s_ref, wq_ref, ws_ref, None, ms, ns)
        assert_close_bf16(yb[ms, ns], ref, orc, f"{name} sampled")
        if name == "up":
            outs["up"] = y
            outs["up_bits"] = yb
        del wt, y
    # ---- act-quant of the MLP-up output, then the down projection
    lin = lins["down"]
    uq, us = w8.quantize_act(outs["up"])
    uq_ref, us_ref = orc.block_quantize(outs["up_bits"])
    assert_codes_equal(uq, us, uq_ref, us_ref, "down input")
    w = wl.w(lin)
    wt = w8.W8A8Weight(dev_bf16(w))
    wq_ref, ws_ref = orc.block_quantize(w)
    assert_codes_equal(wt.wq, wt.ws, wq_ref, ws_ref, "down weight")
    yd = host_bits(w8.linear_prequant(uq, us, wt))
    ms, ns = r.integers(0, M, 4096), r.integers(0, lin["N"], 4096)
    ref = orc.w8a8_linear_at(uq_ref, us_ref, wq_ref, ws_ref, None, ms, ns)
    assert_close_bf16(yd[ms, ns], ref, orc, "down sampled (given the GPU's up output)")
    # ---- the oracle's chain from x on three strips: its own up output, BF16-rounded,
    # quantized, through the down linear
    for mb in STRIPS:
        up_bits = orc.f32_to_bf16(refs[mb])
        cq, cs = orc.block_quantize(up_bits)
        ref = orc.w8a8_linear(cq, cs, wq_ref, ws_ref, None)
        assert_close_bf16(yd[128 * mb:128 * (mb + 1)], ref, orc, f"chain down strip {mb}")
