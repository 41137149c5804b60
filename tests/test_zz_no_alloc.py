"""w8a8_linear_noalloc: the W8A8 linear for callers that cannot allocate device memory
(its quantized activations live in scratch built into the library).  Called through the
C ABI and compared with w8a8_linear, whose caller provides that workspace: both run the
same quantizer and GEMM on the same inputs, so the outputs must be equal bit for bit (a
tolerance would hide a scratch mix-up that perturbs a few codes).  One case is also
checked against the oracle, and one goes through the Python wrapper.  Collected last on
purpose: if it fails, a run that stops at the first failure has already run every other
test.  Passes alone in a fresh process and after the rest of the suite."""
import ctypes

import numpy as np
import pytest
import torch

import block_wise_w8a8_b200 as w8
from gpu_util import assert_close_bf16, host_bits

pytestmark = pytest.mark.gpu


def _noalloc(x, wt, bias, y):
    L = w8.lib()
    path = ctypes.c_int(-1)
    K = x.shape[-1]
    M = x.numel() // K
    rc = L.w8a8_linear_noalloc(ctypes.c_void_p(x.data_ptr()), M, K, wt.record(),
                               ctypes.c_void_p(0 if bias is None else bias.data_ptr()),
                               ctypes.c_void_p(y.data_ptr()), ctypes.byref(path),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, path.value


def _same(a, b):
    """Equal bit for bit (BF16 patterns)."""
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)), \
        f"{int((a.view(torch.int16) != b.view(torch.int16)).sum())} outputs differ"


def _inputs(M, K, N, seed, bias=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((M, K), generator=g).bfloat16().cuda()
    w = (torch.randn((N, K), generator=g) * K ** -0.5).bfloat16().cuda()
    b = (torch.randn((N,), generator=g) * 0.1).bfloat16().cuda() if bias else None
    return x, w8.W8A8Weight(w), b


def test_two_calls_in_a_row_match_linear():
    """Two calls in a row with different inputs and shapes: the second reuses scratch
    that still holds the first call's codes, and must not depend on them."""
    for (M, K, N, seed) in [(512, 1024, 768, 21), (256, 2048, 384, 22)]:
        x, wt, b = _inputs(M, K, N, seed)
        y_ref = w8.linear(x, wt, b)
        y = torch.empty_like(y_ref)
        rc, path = _noalloc(x, wt, b, y)
        assert rc == 0, w8.lib().w8a8_status_string(rc)
        assert path == w8.PATH_INT8
        torch.cuda.synchronize()
        _same(y, y_ref)
    assert w8.device_error() == 0


def test_against_the_oracle_through_the_wrapper(orc):
    """The Python wrapper, on data that fills the scratch's first call with other codes:
    the output equals w8a8_linear's bits and is within the tolerance of the oracle run on
    its own codes."""
    x0, wt0, b0 = _inputs(1024, 4096, 256, 25)
    y0 = torch.empty((1024, 256), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(x0, wt0, b0, y0)[0] == 0
    M, K, N = 384, 1536, 640
    g = torch.Generator().manual_seed(26)
    xb = torch.randn((M, K), generator=g).bfloat16()
    wb = (torch.randn((N, K), generator=g) * 0.05).bfloat16()
    bb = (torch.randn((N,), generator=g) * 0.1).bfloat16()
    wt = w8.W8A8Weight(wb.cuda())
    y, path = w8.linear_noalloc(xb.cuda(), wt, bb.cuda(), return_path=True)
    assert path == w8.PATH_INT8
    _same(y, w8.linear(xb.cuda(), wt, bb.cuda()))
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    xq, xs = orc.block_quantize(bits(xb))
    wq, ws = orc.block_quantize(bits(wb))
    assert_close_bf16(host_bits(y), orc.w8a8_linear(xq, xs, wq, ws, bits(bb)), orc, "noalloc")
    assert w8.device_error() == 0


def test_largest_accepted_shape_and_rejection():
    """M * K = 16 Mi is accepted; one more 128-row block is refused before any launch."""
    x, wt, _ = _inputs(4096, 4096, 256, 23, bias=False)
    y_ref = w8.linear(x, wt, None)
    y = torch.empty_like(y_ref)
    rc, path = _noalloc(x, wt, None, y)
    assert rc == 0 and path == w8.PATH_INT8
    torch.cuda.synchronize()
    _same(y, y_ref)
    xb = torch.zeros((4096 + 128, 4096), dtype=torch.bfloat16, device="cuda")
    yb = torch.empty((4096 + 128, 256), dtype=torch.bfloat16, device="cuda")
    rc, path = _noalloc(xb, wt, None, yb)
    assert rc == 5 and path == w8.PATH_NONE          # W8A8_ERR_WORKSPACE
    assert w8.device_error() == 0


def test_guard_shapes_take_bf16_path():
    x, wt, b = _inputs(1000, 384, 256, 24)
    y_ref, p_ref = w8.linear(x, wt, b, return_path=True)
    y = torch.empty_like(y_ref)
    rc, path = _noalloc(x, wt, b, y)
    assert rc == 0 and path == p_ref == w8.PATH_BF16
    torch.cuda.synchronize()
    _same(y, y_ref)
    assert w8.device_error() == 0
