"""The Python binding's buffer checks, on the CPU: a caller-supplied output or input
buffer of the wrong dtype, shape, device or layout is refused before the library is
called (the library would otherwise write or read out of bounds)."""
import pytest
import torch

import block_wise_w8a8_b200 as w8


def test_out_buffer_checks():
    ok = torch.empty((4, 8), dtype=torch.bfloat16)
    assert w8._out(ok, (4, 8), torch.bfloat16, "cpu", "out") is ok
    fresh = w8._out(None, (2, 3), torch.int8, "cpu", "xq")
    assert fresh.shape == (2, 3) and fresh.dtype == torch.int8
    with pytest.raises(TypeError):
        w8._out(ok.float(), (4, 8), torch.bfloat16, "cpu", "out")
    with pytest.raises(ValueError):
        w8._out(ok, (4, 16), torch.bfloat16, "cpu", "out")          # too small
    with pytest.raises(ValueError):
        w8._out(ok[:, :4], (4, 4), torch.bfloat16, "cpu", "out")     # not contiguous
    with pytest.raises(ValueError):
        w8._out(ok, (4, 8), torch.bfloat16, "meta", "out")           # wrong device
    with pytest.raises(TypeError):
        w8._out([1, 2], (2,), torch.bfloat16, "cpu", "out")
    with pytest.raises(TypeError):
        w8._in(None, (2,), torch.float32, "cpu", "xs")


def test_wrappers_refuse_host_tensors_before_the_library():
    saved = w8._lib
    w8._lib = None

    def boom(*a, **k):
        raise AssertionError("the library must not be reached")
    old_lib = w8.lib
    w8.lib = boom
    try:
        x = torch.zeros((128, 128), dtype=torch.bfloat16)
        with pytest.raises(ValueError):
            w8.quantize_act(x)
        with pytest.raises(ValueError):
            w8.bf16_linear(x, x)
        with pytest.raises(ValueError):
            w8.rmsnorm_quantize_act(x, None)
        with pytest.raises(TypeError):
            w8.linear_host(x.to(torch.float32), None)   # not BF16
    finally:
        w8.lib = old_lib
        w8._lib = saved
