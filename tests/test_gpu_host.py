"""w8a8_linear_host: the W8A8 linear on host buffers, streamed through the GPU in chunks
of rows.  Same kernels and same guard as w8a8_linear, so its output equals w8a8_linear on
a device copy of the input bit for bit; the oracle anchors both.  Covers the INT8 path
with whole and ragged last chunks, the BF16 guard path, bias, pageable host memory,
completion on the caller's stream, and the argument errors."""
import ctypes

import numpy as np
import pytest
import torch

import block_wise_w8a8_b200 as w8
from gpu_util import assert_close_bf16, dev_bf16, host_bits
from synth import f64_to_bf16_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def _host(bits, pin=True):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pin else t.clone()


def _rand_bits(shape, seed, scale=1.0):
    return f64_to_bf16_bits(np.random.default_rng(seed).standard_normal(shape) * scale)


def _same(y_host, y_dev):
    assert torch.equal(y_host.view(torch.int16), y_dev.cpu().view(torch.int16))


@pytest.mark.parametrize("chunk", [0, 128, 384])
def test_int8_path_equals_device_linear(orc, chunk):
    """Audio-stream linear M=1024, K=2048, N=8192: default chunks (512 rows), 8 chunks of
    128, and chunks of 384 with a ragged last chunk of 256."""
    wl = workload("audio_2048x8192")
    w = wl.w(wl.linears[0])
    wt = w8.W8A8Weight(dev_bf16(w))
    x = wl.x(1024, 2048)
    y_dev = w8.linear(dev_bf16(x), wt, None)
    y_host, path = w8.linear_host(_host(x), wt, None, chunk_rows=chunk, return_path=True)
    torch.cuda.current_stream().synchronize()
    assert path == w8.PATH_INT8
    _same(y_host, y_dev)
    xq, xs = orc.block_quantize(x)
    wq, ws = orc.block_quantize(w)
    ref = orc.w8a8_linear(xq, xs, wq, ws, None, m0=896, rows=128)
    assert_close_bf16(host_bits(y_host)[896:], ref, orc, "last rows")


def test_int8_path_with_bias_and_pageable_memory(orc):
    M, K, N = 640, 256, 384
    x, w, b = _rand_bits((M, K), 41), _rand_bits((N, K), 42, 0.05), _rand_bits((N,), 43, 0.1)
    wt = w8.W8A8Weight(dev_bf16(w))
    bd = dev_bf16(b)
    y_dev = w8.linear(dev_bf16(x), wt, bd)
    for pin in (True, False):
        out = torch.empty((M, N), dtype=torch.bfloat16)
        out = out.pin_memory() if pin else out
        y_host, path = w8.linear_host(_host(x, pin), wt, bd, out=out, chunk_rows=256,
                                      return_path=True)
        torch.cuda.current_stream().synchronize()
        assert path == w8.PATH_INT8 and y_host is out
        _same(y_host, y_dev)
    xq, xs = orc.block_quantize(x)
    wq, ws = orc.block_quantize(w)
    assert_close_bf16(host_bits(y_host), orc.w8a8_linear(xq, xs, wq, ws, b), orc, "bias")


def test_bf16_guard_path_equals_device_linear(orc):
    """M = 1000 fails the guard: every chunk (256, 256, 256, 232 rows) takes the BF16 GEMM,
    as w8a8_linear does for the whole input."""
    M, K, N = 1000, 256, 384
    x, w, b = _rand_bits((M, K), 51), _rand_bits((N, K), 52, 0.05), _rand_bits((N,), 53, 0.1)
    wt = w8.W8A8Weight(dev_bf16(w))
    bd = dev_bf16(b)
    y_dev, p_dev = w8.linear(dev_bf16(x), wt, bd, return_path=True)
    y_host, path = w8.linear_host(_host(x), wt, bd, chunk_rows=256, return_path=True)
    torch.cuda.current_stream().synchronize()
    assert p_dev == w8.PATH_BF16 and path == w8.PATH_BF16
    _same(y_host, y_dev)
    assert_close_bf16(host_bits(y_host)[768:], orc.bf16_linear(x, w, b, m0=768, rows=232), orc,
                      "ragged BF16 chunk")


def test_argument_errors():
    L = w8.lib()
    M, K, N = 256, 256, 256
    w = w8.W8A8Weight(dev_bf16(_rand_bits((N, K), 61, 0.05)))
    xh = _host(_rand_bits((M, K), 62))
    yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    need = w8.linear_host_workspace_bytes(M, K, N, 128)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call(x_ptr, y_ptr, ws_bytes, chunk):
        return L.w8a8_linear_host(ctypes.c_void_p(x_ptr), M, K, w.record(), None,
                                  ctypes.c_void_p(y_ptr), ctypes.c_void_p(ws.data_ptr()),
                                  ws_bytes, chunk, None, st)

    assert call(xh.data_ptr(), yh.data_ptr(), need, 128) == 0
    xd = xh.cuda()
    assert call(xd.data_ptr(), yh.data_ptr(), need, 128) == 1        # x in device memory
    assert call(xh.data_ptr(), 0, need, 128) == 1                     # no output
    assert call(xh.data_ptr(), yh.data_ptr(), need, 100) == 1        # chunk not a multiple of 128
    assert call(xh.data_ptr(), yh.data_ptr(), need - 1, 128) == 5    # workspace too small
    with pytest.raises(ValueError):
        w8.linear_host(xd, w)
    assert L.w8a8_linear_host_chunk_rows(4096, 4096) == 512
    assert L.w8a8_linear_host_chunk_rows(300, 16384) == 128
    torch.cuda.current_stream().synchronize()
