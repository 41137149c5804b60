"""CUDA path vs the CPU oracle on the same seeded inputs, through the C ABI.

Bit-exact: INT8 codes, FP32 block scales, INT32 per-K-block sums, fused-RMSNorm codes.
Toleranced: BF16 outputs, |y - bf16(ref)| <= 1e-2 + 1e-2 |bf16(ref)| against the oracle's
FP32 output.  Small shapes span several 128 x 256 tiles and a ragged (128-wide) N tail;
the full-size workloads are checked in full for codes and scales and on row slices plus
sampled coordinates for outputs."""
import numpy as np
import pytest
import torch

import block_wise_w8a8_b200 as w8
from gpu_util import assert_close_bf16, dev_bf16, host_bits
from synth import bf16_bits_to_f32, f64_to_bf16_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def _rand_bits(shape, seed, scale=1.0, kind="normal"):
    r = np.random.default_rng(seed)
    if kind == "t3":
        v = np.clip(r.standard_t(3, shape), -64, 64) * scale
    else:
        v = r.standard_normal(shape) * scale
    return f64_to_bf16_bits(v)


def _special_blocks(rows, cols, seed):
    """A matrix whose blocks exercise the edge cases: zeros, constants, exact ties,
    values on the INT8 grid, huge outliers, tiny subnormal-range values."""
    r = np.random.default_rng(seed)
    x = r.standard_normal((rows, cols))
    kinds = ["zero", "const", "tie", "grid", "outlier", "tiny", "neg_const", "normal"]
    k = 0
    for rb in range(rows // 128):
        for cb in range(cols // 128):
            blk = x[rb * 128:(rb + 1) * 128, cb * 128:(cb + 1) * 128]
            kind = kinds[k % len(kinds)]
            k += 1
            if kind == "zero":
                blk[:] = 0.0
            elif kind == "const":
                blk[:] = 2.75
            elif kind == "neg_const":
                blk[:] = -0.3
            elif kind == "tie":
                ks = r.integers(-127, 127, blk.shape)
                blk[:] = (ks + 0.5) * 2.0 ** -3
                blk[0, 0] = 127 * 2.0 ** -3
            elif kind == "grid":
                blk[:] = r.integers(-127, 128, blk.shape) * 2.0 ** 5
                blk[3, 3] = 127 * 2.0 ** 5
            elif kind == "outlier":
                blk[7, 9] = 3.0e4
            elif kind == "tiny":
                blk[:] *= 1e-38
    return f64_to_bf16_bits(x)


# ------------------------------------------------------------------ quantization

@pytest.mark.parametrize("shape", [(128, 128), (256, 256), (384, 640), (128, 1152), (1024, 384)])
def test_quantize_act_bit_exact(orc, shape):
    x = _rand_bits(shape, 100 + shape[0] + shape[1], kind="t3")
    xq, xs = w8.quantize_act(dev_bf16(x))
    q_ref, s_ref = orc.block_quantize(x)
    np.testing.assert_array_equal(xs.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(xq.cpu().numpy(), q_ref)


def test_quantize_special_blocks(orc):
    x = _special_blocks(512, 512, 7)
    xq, xs = w8.quantize_act(dev_bf16(x))
    q_ref, s_ref = orc.block_quantize(x)
    np.testing.assert_array_equal(xs.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(xq.cpu().numpy(), q_ref)
    wq, ws = w8.quantize_weight(dev_bf16(x))
    np.testing.assert_array_equal(wq.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(ws.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_quantize_near_ties_exhaustive(orc):
    """Every positive and negative BF16 value below absmax in blocks with non-power-of-two
    scales: covers the entries where the reciprocal estimate sits next to a half-integer,
    which the kernel recomputes with the IEEE division."""
    pos = np.arange(1, 0x7F80, dtype=np.uint16)
    posf = bf16_bits_to_f32(pos).astype(np.float64)
    blocks = []
    for A in [1.7421875, 23.625, 0.0146484375, 97.5, 3.0]:
        vals = posf[posf <= A]
        vals = np.concatenate([vals, -vals])
        n = 128 * 128 - 1
        for s in range(0, vals.size, n):
            blk = np.zeros(128 * 128)
            blk[0] = A
            chunk = vals[s:s + n]
            blk[1:1 + chunk.size] = chunk
            blocks.append(blk.reshape(128, 128))
    x = f64_to_bf16_bits(np.concatenate(blocks, 0))
    xq, xs = w8.quantize_act(dev_bf16(x))
    q_ref, s_ref = orc.block_quantize(x)
    np.testing.assert_array_equal(xs.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(xq.cpu().numpy(), q_ref)


# ------------------------------------------------------------------ INT32 block sums

@pytest.mark.parametrize("M,K,N", [(128, 128, 128), (256, 256, 256), (384, 512, 640),
                                   (256, 1024, 384)])
def test_block_sums_bit_exact(orc, M, K, N):
    r = np.random.default_rng(M + K + N)
    xq = r.integers(-127, 128, (M, K)).astype(np.int8)
    wq = r.integers(-127, 128, (N, K)).astype(np.int8)
    xq[0, :] = 127
    wq[0, :] = 127
    xq[1, :] = -127
    got = w8.debug_block_sums(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda())
    ref = orc.block_sums(xq, wq)
    np.testing.assert_array_equal(got.cpu().numpy(), ref)


def test_block_sums_config_slice(orc):
    """The 4096^3 workload's quantized operands: a 256 x 512 corner and a middle slice."""
    wl = workload("attn_proj_4096")
    lin = wl.linears[0]
    x = wl.x(4096, 4096, nrows=256)
    w = wl.w(lin, row0=1024, nrows=512)
    xq, _ = orc.block_quantize(x)
    wq, _ = orc.block_quantize(w)
    got = w8.debug_block_sums(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda())
    np.testing.assert_array_equal(got.cpu().numpy(), orc.block_sums(xq, wq))


@pytest.mark.parametrize("m0,rows,n0,cols", [(0, 384, 0, 640), (5, 100, 130, 300),
                                              (129, 1, 639, 1), (256, 128, 256, 384)])
def test_block_sums_windows(orc, m0, rows, n0, cols):
    """Windows with any offsets and sizes: the main loop runs on the 128-aligned rows and
    columns around them, and only the window is written."""
    r = np.random.default_rng(m0 + rows + n0 + cols)
    M, K, N = 384, 512, 640
    xq = r.integers(-127, 128, (M, K)).astype(np.int8)
    wq = r.integers(-127, 128, (N, K)).astype(np.int8)
    got = w8.debug_block_sums(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(),
                              m0, rows, n0, cols)
    np.testing.assert_array_equal(got.cpu().numpy(), orc.block_sums(xq, wq, m0, rows, n0, cols))


def test_block_sums_mlp_up_full_size_windows(orc):
    """The 16384 x 4096 x 16384 workload's own codes (quantized by the oracle): INT32 block
    sums on three windows of the full-size GEMM (first tile, an unaligned window in the
    middle, the last tile), bit for bit."""
    wl = workload("mlp_up_16384")
    lin = wl.linears[0]
    xq, _ = orc.block_quantize(wl.x(16384, 4096))
    wq, _ = orc.block_quantize(wl.w(lin))
    dx, dw = torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda()
    for m0, rows, n0, cols in ((0, 128, 0, 256), (8191, 300, 9000, 333), (16256, 128, 16128, 256)):
        got = w8.debug_block_sums(dx, dw, m0, rows, n0, cols)
        np.testing.assert_array_equal(got.cpu().numpy(), orc.block_sums(xq, wq, m0, rows, n0, cols),
                                      err_msg=f"window {m0},{rows},{n0},{cols}")


# ------------------------------------------------------------------ W8A8 linear

def _oracle_linear(orc, x, w, bias, m0=0, rows=None):
    xq, xs = orc.block_quantize(x)
    wq, ws = orc.block_quantize(w)
    return orc.w8a8_linear(xq, xs, wq, ws, bias, m0=m0, rows=rows)


@pytest.mark.parametrize("M,K,N,with_bias", [(128, 128, 128, True), (256, 256, 256, True),
                                             (384, 512, 640, False), (640, 384, 896, True),
                                             (128, 2048, 256, True), (1152, 256, 128, False)])
def test_linear_small(orc, M, K, N, with_bias):
    x = _rand_bits((M, K), M * 7 + K, kind="t3")
    w = _rand_bits((N, K), N * 3 + K, scale=0.05)
    b = _rand_bits((N,), N, scale=0.1) if with_bias else None
    wt = w8.W8A8Weight(dev_bf16(w))
    y, path = w8.linear(dev_bf16(x), wt, None if b is None else dev_bf16(b), return_path=True)
    assert path == w8.PATH_INT8
    assert_close_bf16(host_bits(y), _oracle_linear(orc, x, w, b), orc, f"{M}x{K}x{N}")
    # prequant entry point gives identical bits
    xq, xs = w8.quantize_act(dev_bf16(x))
    y2 = w8.linear_prequant(xq, xs, wt, None if b is None else dev_bf16(b))
    np.testing.assert_array_equal(host_bits(y2), host_bits(y))


def test_linear_config_256(orc):
    """The 256^3 workload (seed 0) in full."""
    wl = workload("linear_256")
    lin = wl.linears[0]
    x, w, b = wl.x(256, 256), wl.w(lin), wl.bias(lin)
    wt = w8.W8A8Weight(dev_bf16(w))
    y, path = w8.linear(dev_bf16(x), wt, dev_bf16(b), return_path=True)
    assert path == w8.PATH_INT8
    assert_close_bf16(host_bits(y), _oracle_linear(orc, x, w, b), orc, "linear_256")
    xq, xs = w8.quantize_act(dev_bf16(x))
    q_ref, s_ref = orc.block_quantize(x)
    np.testing.assert_array_equal(xq.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(wt.wq.cpu().numpy(), orc.block_quantize(w)[0])


def _sampled_check(orc, x, w, b, y_bits, nsamp=4096, seed=0, slice_rows=256):
    xq, xs = orc.block_quantize(x)
    wq, ws = orc.block_quantize(w)
    M, N = y_bits.shape
    ref = orc.w8a8_linear(xq, xs, wq, ws, b, m0=0, rows=slice_rows)
    assert_close_bf16(y_bits[:slice_rows], ref, orc, "row slice")
    r = np.random.default_rng(seed)
    ms = r.integers(0, M, nsamp)
    ns = r.integers(0, N, nsamp)
    ref_s = orc.w8a8_linear_at(xq, xs, wq, ws, b, ms, ns)
    assert_close_bf16(y_bits[ms, ns], ref_s, orc, "sampled")
    return xq, xs, wq, ws


def test_linear_config_4096(orc):
    """The 4096^3 attention-projection workload (outlier channels): codes and scales of
    both operands bit-exact in full; outputs on 256 rows plus 4096 sampled points."""
    wl = workload("attn_proj_4096")
    lin = wl.linears[0]
    x, w = wl.x(4096, 4096), wl.w(lin)
    wt = w8.W8A8Weight(dev_bf16(w))
    xd = dev_bf16(x)
    y, path = w8.linear(xd, wt, None, return_path=True)
    assert path == w8.PATH_INT8
    xq, xs, wq, ws = _sampled_check(orc, x, w, None, host_bits(y))
    gq, gs = w8.quantize_act(xd)
    np.testing.assert_array_equal(gq.cpu().numpy(), xq)
    np.testing.assert_array_equal(gs.cpu().numpy().view(np.uint32), xs.view(np.uint32))
    np.testing.assert_array_equal(wt.wq.cpu().numpy(), wq)
    np.testing.assert_array_equal(wt.ws.cpu().numpy().view(np.uint32), ws.view(np.uint32))


@pytest.mark.slow
def test_linear_config_mlp_up(orc):
    """M=16384 K=4096 N=16384 with Student-t(3) activations and bias."""
    wl = workload("mlp_up_16384")
    lin = wl.linears[0]
    x, w, b = wl.x(16384, 4096), wl.w(lin), wl.bias(lin)
    wt = w8.W8A8Weight(dev_bf16(w))
    xd = dev_bf16(x)
    y, path = w8.linear(xd, wt, dev_bf16(b), return_path=True)
    assert path == w8.PATH_INT8
    xq, xs, wq, ws = _sampled_check(orc, x, w, b, host_bits(y), seed=2)
    gq, gs = w8.quantize_act(xd)
    np.testing.assert_array_equal(gq.cpu().numpy(), xq)
    np.testing.assert_array_equal(gs.cpu().numpy().view(np.uint32), xs.view(np.uint32))
    np.testing.assert_array_equal(wt.wq.cpu().numpy(), wq)


# ------------------------------------------------------------------ guard + BF16 path

def test_guard_audio_config(orc):
    """K=2048 N=8192: M=1024 takes INT8; M=1000 (M fails) and K=2000 (K fails, the weight
    cannot be block-quantized) take the BF16 GEMM."""
    wl = workload("audio_2048x8192")
    lin8, lin_m, lin_k = wl.linears
    w = wl.w(lin8)
    wt = w8.W8A8Weight(dev_bf16(w))
    x = wl.x(1024, 2048)
    y, path = w8.linear(dev_bf16(x), wt, None, return_path=True)
    assert path == w8.PATH_INT8
    _sampled_check(orc, x, w, None, host_bits(y), seed=3)
    # M = 1000: the first 1000 rows of the same activation stream
    x1000 = wl.x(1000, 2048)
    y1, path1 = w8.linear(dev_bf16(x1000), wt, None, return_path=True)
    assert path1 == w8.PATH_BF16
    yb = host_bits(y1)
    assert_close_bf16(yb[:200], orc.bf16_linear(x1000, w, None, m0=0, rows=200), orc, "M=1000")
    assert_close_bf16(yb[900:], orc.bf16_linear(x1000, w, None, m0=900, rows=100), orc, "M tail")
    # K = 2000
    wk = wl.w(lin_k)
    wtk = w8.W8A8Weight(dev_bf16(wk))
    assert wtk.wq is None
    xk = wl.x(1024, 2000, stream=wl.extra["x_stream_k2000"])
    y2, path2 = w8.linear(dev_bf16(xk), wtk, None, return_path=True)
    assert path2 == w8.PATH_BF16
    r = np.random.default_rng(5)
    ms, ns = r.integers(0, 1024, 4096), r.integers(0, 8192, 4096)
    assert_close_bf16(host_bits(y2)[ms, ns], orc.bf16_linear_at(xk, wk, None, ms, ns), orc, "K=2000")


@pytest.mark.parametrize("M,K,N", [(1, 8, 1), (100, 200, 72), (129, 136, 257), (300, 64, 520),
                                   (77, 13, 35), (64, 0, 16), (130, 1000, 390)])
def test_bf16_linear_shapes(orc, M, K, N):
    x = _rand_bits((M, K), M + 3 * K + 1)
    w = _rand_bits((N, K), N + K + 2, scale=0.1)
    b = _rand_bits((N,), N + 9, scale=0.5)
    y = w8.bf16_linear(dev_bf16(x), dev_bf16(w), dev_bf16(b))
    assert_close_bf16(host_bits(y), orc.bf16_linear(x, w, b), orc, f"bf16 {M}x{K}x{N}")


def test_guard_non_multiple_n_and_bias(orc):
    M, K, N = 256, 384, 200
    x = _rand_bits((M, K), 11)
    w = _rand_bits((N, K), 12, scale=0.05)
    b = _rand_bits((N,), 13)
    wt = w8.W8A8Weight(dev_bf16(w))
    assert wt.wq is None
    y, path = w8.linear(dev_bf16(x), wt, dev_bf16(b), return_path=True)
    assert path == w8.PATH_BF16
    assert_close_bf16(host_bits(y), orc.bf16_linear(x, w, b), orc, "N=200")


def test_empty_inputs():
    w = torch.zeros((256, 128), dtype=torch.bfloat16, device="cuda")
    wt = w8.W8A8Weight(w)
    y, path = w8.linear(torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda"), wt,
                        return_path=True)
    assert y.shape == (0, 256) and path == w8.PATH_NONE
    xq, xs = w8.quantize_act(torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda"))
    assert xq.shape == (0, 256)


# ------------------------------------------------------------------ fused RMSNorm

def _check_rmsnorm(orc, x, g, eps, xq, xs, rstd, m0=0):
    """rstd bit-exact except (documented) rows where FP64 sums in different orders round
    to neighbouring FP32 values; codes and scales bit-exact given the kernel's rstd."""
    y_ref, r_ref = orc.rmsnorm(x, g, eps, m0=m0, rows=rstd.size)
    diff = np.nonzero(rstd.view(np.uint32) != r_ref.view(np.uint32))[0]
    assert diff.size <= max(1, rstd.size // 100000), diff[:10]
    for i in diff:
        assert abs(int(rstd.view(np.int32)[i]) - int(r_ref.view(np.int32)[i])) <= 1
    y_use = orc.rmsnorm_apply(x, g, rstd, m0=m0)
    q_ref, s_ref = orc.block_quantize(y_use)
    np.testing.assert_array_equal(xs.view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(xq, q_ref)
    return diff.size


@pytest.mark.parametrize("M,K", [(128, 128), (256, 1024), (384, 4096), (128, 16384), (1024, 640)])
def test_rmsnorm_quantize_small(orc, M, K):
    x = _rand_bits((M, K), M + K)
    x[0, :] = 0          # an all-zero row: rstd = 1/sqrt(eps)
    g = f64_to_bf16_bits(np.random.default_rng(K).uniform(0.5, 1.5, K))
    xq, xs, rstd = w8.rmsnorm_quantize_act(dev_bf16(x), dev_bf16(g), 1e-6)
    _check_rmsnorm(orc, x, g, 1e-6, xq.cpu().numpy(), xs.cpu().numpy(), rstd.cpu().numpy())


# ------------------------------------------------------------------ errors

def test_error_codes():
    L = w8.lib()
    dev = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    host = torch.zeros((256, 256), dtype=torch.bfloat16)
    q = torch.empty((256, 256), dtype=torch.int8, device="cuda")
    s = torch.empty((2, 2), dtype=torch.float32, device="cuda")
    st = w8._stream(dev.device)
    assert L.w8a8_quantize_act(host.data_ptr(), 256, 256, q.data_ptr(), s.data_ptr(), st) == 3
    assert L.w8a8_quantize_act(dev.data_ptr(), 256, 200, q.data_ptr(), s.data_ptr(), st) == 2
    assert L.w8a8_quantize_act(dev.data_ptr() + 2, 128, 128, q.data_ptr(), s.data_ptr(), st) == 4
    assert L.w8a8_quantize_act(None, 128, 128, q.data_ptr(), s.data_ptr(), st) == 1
    assert L.w8a8_quantize_act(dev.data_ptr(), -128, 128, q.data_ptr(), s.data_ptr(), st) == 1
    wt = w8.W8A8Weight(dev)
    y = torch.empty((256, 256), dtype=torch.bfloat16, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    path = w8.ctypes.c_int(-1)
    rc = L.w8a8_linear(dev.data_ptr(), 256, 256, wt.record(), None, y.data_ptr(),
                       small.data_ptr(), 16, w8.ctypes.byref(path), st)
    assert rc == 5
    rc = L.w8a8_linear(host.data_ptr(), 256, 256, wt.record(), None, y.data_ptr(),
                       None, 0, w8.ctypes.byref(path), st)
    assert rc == 3
    with pytest.raises(TypeError):
        w8.linear(dev.float(), wt)
    with pytest.raises(ValueError):
        w8.linear(host, wt)
    sums = torch.empty((100, 10, 2), dtype=torch.int32, device="cuda")
    bs = L.w8a8_debug_block_sums
    assert bs(q.data_ptr(), q.data_ptr(), 256, 256, 256, 200, 100, 0, 10, sums.data_ptr(), st) == 1
    assert bs(q.data_ptr(), q.data_ptr(), 256, 256, 256, 0, 100, -1, 10, sums.data_ptr(), st) == 1
    assert bs(q.data_ptr(), q.data_ptr(), 256, 200, 256, 0, 100, 0, 10, sums.data_ptr(), st) == 2
    assert bs(q.data_ptr(), q.data_ptr(), 256, 256, 256, 0, 0, 0, 10, sums.data_ptr(), st) == 0
    torch.cuda.synchronize()


def test_bounded_wait_reports_timeout():
    """A wait that nothing satisfies gives up after its limit and reports through the
    device error word; the context stays usable afterwards."""
    w8.debug_wait_timeout(20_000_000)
    assert w8.device_error() == w8.DEVERR_TIMEOUT
    assert w8.device_error() == 0
    x = torch.ones((128, 128), dtype=torch.bfloat16, device="cuda")
    xq, xs = w8.quantize_act(x)
    assert torch.all(xq == 127)
    assert xs.item() == float(np.float32(1.0) / np.float32(127.0))
