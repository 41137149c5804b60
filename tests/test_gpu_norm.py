"""RMSNorm + block quantizer, plain and modulated (TurboDiffusion article, inference list
item 5; TurboT2VA paper, fused-operator paragraph), on the GPU through the C ABI, against
the oracle.

The library runs one of two forms by shape: below 192 rows per SM a one-grid kernel whose
row sums of squares are split across a cluster, from there on a row-statistics grid that
sums each row in column order followed by the normalising block quantizer.  On the
two-grid form rstd must equal the oracle's bit for bit on every row.  On the one-grid form
it may differ on rows where the two FP64 sums, taken in different orders, round to
neighbouring FP32 values (at most one ulp, on a vanishing fraction of rows).  Given the
kernel's rstd, codes and scales must equal the oracle's bit for bit on both.  Shapes cover
every cluster size (C = min(4, K / 128)), 1 to 128 blocks per CTA and strip, block counts
per CTA that are not a multiple of the four consumer groups or differ between the CTAs of a
cluster, more strips than clusters, gamma absent, and eps = 0 (the exact conversion path);
the special rows (zeros, subnormals, eps = 0) and the near-tie sweep run on both forms."""
import numpy as np
import pytest
import torch

import block_wise_w8a8_b200 as w8
from gpu_util import dev_bf16
from synth import f64_to_bf16_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def _rows(shape, seed, zero_row=True, tiny_row=True):
    r = np.random.default_rng(seed)
    x = r.standard_normal(shape) * np.exp(r.uniform(-4, 4, (shape[0], 1)))
    if zero_row:
        x[0] = 0.0                                  # rstd = 1 / sqrt(eps)
    if tiny_row and shape[0] > 1:
        x[1] = r.standard_normal(shape[1]) * 1e-39  # subnormal BF16 values
    if shape[0] > 2:
        x[2, ::3] = 0.0                             # zeros inside a row
    return f64_to_bf16_bits(x)


def split_rows():
    """The smallest M (a multiple of 128) that takes the two-grid form on this GPU."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return -(-192 * sms // 128) * 128


def _tile_rows(x, M):
    """x repeated down to M rows (M a multiple of x's row count)."""
    assert M % x.shape[0] == 0
    return np.tile(x, (M // x.shape[0], 1))


def _check(orc, x, g, eps, xq, xs, rstd, mod=None, exact_rstd=False):
    """mod = (scale_bits, shift_bits, T) for the modulated operation; exact_rstd for
    results of the two-grid form."""
    if mod is None:
        _, r_ref = orc.rmsnorm(x, g if g is not None else f64_to_bf16_bits(np.ones(x.shape[1])), eps)
    else:
        _, r_ref = orc.mod_rmsnorm(x, g, mod[0], mod[1], mod[2], eps)
    diff = np.nonzero(rstd.view(np.uint32) != r_ref.view(np.uint32))[0]
    assert diff.size <= (0 if exact_rstd else max(1, rstd.size // 100000)), diff[:10]
    for i in diff:
        assert abs(int(rstd.view(np.int32)[i]) - int(r_ref.view(np.int32)[i])) <= 1
    if mod is None:
        gg = g if g is not None else f64_to_bf16_bits(np.ones(x.shape[1]))
        y = orc.rmsnorm_apply(x, gg, rstd)
    else:
        y = orc.mod_rmsnorm_apply(x, g, mod[0], mod[1], mod[2], rstd)
    q_ref, s_ref = orc.block_quantize(y)
    np.testing.assert_array_equal(xs.view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(xq, q_ref)


SHAPES = [(128, 128),      # C = 1, one block
          (256, 384),      # C = 3, one block per CTA
          (384, 896),      # C = 4, seven blocks: 2, 2, 2, 1 per CTA
          (1152, 2048),    # nine strips, 4 blocks per CTA
          (256, 2560),     # 20 blocks: 5 per CTA, not a multiple of the 4 groups
          (384, 3968),     # 31 blocks: 8, 8, 8, 7 per CTA
          (2304, 4096),    # 18 strips of the chain's row length, 8 blocks per CTA
          (256, 6144),     # 12 blocks per CTA
          (256, 7168),     # 14 blocks per CTA: not a multiple of the 4 groups
          (128, 8192),     # 16 blocks per CTA
          (128, 65536)]    # 128 blocks per CTA: the longest rows tested


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("with_gamma", [True, False])
def test_rmsnorm_quantize(orc, M, K, with_gamma):
    x = _rows((M, K), M * 7 + K)
    g = f64_to_bf16_bits(np.random.default_rng(K).uniform(0.5, 1.5, K)) if with_gamma else None
    xq, xs, rstd = w8.rmsnorm_quantize_act(dev_bf16(x), None if g is None else dev_bf16(g), 1e-6)
    _check(orc, x, g, 1e-6, xq.cpu().numpy(), xs.cpu().numpy(), rstd.cpu().numpy())


@pytest.mark.parametrize("M,K,T", [(256, 384, 128), (384, 896, 384), (512, 6144, 256),
                                   (256, 7168, 128), (640, 1024, 128), (1024, 2560, 256),
                                   (2304, 4096, 768)])
@pytest.mark.parametrize("with_gamma", [True, False])
def test_mod_rmsnorm_quantize(orc, M, K, T, with_gamma):
    r = np.random.default_rng(M + K + T)
    x = _rows((M, K), M * 5 + K)
    g = f64_to_bf16_bits(r.uniform(0.5, 1.5, K)) if with_gamma else None
    sc = f64_to_bf16_bits(r.standard_normal((M // T, K)) * 0.5)
    sh = f64_to_bf16_bits(r.standard_normal((M // T, K)) * 0.5)
    sc[0, :7] = f64_to_bf16_bits(np.full(7, -1.0))   # 1 + scale = 0: y = shift
    xq, xs, rstd = w8.rmsnorm_mod_quantize_act(dev_bf16(x), None if g is None else dev_bf16(g),
                                               dev_bf16(sc), dev_bf16(sh), 1e-6)
    _check(orc, x, g, 1e-6, xq.cpu().numpy(), xs.cpu().numpy(), rstd.cpu().numpy(), (sc, sh, T))


@pytest.mark.parametrize("two_grid", [False, True])
@pytest.mark.parametrize("modulated", [False, True])
def test_eps_zero_exact_squares(orc, modulated, two_grid):
    """eps = 0 takes the exact FP64 conversion: rows of subnormal and mixed magnitudes."""
    M, K = 256, 1024
    x = _rows((M, K), 99, zero_row=False)
    # row 1 is subnormal but for one normal value, so that rstd stays finite
    x[1, 5] = f64_to_bf16_bits(np.array([1.0]))[0]
    x[3, 0] = f64_to_bf16_bits(np.array([2.0 ** -126]))[0]
    if two_grid:
        M = split_rows()
        x = _tile_rows(x, M) if M % 256 == 0 else _tile_rows(x[:128], M)
    g = f64_to_bf16_bits(np.random.default_rng(5).uniform(0.5, 1.5, K))
    if modulated:
        r = np.random.default_rng(6)
        sc = f64_to_bf16_bits(r.standard_normal((M // 128, K)) * 0.5)
        sh = f64_to_bf16_bits(r.standard_normal((M // 128, K)) * 0.5)
        xq, xs, rstd = w8.rmsnorm_mod_quantize_act(dev_bf16(x), dev_bf16(g), dev_bf16(sc),
                                                   dev_bf16(sh), 0.0)
        _check(orc, x, g, 0.0, xq.cpu().numpy(), xs.cpu().numpy(), rstd.cpu().numpy(), (sc, sh, 128),
               exact_rstd=two_grid)
    else:
        xq, xs, rstd = w8.rmsnorm_quantize_act(dev_bf16(x), dev_bf16(g), 0.0)
        _check(orc, x, g, 0.0, xq.cpu().numpy(), xs.cpu().numpy(), rstd.cpu().numpy(),
               exact_rstd=two_grid)


@pytest.mark.parametrize("K", [128, 640, 4096])
@pytest.mark.parametrize("modulated", [False, True])
@pytest.mark.parametrize("with_gamma", [True, False])
def test_two_grid_form(orc, K, modulated, with_gamma):
    """The two-grid form on every row: rows of widely spread magnitudes, a zero row, a
    subnormal row and zeros inside rows (_rows), rstd bit-exact on every row; one
    modulation row per 256 rows; then the same call without a caller's rstd buffer gives
    the same codes and scales."""
    M = split_rows()
    x = _rows((M, K), K + 3)
    r = np.random.default_rng(K)
    g = f64_to_bf16_bits(r.uniform(0.5, 1.5, K)) if with_gamma else None
    gd = None if g is None else dev_bf16(g)
    T = 256 if M % 256 == 0 else 128
    sc = f64_to_bf16_bits(r.standard_normal((M // T, K)) * 0.5)
    sh = f64_to_bf16_bits(r.standard_normal((M // T, K)) * 0.5)
    scd, shd = dev_bf16(sc), dev_bf16(sh)
    if modulated:
        xq, xs, rstd = w8.rmsnorm_mod_quantize_act(dev_bf16(x), gd, scd, shd, 1e-6)
    else:
        xq, xs, rstd = w8.rmsnorm_quantize_act(dev_bf16(x), gd, 1e-6)
    _check(orc, x, g, 1e-6, xq.cpu().numpy(), xs.cpu().numpy(), rstd.cpu().numpy(),
           (sc, sh, T) if modulated else None, exact_rstd=True)
    # without rstd_out: the library takes M floats of stream-ordered scratch
    L = w8.lib()
    st = w8._stream(torch.device("cuda"))
    xd = dev_bf16(x)
    q2 = torch.empty_like(xq)
    s2 = torch.empty_like(xs)
    P = lambda t: None if t is None else t.data_ptr()
    if modulated:
        rc = L.w8a8_rmsnorm_mod_quantize_act(P(xd), P(gd), P(scd), P(shd), T, 1e-6,
                                             M, K, P(q2), P(s2), None, st)
    else:
        rc = L.w8a8_rmsnorm_quantize_act(P(xd), P(gd), 1e-6, M, K, P(q2), P(s2), None, st)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(q2, xq) and torch.equal(s2.view(torch.int32), xs.view(torch.int32))


@pytest.mark.parametrize("modulated", [False, True])
def test_hires_chain_norm_sampled(orc, modulated):
    """The M = 32768, K = 4096 chain input (one sample, T = M): the whole launch runs, and
    three 128-row strips (first, one in the middle, last) match the oracle."""
    wl = workload("hires_chain_32768")
    M, K = 32768, 4096
    eps = wl.extra["eps"]
    x = wl.x(M, K)
    g = wl.gamma(K)
    if modulated:
        sc, sh = wl.modulation(1, K)
        xq, xs, rstd = w8.rmsnorm_mod_quantize_act(dev_bf16(x), dev_bf16(g), dev_bf16(sc),
                                                   dev_bf16(sh), eps)
    else:
        xq, xs, rstd = w8.rmsnorm_quantize_act(dev_bf16(x), dev_bf16(g), eps)
    xq, xs, rstd = xq.cpu().numpy(), xs.cpu().numpy(), rstd.cpu().numpy()
    exact = M >= split_rows()
    if exact:
        # every row's rstd (the oracle's normalisation of all rows is cheap; its
        # quantization of all of them is not needed for this)
        _, r_ref = orc.rmsnorm(x, g, eps)
        np.testing.assert_array_equal(rstd.view(np.uint32), r_ref.view(np.uint32))
    for mb in (0, 137, 255):
        rows = slice(mb * 128, (mb + 1) * 128)
        xr = x[rows]
        if modulated:
            _check(orc, xr, g, eps, xq[rows], xs[mb:mb + 1], rstd[rows], (sc, sh, 128), exact_rstd=exact)
        else:
            _check(orc, xr, g, eps, xq[rows], xs[mb:mb + 1], rstd[rows], exact_rstd=exact)


def test_mod_errors():
    L = w8.lib()
    st = w8._stream(torch.device("cuda"))
    x = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    m = torch.zeros((2, 256), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((256, 256), dtype=torch.int8, device="cuda")
    s = torch.empty((2, 2), dtype=torch.float32, device="cuda")
    f = L.w8a8_rmsnorm_mod_quantize_act
    P = lambda t: t.data_ptr()
    assert f(P(x), None, P(m), P(m), 128, 1e-6, 256, 256, P(q), P(s), None, st) == 0
    assert f(P(x), None, P(m), P(m), 0, 1e-6, 256, 256, P(q), P(s), None, st) == 1
    assert f(P(x), None, P(m), P(m), 64, 1e-6, 256, 256, P(q), P(s), None, st) == 2
    assert f(P(x), None, P(m), P(m), 384, 1e-6, 256, 256, P(q), P(s), None, st) == 2
    assert f(P(x), None, P(m) + 2, P(m), 128, 1e-6, 256, 256, P(q), P(s), None, st) == 4
    host = torch.zeros((2, 256), dtype=torch.bfloat16)
    assert f(P(x), None, P(m), P(host), 128, 1e-6, 256, 256, P(q), P(s), None, st) == 3
    assert f(P(x), None, P(m), P(m), 128, -1.0, 256, 256, P(q), P(s), None, st) == 1
    assert L.w8a8_rmsnorm_quantize_act(P(x), None, 1e-6, 256, 200, P(q), P(s), None, st) == 2
    torch.cuda.synchronize()


@pytest.mark.parametrize("two_grid", [False, True])
@pytest.mark.parametrize("modulated", [False, True])
@pytest.mark.parametrize("eps", [0.0, 1e-6])
def test_fused_codes_near_ties_exhaustive(orc, modulated, eps, two_grid):
    """Every BF16 value of both signs in [A/512, A] as a normalised value, for five block
    absmaxes A that are not powers of two: the rows' RMS is 1 (rstd exactly 1.0), so the
    kernel quantizes the input values themselves, and its codes and scales must equal the
    oracle's bit for bit, near-ties included (one-grid form: eps = 0 takes the exact-square
    instantiation, eps = 1e-6 the scaled one; modulated with zero scale and shift).  On
    the two-grid form the sweep's strips are repeated down to the form's row count."""
    from norm_sweep import ABSMAXES, unit_rms_rows
    K = 4096
    x = unit_rms_rows(K, eps)
    if two_grid:
        base = x.shape[0]
        M = -(-split_rows() // base) * base
        x = _tile_rows(x, M)
    M = x.shape[0]
    if modulated:
        z = np.zeros((1, K), dtype=np.uint16)
        xq, xs, rstd = w8.rmsnorm_mod_quantize_act(dev_bf16(x), None, dev_bf16(z), dev_bf16(z), eps)
    else:
        xq, xs, rstd = w8.rmsnorm_quantize_act(dev_bf16(x), None, eps)
    rstd = rstd.cpu().numpy()
    assert np.all(rstd == 1.0)
    xq, xs = xq.cpu().numpy(), xs.cpu().numpy()
    q_ref, s_ref = orc.block_quantize(x)            # rstd = 1: the normalised values are x
    np.testing.assert_array_equal(xs.view(np.uint32), s_ref.view(np.uint32))
    for i, A in enumerate(ABSMAXES):
        assert xs[i, 0] == np.float32(np.float32(A) / np.float32(127.0))
    np.testing.assert_array_equal(xq, q_ref)
    if modulated:
        _check(orc, x, None, eps, xq, xs, rstd, (z, z, M))
    else:
        _check(orc, x, None, eps, xq, xs, rstd)

