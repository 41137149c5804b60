"""Pins of the CPU oracle: checks against things other than the oracle itself.

Each pin takes an `oracle.Oracle` and raises AssertionError when the oracle disagrees with
a closed form, an exact rational computation, a brute-force library computation, an
invariant, or a special case that reduces to one of those.  test_oracle_pins.py runs them
against the oracle as built; test_oracle_mutants.py runs them against copies of oracle.c
with one plausible mistake planted each, and requires every mutant to fail some pin.

Where a pin needs the correctly rounded FP32 quotient of two FP32 numbers it divides in
float64 and rounds to float32: for division, rounding first to 53 bits and then to 24
bits gives the correctly rounded 24-bit result because 53 >= 2*24 + 2 (Figueroa, "When
is double rounding innocuous?", SIGNUM 1995).
"""
import numpy as np

from synth import bf16_bits_to_f32, f64_to_bf16_bits

B = 128


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(v):
    return f64_to_bf16_bits(np.asarray(v, dtype=np.float64))


def _f32(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def _blocks(a, rb, cb):
    return a[rb * B:(rb + 1) * B, cb * B:(cb + 1) * B]


def _div_f32(x, s):
    """Correctly rounded FP32 quotient (see module docstring)."""
    return (np.asarray(x, np.float64) / np.asarray(s, np.float64)).astype(np.float32)


def _rne_int(v):
    """Round half to even to an integer (numpy's rint is half-to-even)."""
    return np.rint(np.asarray(v, np.float64))


# ------------------------------------------------------------------------ quantization

def pin_scale_power_of_two(o):
    """A block whose largest magnitude is 127 * 2^e has scale exactly 2^e, and its codes
    are rint(x / 2^e), a division that is exact.  The block grid is 2 x 3 (non-square),
    each block with its own exponent, so a transposed or shifted scale index fails."""
    r = _rng(1)
    exps = np.array([[-9, -4, 0], [3, -1, -6]])
    x = np.empty((2 * B, 3 * B))
    for rb in range(2):
        for cb in range(3):
            blk = r.uniform(-1, 1, (B, B)) * 127.0 * 2.0 ** exps[rb, cb]
            blk[r.integers(B), r.integers(B)] = (-1) ** (rb + cb) * 127.0 * 2.0 ** exps[rb, cb]
            x[rb * B:(rb + 1) * B, cb * B:(cb + 1) * B] = blk
    xb = _bf16(x)
    # bf16 rounding can push an entry above 127 * 2^e only by rounding 127*2^e*u up to
    # 128 * 2^e; clip those back so that the intended absmax stays the largest.
    xf = _f32(xb)
    for rb in range(2):
        for cb in range(3):
            lim = 127.0 * 2.0 ** exps[rb, cb]
            v = _blocks(xf, rb, cb)
            v[np.abs(v) > lim] = np.sign(v[np.abs(v) > lim]) * lim
    xb = _bf16(xf)
    q, s = o.block_quantize(xb)
    assert s.shape == (2, 3)
    np.testing.assert_array_equal(s, (2.0 ** exps).astype(np.float32))
    expect = np.empty_like(xf)
    for rb in range(2):
        for cb in range(3):
            expect[rb * B:(rb + 1) * B, cb * B:(cb + 1) * B] = _rne_int(
                _blocks(_f32(xb), rb, cb) * 2.0 ** -exps[rb, cb])
    np.testing.assert_array_equal(q.astype(np.int64), expect.astype(np.int64))


def pin_grid_roundtrip(o):
    """Inputs on the INT8 grid, x = c * 2^e with integer c in [-127, 127] and some |c| =
    127 in each block, come back as codes c and scale 2^e exactly."""
    r = _rng(2)
    c = r.integers(-127, 128, (3 * B, 2 * B))
    exps = np.array([[-3, 2], [0, -12], [5, -1]])
    for rb in range(3):
        for cb in range(2):
            c[rb * B + 7, cb * B + 11] = 127 if (rb + cb) % 2 else -127
    x = c.astype(np.float64)
    for rb in range(3):
        for cb in range(2):
            x[rb * B:(rb + 1) * B, cb * B:(cb + 1) * B] *= 2.0 ** exps[rb, cb]
    q, s = o.block_quantize(_bf16(x))
    np.testing.assert_array_equal(q.astype(np.int64), c)
    np.testing.assert_array_equal(s, (2.0 ** exps).astype(np.float32))


def pin_zero_and_constant_blocks(o):
    """An all-zero block has scale 1 and codes 0; a constant block c has codes
    sign(c) * 127 and scale fl(|c| / 127)."""
    consts = np.array([[0.0, 3.0, -0.0078125, 0.0], [-250.0, 0.0, 1.5, 1e-3]])
    x = np.zeros((2 * B, 4 * B))
    for rb in range(2):
        for cb in range(4):
            x[rb * B:(rb + 1) * B, cb * B:(cb + 1) * B] = consts[rb, cb]
    xb = _bf16(x)
    cf = _f32(_bf16(consts))
    q, s = o.block_quantize(xb)
    exp_s = np.where(cf == 0, 1.0, _div_f32(np.abs(cf), 127.0)).astype(np.float32)
    np.testing.assert_array_equal(s, exp_s)
    for rb in range(2):
        for cb in range(4):
            np.testing.assert_array_equal(_blocks(q, rb, cb), int(np.sign(cf[rb, cb]) * 127))


def pin_ties_to_even(o):
    """With scale 2^e (absmax 127 * 2^e) an entry (k + 1/2) * 2^e is an exact tie and
    must round to the even neighbour: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2, -1.5 -> -2."""
    e = -4
    ks = np.arange(-127, 127)                      # k + 0.5 spans (-126.5 .. 126.5)
    vals = (ks + 0.5) * 2.0 ** e
    x = np.zeros((B, B))
    flat = x.reshape(-1)
    flat[:ks.size] = vals
    flat[-1] = 127.0 * 2.0 ** e
    q, s = o.block_quantize(_bf16(x))
    assert s[0, 0] == np.float32(2.0 ** e)
    expect = np.where(ks % 2 == 0, ks, ks + 1)      # even neighbour of k + 0.5
    np.testing.assert_array_equal(q.reshape(-1)[:ks.size].astype(np.int64), expect)


def pin_division_exact(o):
    """Codes equal rint(fl32(x / s)) with a correctly rounded quotient, over every BF16
    value in [-absmax, absmax] for several scales that are not powers of two.  The set
    is checked to contain entries where rint(x * fl32(1 / s)) differs, so a reciprocal
    multiply in place of the division fails here."""
    r = _rng(3)
    pos = np.arange(1, 0x7F80, dtype=np.uint16)      # all positive finite BF16 patterns
    posf = _f32(pos)
    differs_total = 0
    for A in [1.7421875, 23.625, 0.0146484375, 97.5]:
        a_bits = _bf16([A])[0]
        Af = float(_f32(np.array([a_bits]))[0])
        cand = posf[posf <= Af]
        vals = np.concatenate([cand, -cand])
        r.shuffle(vals)
        n = vals.size
        nblk = -(-n // (B * B - 1))
        x = np.zeros((nblk * B, B))
        for b in range(nblk):
            chunk = vals[b * (B * B - 1):(b + 1) * (B * B - 1)]
            blk = np.zeros(B * B)
            blk[0] = Af
            blk[1:1 + chunk.size] = chunk
            x[b * B:(b + 1) * B] = blk.reshape(B, B)
        xb = _bf16(x)
        q, s = o.block_quantize(xb)
        s_exp = _div_f32(Af, 127.0)
        np.testing.assert_array_equal(s, np.full_like(s, s_exp))
        xf = _f32(xb)
        expect = np.clip(_rne_int(_div_f32(xf, s_exp)), -127, 127)
        np.testing.assert_array_equal(q.astype(np.int64), expect.astype(np.int64))
        recip = np.float32(1.0) / np.float32(s_exp)
        alt = _rne_int((xf.astype(np.float32) * recip).astype(np.float32))
        differs_total += int(np.count_nonzero(alt != expect))
    assert differs_total > 0, "test set has no entry that separates x/s from x*(1/s)"


def pin_error_bound_and_range(o):
    """|x - q s| <= s (1/2 + 2^-17) for every entry (the FP32 quotient is within
    127 * 2^-24 of x/s), |q| <= 127, and each block's largest-magnitude entry gets
    code +-127 with its sign."""
    r = _rng(4)
    t = r.standard_t(3, (4 * B, 3 * B)) * np.exp(r.uniform(-6, 6, (4 * B, 1)))
    t[:, 17] *= 40.0
    xb = _bf16(t)
    xf = _f32(xb)
    q, s = o.block_quantize(xb)
    assert np.all(np.abs(q.astype(np.int64)) <= 127)
    srep = np.repeat(np.repeat(s.astype(np.float64), B, 0), B, 1)
    err = np.abs(xf - q.astype(np.float64) * srep)
    assert np.all(err <= srep * (0.5 + 2.0 ** -17)), float((err / srep).max())
    for rb in range(4):
        for cb in range(3):
            v = _blocks(xf, rb, cb)
            i = np.unravel_index(np.argmax(np.abs(v)), v.shape)
            assert _blocks(q, rb, cb)[i] == (127 if v[i] > 0 else -127)


def pin_block_locality(o):
    """Changing one entry changes only its own 128 x 128 block's scale and codes."""
    r = _rng(5)
    x = _bf16(r.standard_normal((3 * B, 2 * B)))
    q0, s0 = o.block_quantize(x)
    for (i, j) in [(5, 200), (300, 3), (129, 130), (383, 255)]:
        x1 = x.copy()
        x1[i, j] = _bf16([60.0])[0]
        q1, s1 = o.block_quantize(x1)
        rb, cb = i // B, j // B
        mask_s = np.ones_like(s0, bool)
        mask_s[rb, cb] = False
        np.testing.assert_array_equal(s1[mask_s], s0[mask_s])
        assert s1[rb, cb] != s0[rb, cb]
        mask_q = np.ones_like(q0, bool)
        mask_q[rb * B:(rb + 1) * B, cb * B:(cb + 1) * B] = False
        np.testing.assert_array_equal(q1[mask_q], q0[mask_q])


def pin_sign_symmetry(o):
    """quantize(-x) = -quantize(x) with the same scales."""
    r = _rng(6)
    x = _bf16(r.standard_normal((B, 2 * B)) * 3)
    q, s = o.block_quantize(x)
    qn, sn = o.block_quantize(x ^ np.uint16(0x8000))
    np.testing.assert_array_equal(sn, s)
    np.testing.assert_array_equal(qn.astype(np.int64), -q.astype(np.int64))


def pin_bf16_rounding_ties(o):
    """The FP32 -> BF16 helper rounds to nearest, ties to even."""
    vals = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -9,
                     1.0 + 2.0 ** -8 + 2.0 ** -20, 256.5], dtype=np.float32)
    expect = np.array([1.0, 1.0 + 2 * 2.0 ** -7, -1.0, 1.0, 1.0 + 2.0 ** -7, 256.0])
    got = _f32(o.f32_to_bf16(vals))
    np.testing.assert_array_equal(got, expect)


# ------------------------------------------------------------------------ block sums

def pin_block_sums_bruteforce(o):
    """INT32 per-K-block sums equal an int64 einsum of the codes (non-square shapes)."""
    r = _rng(7)
    M, K, N = 2 * B, 3 * B, B
    xq = r.integers(-127, 128, (M, K)).astype(np.int8)
    wq = r.integers(-127, 128, (N, K)).astype(np.int8)
    xq[0, :] = 127
    wq[0, :] = 127
    xq[1, :] = -127
    got = o.block_sums(xq, wq)
    ref = np.einsum("mbk,nbk->mnb", xq.astype(np.int64).reshape(M, K // B, B),
                    wq.astype(np.int64).reshape(N, K // B, B))
    np.testing.assert_array_equal(got.astype(np.int64), ref)
    assert got[0, 0, 0] == 128 * 127 * 127 and got[1, 0, 0] == -128 * 127 * 127
    sub = o.block_sums(xq, wq, m0=B, rows=3, n0=5, cols=4)
    np.testing.assert_array_equal(sub.astype(np.int64), ref[B:B + 3, 5:9])


# ------------------------------------------------------------------------ linear

def _dequant(q, s):
    return q.astype(np.float64) * np.repeat(np.repeat(s.astype(np.float64), B, 0), B, 1)


def pin_linear_dequant_bruteforce(o):
    """FP32 output vs a float64 GEMM of the dequantized operands plus bias, within the
    FP32 rounding bound (KB + 3) * 2^-23 * sum |terms|.  K blocks carry very different
    scales, so a dropped or misindexed scale is far outside the bound."""
    r = _rng(8)
    M, K, N = 2 * B, 4 * B, 3 * B
    x = r.standard_normal((M, K)) * np.repeat(2.0 ** np.array([0, 6, -5, 3]), B)[None, :]
    w = r.standard_normal((N, K)) * np.repeat(2.0 ** np.array([-2, 1, 4, -7]), B)[None, :]
    w *= np.repeat(np.array([1.0, 9.0, 0.25]), B)[:, None]
    bias = _bf16(r.standard_normal(N))
    xq, xs = o.block_quantize(_bf16(x))
    wq, ws = o.block_quantize(_bf16(w))
    y = o.w8a8_linear(xq, xs, wq, ws, bias).astype(np.float64)
    xd, wd = _dequant(xq, xs), _dequant(wq, ws)
    ref = xd @ wd.T + _f32(bias)[None, :]
    mag = np.abs(xd) @ np.abs(wd).T + np.abs(_f32(bias))[None, :]
    bound = (K // B + 3) * 2.0 ** -23 * mag + 1e-30
    assert np.all(np.abs(y - ref) <= bound), float((np.abs(y - ref) / bound).max())
    rows = o.w8a8_linear(xq, xs, wq, ws, bias, m0=B + 3, rows=5)
    np.testing.assert_array_equal(rows, y[B + 3:B + 8].astype(np.float32))


def pin_linear_grid_exact(o):
    """Grid inputs x = c 2^ex, w = c' 2^ew per block: every intermediate is exact in
    FP32, so the output equals the integer sum of c c' 2^(ex + ew) exactly."""
    r = _rng(9)
    M, K, N = B, 2 * B, 2 * B
    cx = r.integers(-127, 128, (M, K))
    cw = r.integers(-127, 128, (N, K))
    ex = np.array([[-3, -4]])
    ew = np.array([[-5, -3], [-4, -4]])
    for cb in range(2):
        cx[0, cb * B] = 127
        for nb in range(2):
            cw[nb * B, cb * B + 1] = -127
    x = cx * np.repeat(2.0 ** ex[0], B)[None, :]
    w = cw.astype(np.float64)
    for nb in range(2):
        w[nb * B:(nb + 1) * B] *= np.repeat(2.0 ** ew[nb], B)[None, :]
    bias = _bf16(np.full(N, 0.5))
    xq, xs = o.block_quantize(_bf16(x))
    wq, ws = o.block_quantize(_bf16(w))
    np.testing.assert_array_equal(xq.astype(np.int64), cx)
    y = o.w8a8_linear(xq, xs, wq, ws, bias).astype(np.float64)
    ref = np.zeros((M, N))
    for kb in range(2):
        for nb in range(2):
            p = cx[:, kb * B:(kb + 1) * B] @ cw[nb * B:(nb + 1) * B, kb * B:(kb + 1) * B].T
            ref[:, nb * B:(nb + 1) * B] += p * 2.0 ** (ex[0, kb] + ew[nb, kb])
    ref += 0.5
    np.testing.assert_array_equal(y, ref)


def pin_linear_bias_once(o):
    """Zero weights: every output equals its bias exactly (added once, per column)."""
    r = _rng(10)
    xq, xs = o.block_quantize(_bf16(r.standard_normal((B, 2 * B))))
    wq = np.zeros((3 * B, 2 * B), np.int8)
    ws = np.ones((3, 2), np.float32)
    bias = _bf16(r.standard_normal(3 * B))
    y = o.w8a8_linear(xq, xs, wq, ws, bias)
    np.testing.assert_array_equal(y, np.broadcast_to(_f32(bias).astype(np.float32), y.shape))
    y0 = o.w8a8_linear(xq, xs, wq, ws, None)
    assert np.all(y0 == 0)


def pin_linear_sampled(o):
    """The sampled entry point returns the full output's entries at those coordinates."""
    r = _rng(11)
    xq, xs = o.block_quantize(_bf16(r.standard_normal((2 * B, 2 * B))))
    wq, ws = o.block_quantize(_bf16(r.standard_normal((3 * B, 2 * B))))
    bias = _bf16(r.standard_normal(3 * B))
    y = o.w8a8_linear(xq, xs, wq, ws, bias)
    ms = r.integers(0, 2 * B, 50)
    ns = r.integers(0, 3 * B, 50)
    np.testing.assert_array_equal(o.w8a8_linear_at(xq, xs, wq, ws, bias, ms, ns), y[ms, ns])


# ------------------------------------------------------------------------ RMSNorm

def pin_rmsnorm_constant_rows(o):
    """A constant row c has mean square c^2, so rstd = 1 / sqrt(c^2 + eps) to within one
    FP32 rounding; with gamma = 1 each output is bf16(c * rstd)."""
    K = 512
    cs = np.array([1.0, -3.5, 2.0 ** -10, 0.0078125, 40.0, -2.0 ** -12])
    eps = 1e-6
    x = _bf16(np.repeat(cs[:, None], K, 1))
    cf = _f32(x[:, 0])
    g = _bf16(np.ones(K))
    y, rstd = o.rmsnorm(x, g, eps)
    exact = 1.0 / np.sqrt(cf * cf + float(np.float32(eps)))
    assert np.all(np.abs(rstd - exact) <= exact * 2.0 ** -23), (rstd, exact)
    yv = _f32(y)
    for i in range(len(cs)):
        v = cf[i] * float(rstd[i])
        assert np.all(np.abs(yv[i] - v) <= abs(v) * 2.0 ** -8)


def pin_rmsnorm_gamma_and_bound(o):
    """Random rows: rstd within two FP32 ulps of the float64 formula; outputs within BF16
    rounding of x * rstd * gamma[k] (gamma indexed by column)."""
    r = _rng(12)
    M, K = 6, 384
    x = _bf16(r.standard_normal((M, K)) * np.exp(r.uniform(-3, 3, (M, 1))))
    g = _bf16(r.uniform(0.5, 1.5, K))
    y, rstd = o.rmsnorm(x, g, 1e-6)
    xf = _f32(x)
    exact = 1.0 / np.sqrt((xf * xf).mean(1) + float(np.float32(1e-6)))
    assert np.all(np.abs(rstd - exact) <= exact * 2.0 ** -22)
    v = xf * rstd.astype(np.float64)[:, None] * _f32(g)[None, :]
    assert np.all(np.abs(_f32(y) - v) <= np.abs(v) * 2.0 ** -8 + 1e-38)
    y2 = o.rmsnorm_apply(x, g, rstd)
    np.testing.assert_array_equal(y2, y)
    y3, r3 = o.rmsnorm(x, g, 1e-6, m0=2, rows=3)
    np.testing.assert_array_equal(y3, y[2:5])
    np.testing.assert_array_equal(r3, rstd[2:5])


# ------------------------------------------------------------------------ BF16 fallback

def pin_bf16_permutation(o):
    """A 0/1 selection matrix W[n, pi(n)] = 1 (N != K) gives y[m, n] = x[m, pi(n)] exactly,
    plus an exact bias."""
    r = _rng(13)
    M, K, N = 37, 200, 72
    x = _bf16(r.standard_normal((M, K)))
    pi = r.permutation(K)[:N]
    w = np.zeros((N, K))
    w[np.arange(N), pi] = 1.0
    y = o.bf16_linear(x, _bf16(w), None)
    np.testing.assert_array_equal(y, _f32(x)[:, pi].astype(np.float32))
    bias = _bf16(np.full(N, 0.25))
    yb = o.bf16_linear(x, _bf16(w), bias)
    np.testing.assert_array_equal(yb, (_f32(x)[:, pi] + 0.25).astype(np.float32))


def pin_bf16_textbook(o):
    """Ragged shapes vs a float64 matmul: within one FP32 rounding (plus the bias add)."""
    r = _rng(14)
    M, K, N = 100, 200, 72
    x = _bf16(r.standard_normal((M, K)))
    w = _bf16(r.standard_normal((N, K)) * 0.1)
    bias = _bf16(r.standard_normal(N))
    y = o.bf16_linear(x, w, bias).astype(np.float64)
    ref = _f32(x) @ _f32(w).T + _f32(bias)[None, :]
    mag = np.abs(_f32(x)) @ np.abs(_f32(w)).T + np.abs(_f32(bias))[None, :]
    assert np.all(np.abs(y - ref) <= mag * 2.0 ** -22)
    ms = r.integers(0, M, 30)
    ns = r.integers(0, N, 30)
    np.testing.assert_array_equal(o.bf16_linear_at(x, w, bias, ms, ns),
                                  y[ms, ns].astype(np.float32))


# ---------------------------------------------------------------- per-row operator
# TurboT2VA paper, W8A8 operator paragraph: s = max(||row||_inf, 1e-4) / 127 per activation
# row and per weight output channel, INT32 accumulation over all of K, both scales and the
# bias once.

ROW_EPS32 = np.float32(1e-4)


def pin_row_scale_closed_forms(o):
    """Rows whose absmax is 127 * 2^e get s = 2^e; an all-zero row and a row below the
    floor get the floor's scale fl(1e-4 / 127); the floor row's largest code is the
    correctly rounded quotient (well below 127)."""
    es = [-20, -6, 0, 3, 11]
    K = 200
    x = np.zeros((len(es) + 2, K))
    for i, e in enumerate(es):
        x[i, 7] = -127.0 * 2.0 ** e
        x[i, 8:] = _rng(i).uniform(-1, 1, K - 8) * 2.0 ** e * 100
    x[len(es) + 1, 3] = 2.0 ** -15          # below the 1e-4 floor
    q, s = o.row_quantize(_bf16(x))
    for i, e in enumerate(es):
        assert s[i] == np.float32(2.0 ** e), (i, s[i])
        assert q[i, 7] == -127
    floor = _div_f32(ROW_EPS32, np.float32(127))
    assert s[len(es)] == floor and s[len(es) + 1] == floor
    assert not q[len(es)].any()
    expect = int(np.rint(_div_f32(np.float32(2.0 ** -15), floor)))
    assert q[len(es) + 1, 3] == expect and 0 < expect < 127, expect


def pin_row_grid_roundtrip(o):
    """Inputs c * 2^e with integer |c| <= 127 and some |c| = 127 per row: codes are c."""
    r = _rng(31)
    M, K = 9, 300
    c = r.integers(-127, 128, (M, K))
    c[np.arange(M), r.integers(0, K, M)] = 127 * r.choice([-1, 1], M)
    e = r.integers(-19, 30, M)          # 127 * 2^e stays above the 1e-4 floor
    q, s = o.row_quantize(_bf16(c * 2.0 ** e[:, None]))
    np.testing.assert_array_equal(q.astype(np.int64), c)
    np.testing.assert_array_equal(s, (2.0 ** e).astype(np.float32))


def pin_row_error_bound(o):
    """|x - q s| <= s (1/2 + 2^-17) for rows above the floor; each row's absmax element
    maps to +-127; codes never leave [-127, 127]."""
    r = _rng(32)
    x = r.standard_t(3, (40, 257)) * np.exp(r.uniform(-8, 8, (40, 1)))
    bits = _bf16(x)
    q, s = o.row_quantize(bits)
    xf = _f32(bits)
    sd = s.astype(np.float64)[:, None]
    assert np.all(np.abs(xf - q * sd) <= sd * (0.5 + 2.0 ** -17))
    am = np.argmax(np.abs(xf), axis=1)
    assert np.all(np.abs(q[np.arange(40), am]) == 127)
    assert q.min() >= -127


def pin_row_linear_bruteforce(o):
    """Against a float64 dequantize-then-GEMM on odd shapes, with per-row and per-column
    scales that differ by up to 2^24 (a transposed or swapped scale index fails), within
    the four FP32 roundings of the epilogue."""
    r = _rng(33)
    M, K, N = 6, 333, 9
    xb = _bf16(r.standard_normal((M, K)) * 2.0 ** r.integers(-12, 12, (M, 1)))
    wb = _bf16(r.standard_normal((N, K)) * 2.0 ** r.integers(-12, 12, (N, 1)))
    bb = _bf16(r.standard_normal(N) * 0.1)
    xq, xs = o.row_quantize(xb)
    wq, ws = o.row_quantize(wb)
    out = o.row_linear(xq, xs, wq, ws, bb).astype(np.float64)
    acc = xq.astype(np.int64) @ wq.astype(np.int64).T
    main = acc * xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :]
    ref = main + _f32(bb)[None, :]
    assert np.all(np.abs(out - ref) <= 2.0 ** -22 * (np.abs(main) + np.abs(ref)) + 1e-30)
    # sampled entry point agrees bit for bit
    ms, ns = np.array([0, 5, 3]), np.array([8, 0, 4])
    np.testing.assert_array_equal(o.row_linear_at(xq, xs, wq, ws, bb, ms, ns),
                                  out[ms, ns].astype(np.float32))


def pin_row_int32_to_fp32(o):
    """INT32 sums of 2^24 + 1 and 2^24 + 3 are rounded to FP32 (half to even: 2^24 and
    2^24 + 4) before the scales multiply them.  With unit scales that is the whole
    output; with the weight scale fl(128 / 127) the output is fl(fl(sum) * scale), which
    differs from rounding the exact product once."""
    K = 1042
    differs = []
    for w_absmax in (127.0, 128.0):
        w = np.zeros((1, K))
        w[0, :1040] = w_absmax
        w[0, 1040] = 24.25 if w_absmax == 128.0 else 24.0
        w[0, 1041] = 1
        for extra, sum_f32 in ((9, 2.0 ** 24), (11, 2.0 ** 24 + 4)):
            x = np.zeros((1, K))
            x[0, :1041] = 127
            x[0, 1041] = extra
            xq, xs = o.row_quantize(_bf16(x))
            wq, ws = o.row_quantize(_bf16(w))
            acc = int((xq.astype(np.int64) @ wq.astype(np.int64).T)[0, 0])
            assert xs[0] == 1 and acc == 2 ** 24 + extra - 8, (xs, acc)
            scale = np.float32(xs[0]) * np.float32(ws[0])
            expect = np.float32(np.float32(sum_f32) * scale)
            got = o.row_linear(xq, xs, wq, ws, None)[0, 0]
            assert got == expect, (w_absmax, extra, got, expect)
            if w_absmax == 128.0:
                differs.append(expect != np.float32(np.float64(acc) * np.float64(scale)))
    assert any(differs)     # the case separates the two rounding orders


def pin_row_bias_once(o):
    """All-zero codes: the output is the bias, added once."""
    xq = np.zeros((3, 256), np.int8)
    wq = np.zeros((5, 256), np.int8)
    bb = _bf16(np.array([1.5, -2.25, 0.0, 7.0, -0.125]))
    out = o.row_linear(xq, np.ones(3, np.float32), wq, np.ones(5, np.float32), bb)
    np.testing.assert_array_equal(out, np.tile(_f32(bb).astype(np.float32), (3, 1)))


# ----------------------------------------------- modulated RMSNorm and gated residual

def pin_modrms_identity_is_rmsnorm(o):
    """scale = 0, shift = 0: the modulation is the identity (1 + 0 = 1 and n * 1 + 0 = n
    exactly, up to the sign of a zero), so the output is the plain RMSNorm's, bit for bit
    apart from -0 / +0, for every sample; without gamma it is the RMSNorm with gamma = 1."""
    r = _rng(31)
    M, K, T = 6, 256, 2
    x = _bf16(r.standard_normal((M, K)) * np.exp(r.uniform(-4, 4, (M, 1))))
    g = _bf16(r.uniform(0.5, 1.5, K))
    z = np.zeros((M // T, K), np.uint16)
    y0, r0 = o.rmsnorm(x, g, 1e-6)
    y1, r1 = o.mod_rmsnorm(x, g, z, z, T, 1e-6)
    np.testing.assert_array_equal(r1, r0)
    np.testing.assert_array_equal(y1 & 0x7FFF, y0 & 0x7FFF)
    y2, _ = o.mod_rmsnorm(x, None, z, z, T, 1e-6)
    y3, _ = o.rmsnorm(x, _bf16(np.ones(K)), 1e-6)
    np.testing.assert_array_equal(y2 & 0x7FFF, y3 & 0x7FFF)


def _modrms_case(seed, M, K, T):
    """Rows c (-1)^k with c = 2^j: with eps = 0, rstd = 2^-j exactly and n = +-1; gamma,
    scale and shift are short dyadics, so n * gamma * (1 + scale) + shift is exact in
    FP32 and in BF16 and the output has a closed form."""
    r = _rng(seed)
    js = r.integers(-6, 7, M)
    sgn = np.where(np.arange(K) % 2 == 0, 1.0, -1.0)
    x = (2.0 ** js)[:, None] * sgn[None, :]
    gam = r.choice([0.5, 1.0, 2.0, 4.0], K)
    sc = r.choice([-1.0, -0.5, 0.0, 0.25, 1.0, 3.0], (M // T, K))
    sh = r.choice([-0.75, 0.0, 0.5, 3.0, -2.0], (M // T, K))
    b = np.arange(M) // T
    exact = sgn[None, :] * gam[None, :] * (1.0 + sc[b]) + sh[b]
    return _bf16(x), _bf16(gam), _bf16(sc), _bf16(sh), exact, js


def pin_modrms_closed_form(o):
    """The closed form above on three samples of two rows each (so that m / T, m % 3 and
    a transposed [K, B] modulation index all differ): every output, and rstd = 2^-j."""
    for T, M in ((2, 6), (1, 5), (5, 5)):
        x, g, sc, sh, exact, js = _modrms_case(40 + T, M, 96, T)
        y, rstd = o.mod_rmsnorm(x, g, sc, sh, T, 0.0)
        np.testing.assert_array_equal(rstd, (2.0 ** -js).astype(np.float32))
        np.testing.assert_array_equal(_f32(y), exact)
        # without gamma: gamma = 1 in the closed form
        y2, _ = o.mod_rmsnorm(x, None, sc, sh, T, 0.0)
        b = np.arange(M) // T
        sgn = np.where(np.arange(96) % 2 == 0, 1.0, -1.0)
        np.testing.assert_array_equal(_f32(y2), sgn[None, :] * (1.0 + _f32(sc)[b]) + _f32(sh)[b])


def pin_modrms_error_bound(o):
    """Random rows and modulation: within BF16 rounding (2^-9 relative) plus the FP32
    error of the steps before it, of the float64 value x rstd gamma (1 + scale) + shift,
    rstd itself within two FP32 ulps of the float64 formula."""
    r = _rng(44)
    M, K, T = 8, 384, 4
    x = _bf16(r.standard_normal((M, K)) * np.exp(r.uniform(-3, 3, (M, 1))))
    g = _bf16(r.uniform(0.5, 1.5, K))
    sc = _bf16(r.standard_normal((M // T, K)) * 0.3)
    sh = _bf16(r.standard_normal((M // T, K)) * 0.5)
    y, rstd = o.mod_rmsnorm(x, g, sc, sh, T, 1e-6)
    xf = _f32(x)
    ex_r = 1.0 / np.sqrt((xf * xf).mean(1) + float(np.float32(1e-6)))
    assert np.all(np.abs(rstd - ex_r) <= ex_r * 2.0 ** -22)
    b = np.arange(M) // T
    u = xf * ex_r[:, None] * _f32(g)[None, :] * (1.0 + _f32(sc)[b])
    v = u + _f32(sh)[b]
    err = np.abs(_f32(y) - v)
    assert np.all(err <= np.abs(v) * 2.0 ** -8 + (np.abs(u) + np.abs(_f32(sh)[b])) * 2.0 ** -19 + 1e-38)
    # rows of one sample use that sample's modulation row: a sub-range call agrees, and
    # so does the normalisation applied with the returned rstd
    y3, r3 = o.mod_rmsnorm(x, g, sc, sh, T, 1e-6, m0=3, rows=4)
    np.testing.assert_array_equal(y3, y[3:7])
    np.testing.assert_array_equal(r3, rstd[3:7])
    np.testing.assert_array_equal(o.mod_rmsnorm_apply(x, g, sc, sh, T, rstd[3:7], m0=3), y[3:7])


def pin_gated_closed_form(o):
    """Short dyadic v, residual and gate: r + gate[m / T, n] v is exact in FP32 and BF16;
    three samples of two rows, N = 5 (so m % 3 or a transposed gate index differ)."""
    r = _rng(50)
    M, N, T = 6, 5, 2
    v = r.integers(-8, 9, (M, N)).astype(np.float32)
    res = _bf16(r.choice([-1.5, -0.25, 0.0, 0.75, 6.0], (M, N)))
    gate = _bf16(r.choice([-1.0, 0.0, 0.5, 2.0, 0.25], (M // T, N)))
    out = o.gated_residual(v, res, gate, T, M)
    b = np.arange(M) // T
    np.testing.assert_array_equal(_f32(out), _f32(res) + _f32(gate)[b] * v)
    # the same points given one by one, in another order
    ms, ns = np.indices((M, N)).reshape(2, -1)
    perm = r.permutation(ms.size)
    o2 = o.gated_residual(v[ms[perm], ns[perm]], res[ms[perm], ns[perm]], gate, T, M,
                          ms[perm], ns[perm])
    np.testing.assert_array_equal(o2, out[ms[perm], ns[perm]])


def pin_gated_special_cases(o):
    """gate = 1, residual = 0: the output is bf16(v), the plain linear's rounding; gate =
    0: the residual itself; and one rounding only: v = 1 + 2^-8 (a BF16 tie that rounds
    down on its own) plus r = 2^-9 gives 1 + 2^-7, where rounding v first would give 1."""
    r = _rng(51)
    M, N = 4, 7
    v = (r.standard_normal((M, N)) * 10).astype(np.float32)
    one = _bf16(np.ones((1, N)))
    zero = np.zeros((M, N), np.uint16)
    np.testing.assert_array_equal(o.gated_residual(v, zero, one, M, M), o.f32_to_bf16(v))
    res = _bf16(r.standard_normal((M, N)))
    out = o.gated_residual(v, res, np.zeros((2, N), np.uint16), 2, M)
    np.testing.assert_array_equal(out & 0x7FFF, res & 0x7FFF)
    vt = np.full((1, 1), 1.0 + 2.0 ** -8, np.float32)
    out = o.gated_residual(vt, _bf16(np.full((1, 1), 2.0 ** -9)), _bf16(np.ones((1, 1))), 1, 1)
    assert _f32(out)[0, 0] == 1.0 + 2.0 ** -7, _f32(out)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
