"""Synthetic BF16 tensors for the five linear-layer workloads, addressable by row slice.

Every tensor is a row-major [rows, cols] matrix whose element e = r * cols + c is drawn
from Philox4x32-10 keyed by (seed, stream) at counter e // 4, word e % 4 (normal and
uniform draws), or at counter e (Student-t draws, which use all four words).  The value
is computed in float64, rounded to float32, then to BF16 with round-to-nearest-even.
Only BF16 bit patterns (uint16) leave this module.
"""
import math
import numpy as np

from .philox import philox4x32_10, uniform_open01, normal_pairs

# Stream ids (the second key word).
STREAM_X, STREAM_W, STREAM_BIAS, STREAM_GAMMA, STREAM_OUTLIER = 0, 1, 2, 3, 4
STREAM_MOD_SCALE, STREAM_MOD_SHIFT, STREAM_GATE, STREAM_RESID = 5, 6, 7, 8
STREAM_LAYER0 = 16          # chained linears use 16, 17, ...
STREAM_X_K2000, STREAM_W_K2000 = 32, 33

_CHUNK = 1 << 22            # elements generated per numpy pass


def f64_to_bf16_bits(v):
    """float64 -> float32 (RNE) -> BF16 bit pattern (RNE).  Finite inputs only."""
    b = np.ascontiguousarray(v, dtype=np.float64).astype(np.float32).view(np.uint32)
    # finite float32 patterns are <= 0xFF7FFFFF, so adding 0x8000 cannot wrap
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits):
    """Exact widening of BF16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _words_for_elements(e0, e1, seed, stream):
    """Four words per counter covering elements [e0, e1); returns (words (4, nc), offset)."""
    n0, n1 = e0 // 4, (e1 - 1) // 4 + 1
    w = philox4x32_10(np.arange(n0, n1, dtype=np.uint64), seed, stream)
    return w, e0 - 4 * n0


def _normal_flat(e0, e1, seed, stream):
    w, off = _words_for_elements(e0, e1, seed, stream)
    za, zb = normal_pairs(w[0], w[1])
    zc, zd = normal_pairs(w[2], w[3])
    z = np.stack([za, zb, zc, zd], axis=1).reshape(-1)
    return z[off:off + (e1 - e0)]


def _uniform_flat(e0, e1, seed, stream):
    w, off = _words_for_elements(e0, e1, seed, stream)
    u = uniform_open01(w).T.reshape(-1)
    return u[off:off + (e1 - e0)]


def _student_t3_flat(e0, e1, seed, stream):
    w = philox4x32_10(np.arange(e0, e1, dtype=np.uint64), seed, stream)
    z0, z1 = normal_pairs(w[0], w[1])
    z2, z3 = normal_pairs(w[2], w[3])
    return z0 / np.sqrt((z1 * z1 + z2 * z2 + z3 * z3) / 3.0)


def _fill(rows, cols, row0, nrows, draw, post):
    nrows = rows - row0 if nrows is None else nrows
    assert 0 <= row0 and row0 + nrows <= rows
    out = np.empty(nrows * cols, dtype=np.uint16)
    e_base = row0 * cols
    total = nrows * cols
    step = max(cols, (_CHUNK // cols) * cols)
    for s in range(0, total, step):
        t = min(total, s + step)
        v = draw(e_base + s, e_base + t)
        out[s:t] = f64_to_bf16_bits(post(v, s, t)).reshape(-1)
    return out.reshape(nrows, cols)


def normal_bf16(rows, cols, seed, stream, sigma=1.0, row0=0, nrows=None,
                col_scale=None):
    """N(0, sigma) entries (sigma = standard deviation); optional per-column factor
    (float64 array of length cols) applied before rounding."""
    def post(v, s, t):
        v = v * sigma
        if col_scale is not None:
            v = v.reshape(-1, cols) * col_scale[None, :]
        return v
    return _fill(rows, cols, row0, nrows,
                 lambda a, b: _normal_flat(a, b, seed, stream), post)


def uniform_bf16(rows, cols, seed, stream, lo, hi, row0=0, nrows=None):
    """U(lo, hi) entries."""
    return _fill(rows, cols, row0, nrows,
                 lambda a, b: _uniform_flat(a, b, seed, stream),
                 lambda v, s, t: lo + (hi - lo) * v)


def student_t3_bf16(rows, cols, seed, stream, clip=64.0, row0=0, nrows=None):
    """Student-t with 3 degrees of freedom, Z / sqrt(chi2_3 / 3), clipped to +-clip."""
    return _fill(rows, cols, row0, nrows,
                 lambda a, b: _student_t3_flat(a, b, seed, stream),
                 lambda v, s, t: np.clip(v, -clip, clip))


def outlier_channels(K, seed, fraction=0.01):
    """round(fraction * K) channel indices chosen by a seeded permutation (argsort of K
    uniforms drawn from the outlier stream), returned sorted."""
    count = int(round(fraction * K))
    u = _uniform_flat(0, K, seed, STREAM_OUTLIER)
    return np.sort(np.argsort(u, kind="stable")[:count])


# ----------------------------------------------------------------------------------------
# The five workloads.  Each entry states shapes and how each tensor is drawn; tensors are
# produced lazily (and row-sliced) by workload(name).tensor(...).

class _Workload:
    def __init__(self, name, seed, desc, linears, x_kind, extra=None):
        self.name = name
        self.seed = seed
        self.desc = desc
        self.linears = linears      # list of dicts: name, M, K, N, w_stream, w_sigma, bias
        self.x_kind = x_kind        # "normal", "normal_outliers", "student_t3"
        self.extra = extra or {}

    def x(self, M, K, row0=0, nrows=None, stream=STREAM_X):
        if self.x_kind == "student_t3":
            return student_t3_bf16(M, K, self.seed, stream, 64.0, row0, nrows)
        col_scale = None
        if self.x_kind == "normal_outliers":
            col_scale = np.ones(K)
            col_scale[outlier_channels(K, self.seed)] = 20.0
        return normal_bf16(M, K, self.seed, stream, 1.0, row0, nrows, col_scale)

    def w(self, lin, row0=0, nrows=None):
        return normal_bf16(lin["N"], lin["K"], self.seed, lin["w_stream"], lin["w_sigma"],
                           row0, nrows)

    def bias(self, lin):
        if not lin.get("bias"):
            return None
        return normal_bf16(1, lin["N"], self.seed, STREAM_BIAS, lin["bias"]).reshape(-1)

    def gamma(self, K):
        return uniform_bf16(1, K, self.seed, STREAM_GAMMA, 0.5, 1.5).reshape(-1)

    def modulation(self, B, K, sigma=0.5):
        """Per-sample scale and shift rows [B, K] of the adaptive norm, N(0, sigma) each."""
        return (normal_bf16(B, K, self.seed, STREAM_MOD_SCALE, sigma),
                normal_bf16(B, K, self.seed, STREAM_MOD_SHIFT, sigma))

    def gate(self, B, N, sigma=0.5):
        """Per-sample gate rows [B, N] of the gated residual update, N(0, sigma)."""
        return normal_bf16(B, N, self.seed, STREAM_GATE, sigma)

    def residual(self, M, N, row0=0, nrows=None):
        """The residual stream [M, N] that a gated update adds to, N(0, 1)."""
        return normal_bf16(M, N, self.seed, STREAM_RESID, 1.0, row0, nrows)


def _lin(name, M, K, N, w_stream, w_sigma, bias=None):
    return dict(name=name, M=M, K=K, N=N, w_stream=w_stream, w_sigma=w_sigma, bias=bias)


WORKLOADS = {
    "linear_256": _Workload(
        "linear_256", 0,
        "single W8A8 linear M=K=N=256; x N(0,1), w N(0,0.02), bias N(0,0.01)",
        [_lin("linear", 256, 256, 256, STREAM_W, 0.02, bias=0.01)], "normal"),
    "attn_proj_4096": _Workload(
        "attn_proj_4096", 1,
        "attention projection M=K=N=4096; x N(0,1) with 1% of K channels x20; "
        "w N(0,1/sqrt(K)); no bias",
        [_lin("proj", 4096, 4096, 4096, STREAM_W, 1.0 / 64.0)], "normal_outliers"),
    "mlp_up_16384": _Workload(
        "mlp_up_16384", 2,
        "MLP up-projection M=16384 K=4096 N=16384; x Student-t(3) clipped +-64; "
        "w N(0,1/sqrt(K)); bias N(0,0.01)",
        [_lin("up", 16384, 4096, 16384, STREAM_W, 1.0 / 64.0, bias=0.01)], "student_t3"),
    "audio_2048x8192": _Workload(
        "audio_2048x8192", 3,
        "audio linears K=2048 N=8192 at M=1024 (INT8 path); guard cases M=1000 and "
        "K=2000 take the BF16 GEMM; x N(0,1), w N(0,1/sqrt(K)); no bias",
        [_lin("int8", 1024, 2048, 8192, STREAM_W, 1.0 / math.sqrt(2048)),
         _lin("guard_m1000", 1000, 2048, 8192, STREAM_W, 1.0 / math.sqrt(2048)),
         _lin("guard_k2000", 1024, 2000, 8192, STREAM_W_K2000, 1.0 / math.sqrt(2000))],
        "normal", extra={"x_stream_k2000": STREAM_X_K2000}),
    "hires_chain_32768": _Workload(
        "hires_chain_32768", 4,
        "M=32768 block chain: fused RMSNorm(eps=1e-6, gamma U(0.5,1.5)) + act-quant on "
        "x N(0,1) K=4096, then QKV 4096->12288, out 4096->4096, up 4096->16384, "
        "down 16384->4096 (down consumes up's BF16 output); w N(0,1/sqrt(K)); no bias",
        [_lin("qkv", 32768, 4096, 12288, STREAM_LAYER0 + 0, 1.0 / 64.0),
         _lin("out", 32768, 4096, 4096, STREAM_LAYER0 + 1, 1.0 / 64.0),
         _lin("up", 32768, 4096, 16384, STREAM_LAYER0 + 2, 1.0 / 64.0),
         _lin("down", 32768, 16384, 4096, STREAM_LAYER0 + 3, 1.0 / 128.0)],
        "normal", extra={"eps": 1e-6}),
}


def workload(name):
    return WORKLOADS[name]
