"""CPU oracle for the guarded block-wise W8A8 linear layer (ctypes wrapper of oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by the
CPU-baseline leg of bench.py.  The CUDA product path never imports it.  Arrays cross as
numpy: BF16 as uint16 bit patterns, codes as int8, scales and outputs as float32.

Each function states which passage of the pages it follows; see oracle.c for the
arithmetic itself.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
          "-shared", "-Wall", "-Wextra"]
BLOCK = 128

_lib = None


def build(force=False, extra_flags=(), out=None):
    """Compile oracle.c with gcc.  `extra_flags` and `out` exist for the mutation tests,
    which build deliberately broken copies elsewhere."""
    out = out or _LIB
    if not force and out == _LIB and os.path.exists(out) and \
            os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    cmd = ["gcc", *CFLAGS, *extra_flags, _SRC, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _i64(v):
    return ctypes.c_int64(int(v))


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def load(path=None):
    """Load (building first if needed) and return the ctypes library."""
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
    elif _lib is not None:
        return _lib
    else:
        lib = ctypes.CDLL(build())
    for name in ["oracle_block_quantize", "oracle_block_sums", "oracle_w8a8_linear",
                 "oracle_w8a8_linear_at", "oracle_rmsnorm", "oracle_rmsnorm_apply",
                 "oracle_bf16_linear", "oracle_bf16_linear_at", "oracle_num_threads",
                 "oracle_row_quantize", "oracle_row_linear", "oracle_row_linear_at",
                 "oracle_mod_rmsnorm", "oracle_mod_rmsnorm_apply", "oracle_gated_residual"]:
        getattr(lib, name).restype = ctypes.c_int
    lib.oracle_f32_to_bf16.restype = None
    if path is None:
        _lib = lib
    return lib


class Oracle:
    """Bound wrapper, so that tests can run the same calls against a mutant build."""

    def __init__(self, lib=None):
        self.lib = lib or load()

    # -- quantization (TurboDiffusion article, inference list items 3-4) --------------
    def block_quantize(self, x_bits):
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        r, c = x.shape
        q = np.empty((r, c), dtype=np.int8)
        s = np.empty((r // BLOCK, c // BLOCK), dtype=np.float32)
        rc = self.lib.oracle_block_quantize(_ptr(x), _i64(r), _i64(c), _ptr(q), _ptr(s))
        if rc:
            raise ValueError(f"block_quantize: shape {x.shape} not a multiple of 128")
        return q, s

    # -- INT32 sums per K block (TurboT2VA paper, W8A8 paragraph) ----------------------
    def block_sums(self, xq, wq, m0=0, rows=None, n0=0, cols=None):
        xq = np.ascontiguousarray(xq, dtype=np.int8)
        wq = np.ascontiguousarray(wq, dtype=np.int8)
        M, K = xq.shape
        N = wq.shape[0]
        rows = M - m0 if rows is None else rows
        cols = N - n0 if cols is None else cols
        out = np.empty((rows, cols, K // BLOCK), dtype=np.int32)
        rc = self.lib.oracle_block_sums(_ptr(xq), _ptr(wq), _i64(M), _i64(K), _i64(N),
                                        _i64(m0), _i64(rows), _i64(n0), _i64(cols), _ptr(out))
        if rc:
            raise ValueError("block_sums: bad arguments")
        return out

    # -- FP32 output of the W8A8 linear (TurboT2VA paper, W8A8 paragraph) --------------
    def w8a8_linear(self, xq, xs, wq, ws, bias=None, m0=0, rows=None):
        xq, xs, wq, ws, bias = _prep(xq, xs, wq, ws, bias)
        M, K = xq.shape
        N = wq.shape[0]
        rows = M - m0 if rows is None else rows
        out = np.empty((rows, N), dtype=np.float32)
        rc = self.lib.oracle_w8a8_linear(_ptr(xq), _ptr(xs), _ptr(wq), _ptr(ws), _ptr(bias),
                                         _i64(M), _i64(K), _i64(N), _i64(m0), _i64(rows),
                                         _ptr(out))
        if rc:
            raise ValueError("w8a8_linear: bad arguments")
        return out

    def w8a8_linear_at(self, xq, xs, wq, ws, bias, ms, ns):
        xq, xs, wq, ws, bias = _prep(xq, xs, wq, ws, bias)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        ns = np.ascontiguousarray(ns, dtype=np.int64)
        out = np.empty(ms.size, dtype=np.float32)
        rc = self.lib.oracle_w8a8_linear_at(_ptr(xq), _ptr(xs), _ptr(wq), _ptr(ws), _ptr(bias),
                                            _i64(xq.shape[0]), _i64(xq.shape[1]),
                                            _i64(wq.shape[0]), _ptr(ms), _ptr(ns),
                                            _i64(ms.size), _ptr(out))
        if rc:
            raise ValueError("w8a8_linear_at: bad arguments")
        return out

    # -- per-row / per-output-channel operator (TurboT2VA paper, W8A8 paragraph) --------
    def row_quantize(self, x_bits):
        """Codes and one FP32 scale per row (activation rows or weight output channels)."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        r, c = x.shape
        q = np.empty((r, c), dtype=np.int8)
        s = np.empty(r, dtype=np.float32)
        if self.lib.oracle_row_quantize(_ptr(x), _i64(r), _i64(c), _ptr(q), _ptr(s)):
            raise ValueError("row_quantize: bad arguments")
        return q, s

    def row_linear(self, xq, xs, wq, ws, bias=None, m0=0, rows=None):
        xq, xs, wq, ws, bias = _prep(xq, xs, wq, ws, bias)
        M, K = xq.shape
        N = wq.shape[0]
        rows = M - m0 if rows is None else rows
        out = np.empty((rows, N), dtype=np.float32)
        if self.lib.oracle_row_linear(_ptr(xq), _ptr(xs), _ptr(wq), _ptr(ws), _ptr(bias),
                                      _i64(M), _i64(K), _i64(N), _i64(m0), _i64(rows),
                                      _ptr(out)):
            raise ValueError("row_linear: bad arguments")
        return out

    def row_linear_at(self, xq, xs, wq, ws, bias, ms, ns):
        xq, xs, wq, ws, bias = _prep(xq, xs, wq, ws, bias)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        ns = np.ascontiguousarray(ns, dtype=np.int64)
        out = np.empty(ms.size, dtype=np.float32)
        if self.lib.oracle_row_linear_at(_ptr(xq), _ptr(xs), _ptr(wq), _ptr(ws), _ptr(bias),
                                         _i64(xq.shape[0]), _i64(xq.shape[1]),
                                         _i64(wq.shape[0]), _ptr(ms), _ptr(ns), _i64(ms.size),
                                         _ptr(out)):
            raise ValueError("row_linear_at: bad arguments")
        return out

    # -- RMSNorm (TurboDiffusion article, inference list item 5) -----------------------
    def rmsnorm(self, x_bits, gamma_bits, eps, m0=0, rows=None):
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        g = np.ascontiguousarray(gamma_bits, dtype=np.uint16)
        M, K = x.shape
        rows = M - m0 if rows is None else rows
        y = np.empty((rows, K), dtype=np.uint16)
        rstd = np.empty(rows, dtype=np.float32)
        rc = self.lib.oracle_rmsnorm(_ptr(x), _ptr(g), ctypes.c_float(eps), _i64(M), _i64(K),
                                     _i64(m0), _i64(rows), _ptr(y), _ptr(rstd))
        if rc:
            raise ValueError("rmsnorm: bad arguments")
        return y, rstd

    def rmsnorm_apply(self, x_bits, gamma_bits, rstd, m0=0):
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        g = np.ascontiguousarray(gamma_bits, dtype=np.uint16)
        r = np.ascontiguousarray(rstd, dtype=np.float32)
        M, K = x.shape
        y = np.empty((r.size, K), dtype=np.uint16)
        rc = self.lib.oracle_rmsnorm_apply(_ptr(x), _ptr(g), _ptr(r), _i64(M), _i64(K),
                                           _i64(m0), _i64(r.size), _ptr(y))
        if rc:
            raise ValueError("rmsnorm_apply: bad arguments")
        return y

    # -- modulated RMSNorm and gated residual (TurboT2VA paper, fused-operator paragraph)
    def mod_rmsnorm(self, x_bits, gamma_bits, scale_bits, shift_bits, T, eps, m0=0, rows=None):
        """y = bf16(fl(fl(n * fl(1 + scale[m / T])) + shift[m / T])), n = x * rstd (times
        gamma when given); scale and shift [M / T, K]."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        g = None if gamma_bits is None else np.ascontiguousarray(gamma_bits, dtype=np.uint16)
        sc = np.ascontiguousarray(scale_bits, dtype=np.uint16)
        sh = np.ascontiguousarray(shift_bits, dtype=np.uint16)
        M, K = x.shape
        if T <= 0 or M % T or sc.shape != (M // T, K) or sh.shape != (M // T, K) or \
                (g is not None and g.shape != (K,)):
            raise ValueError("mod_rmsnorm: bad shapes")
        rows = M - m0 if rows is None else rows
        y = np.empty((rows, K), dtype=np.uint16)
        rstd = np.empty(rows, dtype=np.float32)
        rc = self.lib.oracle_mod_rmsnorm(_ptr(x), _ptr(g), _ptr(sc), _ptr(sh), _i64(T),
                                         ctypes.c_float(eps), _i64(M), _i64(K), _i64(m0),
                                         _i64(rows), _ptr(y), _ptr(rstd))
        if rc:
            raise ValueError("mod_rmsnorm: bad arguments")
        return y, rstd

    def mod_rmsnorm_apply(self, x_bits, gamma_bits, scale_bits, shift_bits, T, rstd, m0=0):
        """mod_rmsnorm's normalisation with a given rstd for rows m0 .. m0 + rstd.size."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        g = None if gamma_bits is None else np.ascontiguousarray(gamma_bits, dtype=np.uint16)
        sc = np.ascontiguousarray(scale_bits, dtype=np.uint16)
        sh = np.ascontiguousarray(shift_bits, dtype=np.uint16)
        r = np.ascontiguousarray(rstd, dtype=np.float32)
        M, K = x.shape
        if T <= 0 or M % T or sc.shape != (M // T, K) or sh.shape != (M // T, K):
            raise ValueError("mod_rmsnorm_apply: bad shapes")
        y = np.empty((r.size, K), dtype=np.uint16)
        rc = self.lib.oracle_mod_rmsnorm_apply(_ptr(x), _ptr(g), _ptr(sc), _ptr(sh), _i64(T),
                                               _ptr(r), _i64(M), _i64(K), _i64(m0),
                                               _i64(r.size), _ptr(y))
        if rc:
            raise ValueError("mod_rmsnorm_apply: bad arguments")
        return y

    def gated_residual(self, v, r_bits, gate_bits, T, M, ms=None, ns=None):
        """out = bf16(fl(r + fl(gate[m / T, n] * v))).  With ms, ns: v and r_bits hold the
        values at those points; without: v and r_bits are the full [M, N] arrays."""
        g = np.ascontiguousarray(gate_bits, dtype=np.uint16)
        N = g.shape[1]
        if ms is None:
            shape = np.shape(v)
            ms, ns = np.indices(shape).reshape(2, -1)
        else:
            shape = np.shape(ms)
        v = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
        r = np.ascontiguousarray(r_bits, dtype=np.uint16).reshape(-1)
        ms = np.ascontiguousarray(ms, dtype=np.int64).reshape(-1)
        ns = np.ascontiguousarray(ns, dtype=np.int64).reshape(-1)
        if T <= 0 or M % T or g.shape[0] != M // T or not (v.size == r.size == ms.size == ns.size):
            raise ValueError("gated_residual: bad shapes")
        out = np.empty(ms.size, dtype=np.uint16)
        if self.lib.oracle_gated_residual(_ptr(v), _ptr(r), _ptr(g), _i64(T), _i64(M), _i64(N),
                                          _ptr(ms), _ptr(ns), _i64(ms.size), _ptr(out)):
            raise ValueError("gated_residual: bad arguments")
        return out.reshape(shape)

    # -- BF16 fallback (TurboT2VA paper, guard paragraph) ------------------------------
    def bf16_linear(self, x_bits, w_bits, bias=None, m0=0, rows=None):
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        w = np.ascontiguousarray(w_bits, dtype=np.uint16)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
        M, K = x.shape
        N = w.shape[0]
        rows = M - m0 if rows is None else rows
        out = np.empty((rows, N), dtype=np.float32)
        rc = self.lib.oracle_bf16_linear(_ptr(x), _ptr(w), _ptr(b), _i64(M), _i64(K), _i64(N),
                                         _i64(m0), _i64(rows), _ptr(out))
        if rc:
            raise ValueError("bf16_linear: bad arguments")
        return out

    def bf16_linear_at(self, x_bits, w_bits, bias, ms, ns):
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        w = np.ascontiguousarray(w_bits, dtype=np.uint16)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        ns = np.ascontiguousarray(ns, dtype=np.int64)
        out = np.empty(ms.size, dtype=np.float32)
        rc = self.lib.oracle_bf16_linear_at(_ptr(x), _ptr(w), _ptr(b), _i64(x.shape[0]),
                                            _i64(x.shape[1]), _i64(w.shape[0]), _ptr(ms),
                                            _ptr(ns), _i64(ms.size), _ptr(out))
        if rc:
            raise ValueError("bf16_linear_at: bad arguments")
        return out

    def f32_to_bf16(self, a):
        a = np.ascontiguousarray(a, dtype=np.float32)
        out = np.empty(a.shape, dtype=np.uint16)
        self.lib.oracle_f32_to_bf16(_ptr(a), _i64(a.size), _ptr(out))
        return out

    def num_threads(self):
        return int(self.lib.oracle_num_threads())


def _prep(xq, xs, wq, ws, bias):
    return (np.ascontiguousarray(xq, dtype=np.int8), np.ascontiguousarray(xs, dtype=np.float32),
            np.ascontiguousarray(wq, dtype=np.int8), np.ascontiguousarray(ws, dtype=np.float32),
            None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16))


_default = None


def default():
    """The oracle built from oracle.c as committed."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
