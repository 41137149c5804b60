"""Python binding of libw8a8 (the C ABI in include/w8a8.h).

Argument marshalling only: every step of the W8A8 linear layer runs in the library's
sm_100a kernels.  PyTorch provides device memory and streams.  Tensors must be CUDA,
contiguous, and of the dtype each entry point states; BF16 is the only activation and
weight dtype (a tensor of another dtype is rejected here, before the library is called).
There is no CPU path: without the built library every call raises.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw8a8.so")

PATH_INT8, PATH_BF16, PATH_NONE = 0, 1, 2
DEVERR_NONE, DEVERR_TIMEOUT = 0, 1
_STATUS = {0: "ok", 1: "invalid argument", 2: "shape", 3: "not device memory",
           4: "alignment", 5: "workspace", 6: "CUDA error"}


class W8A8Error(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn}: status {code} ({_STATUS.get(code, '?')})")
        self.code = code


class _Weight(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("w_bf16", ctypes.c_void_p),
                ("wq", ctypes.c_void_p), ("ws", ctypes.c_void_p)]


_lib = None
_SIGS = {
    "w8a8_quantize_weight": [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                             ctypes.c_void_p, ctypes.c_void_p],
    "w8a8_quantize_act": [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                          ctypes.c_void_p, ctypes.c_void_p],
    "w8a8_rmsnorm_quantize_act": [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                  ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p],
    "w8a8_rmsnorm_mod_quantize_act": [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_int64, ctypes.c_float,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p],
    "w8a8_linear_prequant_gated": [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.POINTER(_Weight), ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                   ctypes.c_void_p, ctypes.c_void_p],
    "w8a8_linear": [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(_Weight),
                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                    ctypes.POINTER(ctypes.c_int), ctypes.c_void_p],
    "w8a8_linear_host": [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(_Weight),
                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                         ctypes.c_int64, ctypes.POINTER(ctypes.c_int), ctypes.c_void_p],
    "w8a8_linear_noalloc": [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                            ctypes.POINTER(_Weight), ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.POINTER(ctypes.c_int), ctypes.c_void_p],
    "w8a8_linear_prequant": [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                             ctypes.POINTER(_Weight), ctypes.c_void_p, ctypes.c_void_p,
                             ctypes.c_void_p],
    "w8a8_bf16_linear": [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                         ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p],
    "w8a8_debug_block_sums": [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                              ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                              ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p],
    "w8a8_debug_wait_timeout": [ctypes.c_uint64, ctypes.c_void_p],
    "w8a8_rowwise_quantize": [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                              ctypes.c_void_p, ctypes.c_void_p],
    "w8a8_rowwise_linear": [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_void_p],
}


def lib():
    """The loaded library (ctypes.CDLL).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.w8a8_linear_workspace_bytes.argtypes = [ctypes.c_int64] * 3
        L.w8a8_linear_workspace_bytes.restype = ctypes.c_size_t
        L.w8a8_linear_host_workspace_bytes.argtypes = [ctypes.c_int64] * 4
        L.w8a8_linear_host_workspace_bytes.restype = ctypes.c_size_t
        L.w8a8_linear_host_chunk_rows.argtypes = [ctypes.c_int64] * 2
        L.w8a8_linear_host_chunk_rows.restype = ctypes.c_int64
        L.w8a8_device_error.argtypes = []
        L.w8a8_device_error.restype = ctypes.c_int
        L.w8a8_last_cuda_error.argtypes = []
        L.w8a8_last_cuda_error.restype = ctypes.c_char_p
        L.w8a8_status_string.argtypes = [ctypes.c_int]
        L.w8a8_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(fn, code):
    if code != 0:
        err = W8A8Error(fn, code)
        if code == 6:
            err.args = (err.args[0] + ": " + lib().w8a8_last_cuda_error().decode(),)
        raise err


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out(t, shape, dtype, device, name):
    """A caller-supplied output buffer: checked here, before the library writes into it,
    for type, dtype, exact shape, device and contiguity (a wrong one would be written out
    of bounds); None -> a new tensor."""
    if t is None:
        return torch.empty(tuple(shape), dtype=dtype, device=device)
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != torch.device(device):
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _in(t, shape, dtype, device, name):
    """A required input buffer, checked like an output buffer."""
    if t is None:
        raise TypeError(f"{name} is required")
    return _out(t, shape, dtype, device, name)


def _block_scales(xs, M, K, device, name):
    """A block-scale table [M/128, K/128] float32 on the device."""
    return _out(xs, (M // 128, K // 128), torch.float32, device, name)


def quantize_act(x, xq=None, xs=None):
    """Block-wise 128x128 INT8 quantization of a BF16 [M, K] matrix -> (xq int8 [M, K],
    xs float32 [M/128, K/128])."""
    _need(x, torch.bfloat16, "x")
    M, K = x.shape
    xq = _out(xq, (M, K), torch.int8, x.device, "xq")
    xs = _block_scales(xs, M, K, x.device, "xs")
    _check("w8a8_quantize_act", lib().w8a8_quantize_act(_ptr(x), M, K, _ptr(xq), _ptr(xs),
                                                         _stream(x.device)))
    return xq, xs


def quantize_weight(w):
    """Block-wise 128x128 INT8 quantization of a BF16 weight [N, K] -> (wq, ws)."""
    _need(w, torch.bfloat16, "w")
    N, K = w.shape
    wq = torch.empty((N, K), dtype=torch.int8, device=w.device)
    ws = torch.empty((N // 128, K // 128), dtype=torch.float32, device=w.device)
    _check("w8a8_quantize_weight", lib().w8a8_quantize_weight(_ptr(w), N, K, _ptr(wq), _ptr(ws),
                                                               _stream(w.device)))
    return wq, ws


def rowwise_quantize(x, q=None, s=None):
    """Per-row INT8 quantization of a BF16 [rows, K] matrix (TurboT2VA's post-scale
    operator: s = max(||row||_inf, 1e-4) / 127) -> (q int8 [rows, K], s float32 [rows]).
    For a weight [N, K] this gives its per-output-channel codes and scales."""
    _need(x, torch.bfloat16, "x")
    rows, K = x.shape
    q = _out(q, (rows, K), torch.int8, x.device, "q")
    s = _out(s, (rows,), torch.float32, x.device, "s")
    _check("w8a8_rowwise_quantize", lib().w8a8_rowwise_quantize(_ptr(x), rows, K, _ptr(q), _ptr(s),
                                                                 _stream(x.device)))
    return q, s


def rowwise_linear_prequant(xq, xs, wq, ws, bias=None, out=None):
    """y = bf16(float(xq wq^T) * (xs[m] ws[n]) + bias) with INT32 accumulation over all of K."""
    _need(xq, torch.int8, "xq")
    _need(wq, torch.int8, "wq")
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"wq must be [N, {K}], got {tuple(wq.shape)}")
    _in(xs, (M,), torch.float32, xq.device, "xs")
    _in(ws, (N,), torch.float32, xq.device, "ws")
    if bias is not None:
        _out(bias, (N,), torch.bfloat16, xq.device, "bias")
    y = _out(out, (M, N), torch.bfloat16, xq.device, "out")
    _check("w8a8_rowwise_linear", lib().w8a8_rowwise_linear(
        _ptr(xq), _ptr(xs), M, K, _ptr(wq), _ptr(ws), N, _ptr(bias), _ptr(y), _stream(xq.device)))
    return y


def rowwise_linear(x, wq, ws, bias=None, out=None):
    """The per-row operator on BF16 activations: per-row quantization, then the GEMM."""
    xq, xs = rowwise_quantize(x)
    return rowwise_linear_prequant(xq, xs, wq, ws, bias, out)


def rmsnorm_quantize_act(x, gamma, eps=1e-6, xq=None, xs=None, rstd=None):
    """RMSNorm (FP64 row sums, FP32 rstd, bf16((x * rstd) * gamma); gamma may be None)
    fused with the block quantizer (the normalised values are never stored) -> (xq, xs,
    rstd).  From 192 rows per SM the row sums follow the definition's column order, so rstd
    is exactly the definition's; below that a one-grid kernel splits each row over a
    cluster and rstd may differ by one FP32 ulp on rare rows (see include/w8a8.h)."""
    _need(x, torch.bfloat16, "x")
    if gamma is not None:
        _need(gamma, torch.bfloat16, "gamma")
    M, K = x.shape
    dev = x.device
    if gamma is not None:
        _out(gamma, (K,), torch.bfloat16, dev, "gamma")
    xq = _out(xq, (M, K), torch.int8, dev, "xq")
    xs = _block_scales(xs, M, K, dev, "xs")
    rstd = _out(rstd, (M,), torch.float32, dev, "rstd")
    _check("w8a8_rmsnorm_quantize_act",
           lib().w8a8_rmsnorm_quantize_act(_ptr(x), _ptr(gamma), float(eps), M, K, _ptr(xq),
                                           _ptr(xs), _ptr(rstd), _stream(dev)))
    return xq, xs, rstd


def rmsnorm_mod_quantize_act(x, gamma, scale, shift, eps=1e-6, xq=None, xs=None, rstd=None):
    """Modulated RMSNorm fused with the block quantizer: y = bf16(n * (1 + scale[b]) +
    shift[b]) with n = x * rstd (* gamma), b = m // T, T = M // scale.shape[0] rows per
    modulation row (a multiple of 128) -> (xq, xs, rstd)."""
    _need(x, torch.bfloat16, "x")
    if gamma is not None:
        _need(gamma, torch.bfloat16, "gamma")
    _need(scale, torch.bfloat16, "scale")
    _need(shift, torch.bfloat16, "shift")
    M, K = x.shape
    B = scale.shape[0]
    if scale.shape != (B, K) or shift.shape != (B, K) or B == 0 or M % B:
        raise ValueError(f"scale and shift must be [B, {K}] with B dividing M = {M}")
    dev = x.device
    if gamma is not None:
        _out(gamma, (K,), torch.bfloat16, dev, "gamma")
    xq = _out(xq, (M, K), torch.int8, dev, "xq")
    xs = _block_scales(xs, M, K, dev, "xs")
    rstd = _out(rstd, (M,), torch.float32, dev, "rstd")
    _check("w8a8_rmsnorm_mod_quantize_act",
           lib().w8a8_rmsnorm_mod_quantize_act(_ptr(x), _ptr(gamma), _ptr(scale), _ptr(shift),
                                               M // B, float(eps), M, K, _ptr(xq), _ptr(xs),
                                               _ptr(rstd), _stream(dev)))
    return xq, xs, rstd


class W8A8Weight:
    """A linear layer's weight: the retained BF16 copy plus, when N and K are multiples of
    128, its INT8 codes and block scales (quantized once, at construction)."""

    def __init__(self, w_bf16, wq=None, ws=None):
        _need(w_bf16, torch.bfloat16, "w")
        self.w = w_bf16
        self.N, self.K = w_bf16.shape
        if wq is None and self.N % 128 == 0 and self.K % 128 == 0 and self.N and self.K:
            wq, ws = quantize_weight(w_bf16)
        elif wq is not None:
            _in(wq, (self.N, self.K), torch.int8, w_bf16.device, "wq")
            _in(ws, (self.N // 128, self.K // 128), torch.float32, w_bf16.device, "ws")
        self.wq, self.ws = wq, ws
        self._rec = _Weight(self.N, self.K, w_bf16.data_ptr(),
                            0 if wq is None else wq.data_ptr(),
                            0 if ws is None else ws.data_ptr())

    def record(self):
        return ctypes.byref(self._rec)


def _weight_on(weight, K, device):
    """The weight matches the activations' K and lives on their device."""
    if not isinstance(weight, W8A8Weight):
        raise TypeError("weight must be a W8A8Weight")
    if weight.K != K:
        raise ValueError(f"weight has K = {weight.K}, the activations K = {K}")
    if weight.w.device != torch.device(device):
        raise ValueError(f"weight is on {weight.w.device}, the activations on {device}")


def linear_workspace_bytes(M, K, N):
    return int(lib().w8a8_linear_workspace_bytes(M, K, N))


def linear(x, weight, bias=None, out=None, workspace=None, return_path=False):
    """The guarded W8A8 linear: y = x W^T + bias in BF16.  x: [..., K] BF16 (leading
    dimensions flattened to M).  INT8 path when M, K, N are multiples of 128, else BF16."""
    _need(x, torch.bfloat16, "x")
    if bias is not None:
        _need(bias, torch.bfloat16, "bias")
    K = x.shape[-1]
    M = math.prod(x.shape[:-1])
    N = weight.N
    dev = x.device
    _weight_on(weight, K, dev)
    if bias is not None:
        _out(bias, (N,), torch.bfloat16, dev, "bias")
    out = _out(out, (*x.shape[:-1], N), torch.bfloat16, dev, "out")
    need = linear_workspace_bytes(M, K, N)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    elif workspace is not None:
        _out(workspace, (workspace.numel(),), torch.uint8, dev, "workspace")
    path = ctypes.c_int(-1)
    _check("w8a8_linear", lib().w8a8_linear(
        _ptr(x), M, K, weight.record(), _ptr(bias), _ptr(out), _ptr(workspace),
        0 if workspace is None else workspace.numel(), ctypes.byref(path), _stream(dev)))
    return (out, path.value) if return_path else out


def linear_host_workspace_bytes(M, K, N, chunk_rows=0):
    return int(lib().w8a8_linear_host_workspace_bytes(M, K, N, chunk_rows))


def linear_host(x, weight, bias=None, out=None, workspace=None, chunk_rows=0, return_path=False):
    """w8a8_linear on host buffers: x [..., K] BF16 and the output in CPU memory (pinned
    memory lets the copies overlap with the compute).  The rows stream through the GPU in
    chunks; the result equals linear() on a device copy of x.  The work is enqueued on the
    weight device's current stream, which completes only after the output has landed in
    host memory."""
    if not isinstance(x, torch.Tensor) or x.device.type != "cpu":
        raise ValueError("x must be a CPU tensor (use linear() for device tensors)")
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise TypeError("x must be a contiguous torch.bfloat16 tensor")
    if bias is not None:
        _need(bias, torch.bfloat16, "bias")
    K = x.shape[-1]
    M = math.prod(x.shape[:-1])
    N = weight.N
    dev = weight.w.device
    if weight.K != K:
        raise ValueError(f"weight has K = {weight.K}, the activations K = {K}")
    if bias is not None:
        _out(bias, (N,), torch.bfloat16, dev, "bias")
    if out is None:
        out = torch.empty((*x.shape[:-1], N), dtype=torch.bfloat16, pin_memory=True)
    else:
        _out(out, (*x.shape[:-1], N), torch.bfloat16, "cpu", "out")
    need = linear_host_workspace_bytes(M, K, N, chunk_rows)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    elif workspace is not None:
        _out(workspace, (workspace.numel(),), torch.uint8, dev, "workspace")
    path = ctypes.c_int(-1)
    _check("w8a8_linear_host", lib().w8a8_linear_host(
        _ptr(x), M, K, weight.record(), _ptr(bias), _ptr(out), _ptr(workspace),
        0 if workspace is None else workspace.numel(), chunk_rows, ctypes.byref(path),
        _stream(dev)))
    return (out, path.value) if return_path else out


NOALLOC_MAX_ELEMS = 16777216


def linear_noalloc(x, weight, bias=None, out=None, return_path=False):
    """w8a8_linear for callers that must not allocate device memory: the quantized
    activations live in scratch built into the library (M * K <= 16 Mi on the INT8 path).
    All calls on a device share that scratch, so calls that may overlap on the GPU must be
    ordered (e.g. issued on one stream)."""
    _need(x, torch.bfloat16, "x")
    if bias is not None:
        _need(bias, torch.bfloat16, "bias")
    K = x.shape[-1]
    M = math.prod(x.shape[:-1])
    dev = x.device
    _weight_on(weight, K, dev)
    if bias is not None:
        _out(bias, (weight.N,), torch.bfloat16, dev, "bias")
    out = _out(out, (*x.shape[:-1], weight.N), torch.bfloat16, dev, "out")
    path = ctypes.c_int(-1)
    _check("w8a8_linear_noalloc", lib().w8a8_linear_noalloc(
        _ptr(x), M, K, weight.record(), _ptr(bias), _ptr(out), ctypes.byref(path), _stream(dev)))
    return (out, path.value) if return_path else out


def linear_prequant(xq, xs, weight, bias=None, out=None):
    """The INT8 block-scaled GEMM on already-quantized activations."""
    _need(xq, torch.int8, "xq")
    M, K = xq.shape
    _in(xs, (M // 128, K // 128), torch.float32, xq.device, "xs")
    _weight_on(weight, K, xq.device)
    if bias is not None:
        _out(bias, (weight.N,), torch.bfloat16, xq.device, "bias")
    out = _out(out, (M, weight.N), torch.bfloat16, xq.device, "out")
    _check("w8a8_linear_prequant", lib().w8a8_linear_prequant(
        _ptr(xq), _ptr(xs), M, K, weight.record(), _ptr(bias), _ptr(out), _stream(xq.device)))
    return out


def linear_prequant_gated(xq, xs, weight, resid, gate, bias=None, out=None):
    """The INT8 block-scaled GEMM with the gated residual update in its epilogue:
    out = bf16(resid + gate[m // T] * (xq wq^T + bias)), T = M // gate.shape[0].  out may
    be resid itself (in-place update); by default a new tensor."""
    _need(xq, torch.int8, "xq")
    _need(resid, torch.bfloat16, "resid")
    _need(gate, torch.bfloat16, "gate")
    M, K = xq.shape
    _in(xs, (M // 128, K // 128), torch.float32, xq.device, "xs")
    _weight_on(weight, K, xq.device)
    B = gate.shape[0]
    if resid.shape != (M, weight.N) or gate.shape != (B, weight.N) or B == 0 or M % B:
        raise ValueError(f"resid must be [{M}, {weight.N}] and gate [B, {weight.N}] with B dividing M")
    if resid.device != xq.device or gate.device != xq.device:
        raise ValueError("resid and gate must be on the device of xq")
    if bias is not None:
        _out(bias, (weight.N,), torch.bfloat16, xq.device, "bias")
    out = _out(out, (M, weight.N), torch.bfloat16, xq.device, "out")
    _check("w8a8_linear_prequant_gated", lib().w8a8_linear_prequant_gated(
        _ptr(xq), _ptr(xs), M, K, weight.record(), _ptr(bias), _ptr(resid), _ptr(gate), M // B,
        _ptr(out), _stream(xq.device)))
    return out


def bf16_linear(x, w, bias=None, out=None):
    """The BF16 GEMM the guard falls back to: y = x w^T + bias, any shape."""
    _need(x, torch.bfloat16, "x")
    _need(w, torch.bfloat16, "w")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K or w.device != x.device:
        raise ValueError(f"w must be [N, {K}] on {x.device}")
    if bias is not None:
        _out(bias, (N,), torch.bfloat16, x.device, "bias")
    out = _out(out, (M, N), torch.bfloat16, x.device, "out")
    _check("w8a8_bf16_linear", lib().w8a8_bf16_linear(_ptr(x), _ptr(w), _ptr(bias), _ptr(out),
                                                       M, K, N, _stream(x.device)))
    return out


def debug_block_sums(xq, wq, m0=0, rows=None, n0=0, cols=None):
    """INT32 per-K-block partial products [rows, cols, K/128] of the window rows m0 ..
    m0 + rows - 1, columns n0 .. n0 + cols - 1 (default: everything), from the tensor-core
    main loop."""
    _need(xq, torch.int8, "xq")
    _need(wq, torch.int8, "wq")
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K or wq.device != xq.device:
        raise ValueError(f"wq must be [N, {K}] on {xq.device}")
    rows = M - m0 if rows is None else rows
    cols = N - n0 if cols is None else cols
    out = torch.empty((rows, cols, K // 128), dtype=torch.int32, device=xq.device)
    _check("w8a8_debug_block_sums", lib().w8a8_debug_block_sums(
        _ptr(xq), _ptr(wq), M, K, N, m0, rows, n0, cols, _ptr(out), _stream(xq.device)))
    return out


def debug_wait_timeout(timeout_ns, device=None):
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _check("w8a8_debug_wait_timeout", lib().w8a8_debug_wait_timeout(int(timeout_ns), _stream(dev)))


def device_error():
    """Synchronize and return (and clear) the library's device error word."""
    return int(lib().w8a8_device_error())
