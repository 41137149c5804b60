"""Helpers shared by the GPU tests: moving BF16 bit patterns between numpy and torch,
and the output tolerance of the W8A8 linear."""
import numpy as np
import torch

RTOL = 1e-2
ATOL = 1e-2


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def assert_close_bf16(y_gpu_bits, ref_f32, orc, what=""):
    """|y - bf16(ref)| <= ATOL + RTOL * |bf16(ref)| elementwise (ref = oracle FP32 output)."""
    ref_b = bf16_to_f32(orc.f32_to_bf16(ref_f32)).astype(np.float64)
    y = bf16_to_f32(y_gpu_bits).astype(np.float64)
    err = np.abs(y - ref_b)
    lim = ATOL + RTOL * np.abs(ref_b)
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                           f"worst err {float(err.max())} at {np.unravel_index(np.argmax(err - lim), err.shape)}")
    return float(err.max()), float((err / (np.abs(ref_b) + 1e-30)).max())


def assert_codes_equal(q_gpu, s_gpu, q_ref, s_ref, what=""):
    """GPU codes (int8) and scales (float32) against the oracle's own, bit for bit."""
    q = q_gpu.detach().cpu().numpy() if isinstance(q_gpu, torch.Tensor) else np.asarray(q_gpu)
    s = s_gpu.detach().cpu().numpy() if isinstance(s_gpu, torch.Tensor) else np.asarray(s_gpu)
    s = np.ascontiguousarray(s, dtype=np.float32)
    s_ref = np.ascontiguousarray(s_ref, dtype=np.float32)
    bad_s = s.view(np.uint32) != s_ref.view(np.uint32)
    assert not bad_s.any(), f"{what}: {int(bad_s.sum())} scales differ, first at {np.argwhere(bad_s)[0]}"
    bad_q = q != q_ref
    assert not bad_q.any(), f"{what}: {int(bad_q.sum())} codes differ, first at {np.argwhere(bad_q)[0]}"
