"""Inputs for the exhaustive near-tie sweep through the RMSNorm + quantizer's code arithmetic
(both of the library's forms).

Every row's sum of squares is built so that its RMS is 1 to far better than FP32
precision (Sum x^2 = K (1 - eps) up to a remainder below 2^-40 of it), so rstd is exactly
1.0 in FP32 on any summation order, and the normalised value of every element is the
element itself (gamma absent or 1; zero modulation).  Each 128 x 128 block of the first
128 columns then holds every BF16 value of both signs in [A/512, A] for one block absmax
A (not a power of two), so every value whose quotient by the block scale can lie near a
half-integer is quantized by the fused kernel.  Columns 128 .. 135 hold the filler that
sets the sum of squares; the rest of each row is zero."""
from fractions import Fraction

import numpy as np

from synth import bf16_bits_to_f32

ABSMAXES = (1.7265625, 2.0625, 3.140625, 1.0078125, 1.9921875)   # BF16 values
FILL_COLS = 8


def _bf16_down(v):
    """The largest BF16 value <= v (v > 0, float)."""
    b = int(np.array([v], dtype=np.float32).view(np.uint32)[0]) >> 16
    while float(bf16_bits_to_f32(np.array([b], np.uint16))[0]) > v:
        b -= 1
    return b


def sweep_block(A):
    """128 x 128 BF16 bit patterns: every BF16 value in [A/512, A] with both signs (A first),
    the list repeated to fill the block."""
    lo = int(np.array([A / 512], np.float32).view(np.uint32)[0] >> 16)
    hi = int(np.array([A], np.float32).view(np.uint32)[0] >> 16)
    assert float(bf16_bits_to_f32(np.array([hi], np.uint16))[0]) == A
    pos = np.arange(hi, lo - 1, -1, dtype=np.uint16)         # A first, then downwards
    vals = np.concatenate([pos, pos | np.uint16(0x8000)])
    reps = -(-128 * 128 // vals.size)
    return np.tile(vals, reps)[:128 * 128].reshape(128, 128)


def unit_rms_rows(K, eps):
    """[128 len(ABSMAXES), K] BF16 bits (see the module docstring) for eps in FP32."""
    eps32 = Fraction(float(np.float32(eps)))
    rows = []
    for A in ABSMAXES:
        blk = sweep_block(A)
        for r in range(128):
            row = np.zeros(K, dtype=np.uint16)
            row[:128] = blk[r]
            vals = bf16_bits_to_f32(row[:128]).astype(np.float64)
            T = Fraction(K) * (1 - eps32) - sum(Fraction(float(v)) ** 2 for v in vals)
            assert T > 0
            for j in range(FILL_COLS):
                if T == 0:
                    break
                b = _bf16_down(float(T) ** 0.5)
                while Fraction(float(bf16_bits_to_f32(np.array([b], np.uint16))[0])) ** 2 > T:
                    b -= 1
                f = Fraction(float(bf16_bits_to_f32(np.array([b], np.uint16))[0]))
                row[128 + j] = b
                T -= f * f
            assert T < Fraction(K) * Fraction(1, 2 ** 40), float(T)
            rows.append(row)
    return np.stack(rows)


def near_tie_count(bits, A):
    """How many of the block's values v have v / fl(A / 127) within 2^-9 of a
    half-integer (float64 quotient)."""
    s = float(np.float32(np.float32(A) / np.float32(127.0)))
    q = np.abs(bf16_bits_to_f32(bits).astype(np.float64)) / s
    return int((np.abs(q - np.floor(q) - 0.5) < 2.0 ** -9).sum())
