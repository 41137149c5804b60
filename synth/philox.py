"""Philox4x32-10 counter-based generator, vectorised over counters with numpy.

Definition (Salmon et al., SC 2011, section 3): a 128-bit counter (c0, c1, c2, c3) and a
64-bit key (k0, k1) go through ten rounds.  One round multiplies c0 and c2 by two fixed
32-bit constants, keeps both halves of each 64-bit product, and mixes:

    (c0, c1, c2, c3) <- (hi(B*c2) ^ c1 ^ k0, lo(B*c2), hi(A*c0) ^ c3 ^ k1, lo(A*c0))

after which the key is advanced by the two Weyl constants (golden ratio and sqrt(3) - 1,
scaled to 32 bits).  The round constants below are the published ones.
"""
import numpy as np

_MUL_A = np.uint64(0xD2511F53)
_MUL_B = np.uint64(0xCD9E8D57)
_WEYL_0 = 0x9E3779B9
_WEYL_1 = 0xBB67AE85
_LO32 = np.uint64(0xFFFFFFFF)
_SH32 = np.uint64(32)


def _rounds(w0, w1, w2, w3, k0, k1):
    """Ten rounds in place on uint64 word arrays (each word < 2^32)."""
    pa = np.empty_like(w0)
    pb = np.empty_like(w0)
    t = np.empty_like(w0)
    for _ in range(10):
        np.multiply(w0, _MUL_A, out=pa)
        np.multiply(w2, _MUL_B, out=pb)
        # new c0 = hi(B*c2) ^ c1 ^ k0 ; new c2 = hi(A*c0) ^ c3 ^ k1
        np.right_shift(pb, _SH32, out=t)
        np.bitwise_xor(t, w1, out=w0)
        np.bitwise_xor(w0, np.uint64(k0), out=w0)
        np.right_shift(pa, _SH32, out=t)
        np.bitwise_xor(t, w3, out=w2)
        np.bitwise_xor(w2, np.uint64(k1), out=w2)
        # new c1 = lo(B*c2) ; new c3 = lo(A*c0)
        np.bitwise_and(pb, _LO32, out=w1)
        np.bitwise_and(pa, _LO32, out=w3)
        k0 = (k0 + _WEYL_0) & 0xFFFFFFFF
        k1 = (k1 + _WEYL_1) & 0xFFFFFFFF


def philox4x32_10(counters, key0, key1, c1=None, c2=None, c3=None):
    """Return the four 32-bit output words for each counter.

    counters: uint64 array of counter values; the low 32 bits go to word c0 and the high
    32 bits to word c1 (unless c1 is given explicitly).  c2, c3 default to 0.
    key0, key1: python ints (the seed and the stream id).
    Returns a (4, n) uint32 array.
    """
    n = np.asarray(counters, dtype=np.uint64).reshape(-1)
    out = np.empty((4, n.size), dtype=np.uint32)
    k0 = int(key0) & 0xFFFFFFFF
    k1 = int(key1) & 0xFFFFFFFF
    step = 1 << 16
    for s in range(0, n.size, step):
        e = min(n.size, s + step)
        w0 = n[s:e] & _LO32
        w1 = (n[s:e] >> _SH32) if c1 is None else np.asarray(c1, np.uint64).reshape(-1)[s:e] & _LO32
        w2 = np.zeros_like(w0) if c2 is None else np.asarray(c2, np.uint64).reshape(-1)[s:e] & _LO32
        w3 = np.zeros_like(w0) if c3 is None else np.asarray(c3, np.uint64).reshape(-1)[s:e] & _LO32
        _rounds(w0, w1, w2, w3, k0, k1)
        out[0, s:e] = w0
        out[1, s:e] = w1
        out[2, s:e] = w2
        out[3, s:e] = w3
    return out


def uniform_open01(words):
    """Map 32-bit words to doubles in (0, 1): (w + 0.5) / 2^32."""
    return (words.astype(np.float64) + 0.5) * (1.0 / 4294967296.0)


def normal_pairs(wa, wb):
    """Box-Muller (Box and Muller, 1958) on two words: returns (r cos t, r sin t).

    The radius draws from (0, 1] ((w + 1) / 2^32) so that the logarithm stays finite;
    the angle draws from [0, 1).
    """
    u1 = (wa.astype(np.float64) + 1.0) * (1.0 / 4294967296.0)
    u2 = wb.astype(np.float64) * (1.0 / 4294967296.0)
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    return r * np.cos(t), r * np.sin(t)
