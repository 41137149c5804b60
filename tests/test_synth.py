"""The seeded input generator: Philox4x32-10 known answers, slice consistency and the
distributions each workload states.  No GPU."""
import os

import numpy as np

from synth import (bf16_bits_to_f32, f64_to_bf16_bits, outlier_channels, philox4x32_10,
                   workload)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_philox_known_answers():
    n = 0
    for line in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")):
        line = line.split("#")[0].split()
        if not line:
            continue
        v = [int(t, 16) for t in line]
        ctr = np.array([(v[1] << 32) | v[0]], dtype=np.uint64)
        out = philox4x32_10(ctr, v[4], v[5], c2=[v[2]], c3=[v[3]])[:, 0]
        assert [int(t) for t in out] == v[6:10]
        n += 1
    assert n == 3


def test_bf16_conversion_rne():
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -3.0, 1e-3])
    b = f64_to_bf16_bits(v)
    np.testing.assert_array_equal(bf16_bits_to_f32(b)[:3], [1.0, 1.0 + 2.0 ** -6, -3.0])
    assert abs(bf16_bits_to_f32(b)[3] - 1e-3) <= 1e-3 * 2.0 ** -8


def test_row_slices_match_full():
    w = workload("audio_2048x8192")
    full = w.x(64, 2048)
    np.testing.assert_array_equal(w.x(64, 2048, row0=7, nrows=9), full[7:16])
    t = workload("mlp_up_16384")
    np.testing.assert_array_equal(t.x(32, 4096, row0=30, nrows=2), t.x(32, 4096)[30:32])


def test_distributions():
    w = workload("attn_proj_4096")
    x = bf16_bits_to_f32(w.x(4096, 4096, row0=0, nrows=256)).astype(np.float64)
    ch = outlier_channels(4096, 1)
    assert ch.size == 41 and len(set(ch.tolist())) == 41
    rest = np.setdiff1d(np.arange(4096), ch)
    assert abs(x[:, rest].std() - 1.0) < 0.01 and abs(x[:, rest].mean()) < 0.01
    assert abs(x[:, ch].std() - 20.0) < 0.5
    wt = bf16_bits_to_f32(w.w(w.linears[0], nrows=256)).astype(np.float64)
    assert abs(wt.std() * 64 - 1.0) < 0.01
    t = workload("mlp_up_16384")
    xt = bf16_bits_to_f32(t.x(16384, 4096, nrows=64)).astype(np.float64)
    assert np.abs(xt).max() <= 64.0
    assert abs(np.median(np.abs(xt)) - 0.7649) < 0.02      # median |t_3| = 0.7649
    g = bf16_bits_to_f32(workload("hires_chain_32768").gamma(4096)).astype(np.float64)
    assert g.min() >= 0.5 and g.max() <= 1.5 and abs(g.mean() - 1.0) < 0.02
    b = bf16_bits_to_f32(workload("linear_256").bias(workload("linear_256").linears[0]))
    assert abs(b.std() - 0.01) < 0.002
