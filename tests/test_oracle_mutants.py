"""Plant one plausible mistake at a time in a copy of oracle.c (on the CPU), rebuild it,
and require that some pin catches each mistake.  This shows the pins constrain every
step of the oracle: scales, rounding, division, block indexing, per-block rescale,
bias, RMSNorm, the modulated RMSNorm and gated residual, and the BF16 fallback."""
import os
import shutil

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (id, text in oracle.c, replacement); every replacement keeps all reads in bounds.
MUTANTS = [
    ("divisor_128", "return absmax / 127.0f;", "return absmax / 128.0f;"),
    ("round_half_away", "float q = rintf(x / s);", "float q = roundf(x / s);"),
    ("reciprocal_multiply", "float q = rintf(x / s);", "float q = rintf(x * (1.0f / s));"),
    ("truncate", "float q = rintf(x / s);", "float q = truncf(x / s);"),
    ("clamp_126", "if (q > 127.0f)\n        q = 127.0f;", "if (q > 126.0f)\n        q = 126.0f;"),
    ("no_abs_in_absmax", "float a = fabsf(bf16_to_f32(x[i * cols + j]));",
     "float a = bf16_to_f32(x[i * cols + j]);"),
    ("scale_index_transposed", "s[rb * cb_n + cb] = sc;", "s[cb * rb_n + rb] = sc;"),
    ("zero_block_scale_0", "if (absmax == 0.0f)\n        return 1.0f;",
     "if (absmax == 0.0f)\n        return 0.5f;"),
    ("short_block_sum", "for (int64_t k = kb * BLOCK; k < (kb + 1) * BLOCK; ++k)\n        acc +=",
     "for (int64_t k = kb * BLOCK; k < (kb + 1) * BLOCK - 1; ++k)\n        acc +="),
    ("drop_weight_scale", "const float scale = xs[mb * kbn + kb] * ws[nb * kbn + kb];",
     "const float scale = xs[mb * kbn + kb];"),
    ("first_block_scale_only", "const float scale = xs[mb * kbn + kb] * ws[nb * kbn + kb];",
     "const float scale = xs[mb * kbn] * ws[nb * kbn];"),
    ("reversed_kb_scale", "const float scale = xs[mb * kbn + kb] * ws[nb * kbn + kb];",
     "const float scale = xs[mb * kbn + kb] * ws[nb * kbn + (kbn - 1 - kb)];"),
    ("commuted_product_noop", "const float term = (float)p * scale;",
     "const float term = scale * (float)p;"),
    ("drop_bias", "return acc + b;", "return acc;"),
    ("bias_twice", "return acc + b;", "return acc + b + b;"),
    ("rms_divide_k_minus_1", "const double mean = ss / (double)K;",
     "const double mean = ss / (double)(K - 1);"),
    ("rms_drop_eps", "return (float)(1.0 / sqrt(mean + (double)eps));",
     "return (float)(1.0 / sqrt(mean));"),
    ("rms_drop_gamma", "yrow[k] = f32_to_bf16(t * bf16_to_f32(gamma[k]));",
     "yrow[k] = f32_to_bf16(t);"),
    ("rms_gamma_reversed", "yrow[k] = f32_to_bf16(t * bf16_to_f32(gamma[k]));",
     "yrow[k] = f32_to_bf16(t * bf16_to_f32(gamma[K - 1 - k]));"),
    ("bf16_round_half_up", "u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    ("fallback_w_reversed_k", "(double)bf16_to_f32(w[n * K + k]);",
     "(double)bf16_to_f32(w[n * K + (K - 1 - k)]);"),
    ("fallback_drop_bias", "return (float)acc + b;", "return (float)acc;"),
    ("row_floor_on_scale", "const float sc = (absmax > ROW_EPS ? absmax : ROW_EPS) / 127.0f;",
     "const float sc = (absmax / 127.0f > ROW_EPS ? absmax / 127.0f : ROW_EPS);"),
    ("row_floor_1e-3", "#define ROW_EPS 1e-4f", "#define ROW_EPS 1e-3f"),
    ("row_no_abs", "const float a = fabsf(bf16_to_f32(x[r * cols + j]));",
     "const float a = bf16_to_f32(x[r * cols + j]);"),
    ("row_drop_weight_scale", "const float scale = xs[m] * ws[n];",
     "const float scale = xs[m];"),
    ("row_weight_scale_halved_index", "const float scale = xs[m] * ws[n];",
     "const float scale = xs[m] * ws[n / 2];"),
    ("row_sum_in_double", "const float v = (float)(int32_t)acc * scale;",
     "const float v = (float)((double)acc * (double)scale);"),
    ("row_bias_twice", "return v + b;", "return v + b + b;"),
    ("mod_scale_without_one", "const float a = 1.0f + bf16_to_f32(scale[k]);",
     "const float a = bf16_to_f32(scale[k]);"),
    ("mod_shift_subtracted", "yrow[k] = f32_to_bf16(u + bf16_to_f32(shift[k]));",
     "yrow[k] = f32_to_bf16(u - bf16_to_f32(shift[k]));"),
    ("mod_scale_shift_swapped", "gamma, scale + b * K, shift + b * K, r,",
     "gamma, shift + b * K, scale + b * K, r,"),
    ("mod_sample_index_modulo", "const int64_t b = m / T;\n        const float r = row_rstd(",
     "const int64_t b = m % (M / T);\n        const float r = row_rstd("),
    ("mod_drop_gamma", "n = n * bf16_to_f32(gamma[k]);", "n = n * 1.0f;"),
    ("mod_shift_rounded_in", "const float u = n * a;",
     "const float u = bf16_to_f32(f32_to_bf16(n * a));"),
    ("gated_drop_gate", "const float gv = bf16_to_f32(gate[b * N + ns[t]]) * v[t];",
     "const float gv = v[t];"),
    ("gated_gate_transposed", "const float gv = bf16_to_f32(gate[b * N + ns[t]]) * v[t];",
     "const float gv = bf16_to_f32(gate[ns[t] * (M / T) + b]) * v[t];"),
    ("gated_sample_index_modulo", "const int64_t b = ms[t] / T;",
     "const int64_t b = ms[t] % (M / T);"),
    ("gated_v_rounded_first", "const float gv = bf16_to_f32(gate[b * N + ns[t]]) * v[t];",
     "const float gv = bf16_to_f32(gate[b * N + ns[t]]) * bf16_to_f32(f32_to_bf16(v[t]));"),
]
# commuted_product_noop rewrites without changing the arithmetic (FP32 multiplication
# commutes): it checks that the harness does not report every rewrite as caught.
NOOP = {"commuted_product_noop"}


def _build_mutant(tmp_path, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor not unique: {old!r}"
    src = tmp_path / "oracle.c"
    src.write_text(text.replace(old, new))
    so = str(tmp_path / "libmutant.so")
    import subprocess
    subprocess.run(["gcc", *oracle.CFLAGS, str(src), "-o", so, "-lm"], check=True)
    return oracle.Oracle(oracle.load(so))


@pytest.mark.parametrize("mid,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, mid, old, new):
    o = _build_mutant(tmp_path, old, new)
    failed = []
    for p in pins.ALL_PINS:
        try:
            p(o)
        except AssertionError:
            failed.append(p.__name__)
    if mid in NOOP:
        assert not failed, f"a rewrite with unchanged arithmetic failed pins {failed}"
    else:
        assert failed, f"mutant {mid} passed every pin"
