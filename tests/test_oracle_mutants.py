"""Plant plausible mistakes in copies of the oracle's C source (on the CPU)
and check that the pins catch every one.  This is what makes the pins
trustworthy: a dropped term, a wrong sign, a wrong constant, a swapped index
or a wrong rounding mode anywhere in the oracle fails at least one of them."""
import os
import tempfile

import pytest

import oracle
import oracle_pins

# (name, text to replace, replacement, which occurrence (0-based))
MUTANTS = [
    ("fwht_f64_sign", "v[k + h] = a - b;", "v[k + h] = b - a;", 0),
    ("fwht_f32_sign", "v[k + h] = a - b;", "v[k + h] = b - a;", 1),
    ("fwht_f32_drop_term", "v[k] = a + b;", "v[k] = a;", 1),
    ("fwht_f32_index", "float b = v[k + h];", "float b = v[k + h - (h > 1)];", 0),
    ("fwht_stage_skipped", "for (int h = 1; h < D; h <<= 1)", "for (int h = 2; h < D; h <<= 1)", 1),
    ("lambda_divides", "* lam[i];   /* one rounding  */", "/ lam[i];   /* one rounding  */", 0),
    ("lambda_dropped", "* lam[i];   /* one rounding  */", ";   /* one rounding  */", 0),
    ("sign_dropped", "y[i] = (s[i] < 0) ? -t : t;", "y[i] = t;", 0),
    ("norm_const", "(float)(1.0 / sqrt((double)D))", "(float)(1.0 / (double)D)", 0),
    ("normalise_skipped", "for (int i = 0; i < D; ++i) y[i] = y[i] * c;", "(void)c;", 0),
    ("scale_div8", "kvqo_f32_to_f16(a / 7.0f);", "kvqo_f32_to_f16(a / 8.0f);", 0),
    ("absmax_min", "if (m > a) a = m;", "if (m < a) a = m;", 0),
    ("no_saturation", "if (sb == 0x7C00u) sb = 0x7BFFu;            /* saturate to 65504 */", "", 0),
    ("round_half_away", "rintf(yg[i] * r)", "roundf(yg[i] * r)", 0),
    ("truncate", "rintf(yg[i] * r)", "truncf(yg[i] * r)", 0),
    ("clamp_low_7", "if (t < -8.0f) t = -8.0f;", "if (t < -7.0f) t = -7.0f;", 0),
    ("nibble_order", "packed[b] = (uint8_t)(lo | (hi << 4));", "packed[b] = (uint8_t)(hi | (lo << 4));", 0),
    ("unpack_no_sign_ext", "codes[2 * b] = (int8_t)(lo >= 8 ? lo - 16 : lo);", "codes[2 * b] = (int8_t)lo;", 0),
    ("deq_scale_index", "kvqo_f16_to_f32(scales[i / G]);", "kvqo_f16_to_f32(scales[0]);", 0),
    ("deq_no_norm", "float z = w[i] * c;", "float z = w[i];", 0),
    ("deq_no_sign", "float zs = (s[i] < 0) ? -z : z;                         /* exact */", "float zs = z;", 0),
    ("deq_lambda_mult", "float il = 1.0f / lam[i];", "float il = lam[i];", 0),
    ("unrotate_f64_lambda", "(double)s[i] / lam[i];", "(double)s[i] * lam[i];", 0),
    ("f16_round_trunc", "_Float16 h = (_Float16)f;", "_Float16 h = (_Float16)(f - f * 0x1p-12f);", 0),
    ("ex_int8_qmax", "float qmax = (bits == 4) ? 7.0f : 127.0f;", "float qmax = (bits == 4) ? 7.0f : 126.0f;", 0),
    ("ex_int8_clamp", "float qmin = (bits == 4) ? -8.0f : -128.0f;", "float qmin = (bits == 4) ? -8.0f : -8.0f;", 0),
    ("ex_after_lambda_dropped", "f[i] = lambda_after ? lr[i] * norm_of(i, D, srft)", "f[i] = lambda_after ? norm_of(i, D, srft)", 0),
    ("ex_variant_sign_dropped", "v[i] = (s[i] < 0) ? -t : t;                    /* exact  */", "v[i] = t;", 0),
    ("ex_table_index", "return lam + ((r / lambda_rows) % n_lambda) * (int64_t)D;", "return lam + (r % n_lambda) * (int64_t)D;", 0),
    ("ex_int8_store", "for (int i = 0; i < D; ++i) cr[i] = (uint8_t)q[i];", "for (int i = 0; i < D; ++i) cr[i] = (uint8_t)(q[i] & 0x7F);", 0),
    ("ex_deq_lambda_mult", "f[i] = lambda_after ? norm_of(i, D, srft) / lr[i]", "f[i] = lambda_after ? norm_of(i, D, srft) * lr[i]", 0),
    ("ex_deq_sign_dropped", "float z = (s[i] < 0) ? -w[i] : w[i];                   /* exact */", "float z = w[i];", 0),
    ("ex_deq_before_lambda_mult", "w[i] = lambda_after ? z : z * (1.0f / lr[i]);", "w[i] = lambda_after ? z : z * lr[i];", 0),
    ("ex_deq_int8_unsigned", "for (int i = 0; i < D; ++i) q[i] = (int8_t)cr[i];", "for (int i = 0; i < D; ++i) q[i] = (int8_t)(cr[i] & 0x7F);", 0),
    ("srft_twiddle_sign", "*wi = -sn + 0.0f;", "*wi = sn + 0.0f;", 0),
    # the table before exact roots: cos / sin of 2 pi k / M straight in double
    ("twiddle_unreduced", "    *wr = cr + 0.0f;                            /* -0 -> +0 */\n    *wi = -sn + 0.0f;",
     "    (void)cr; (void)sn;\n    *wr = (float)cos(6.28318530717958647692 * (double)j / (double)M);\n"
     "    *wi = (float)(-sin(6.28318530717958647692 * (double)j / (double)M));", 0),
    ("twiddle_quadrant", "case 1: cr = -s; sn = c; break;", "case 1: cr = s; sn = c; break;", 0),
    ("twiddle_complement", "if (comp) { float t = c; c = s; s = t; }", "(void)comp;", 0),
    ("twiddle_signed_zero", "    *wr = cr + 0.0f;                            /* -0 -> +0 */", "    *wr = cr;", 0),
    ("cmul_trivial_i_sign", "*pr = (wi > 0.0f) ? -di : di;", "*pr = (wi > 0.0f) ? di : -di;", 0),
    ("cmul_fused_sign", "*pr = fmaf(dr, wr, -b);", "*pr = fmaf(dr, wr, b);", 0),
    ("cmul_fused_operand", "*pi_ = fmaf(di, wr, c);", "*pi_ = fmaf(di, wi, c);", 0),
    ("srft_no_sqrt2", "(float)(1.0 / sqrt(2.0 * (double)D))", "(float)(1.0 / sqrt((double)D))", 0),
    ("srft_stage_stride", "kvqo_twiddle(s * p * t, N, &wr, &wi);               /* omega_n^(p t) */",
     "kvqo_twiddle(p * t, N, &wr, &wi);", 0),
    ("srft_butterfly_sign", "br = br + tr;", "br = br - tr;", 0),
    ("radix3_twiddle", "kvqo_twiddle((N / r) * j * t, N, &wr, &wi);     /* omega_r^(j t) */",
     "kvqo_twiddle((N / r) * j, N, &wr, &wi);", 0),
    ("dit_stage_conj", "cmul(yr[q + s * (r * p + t)], yi[q + s * (r * p + t)], wr, -wi, &cr[t], &ci[t]);",
     "cmul(yr[q + s * (r * p + t)], yi[q + s * (r * p + t)], wr, wi, &cr[t], &ci[t]);", 0),
    ("dit_radix_conj", "cmul(cr[t], ci[t], wr, -wi, &tr, &ti);", "cmul(cr[t], ci[t], wr, wi, &tr, &ti);", 0),
    ("srft_odd_part_sign", "float Or = Di, Oi = -Dr;", "float Or = Di, Oi = Dr;", 0),
    ("srft_nyquist_slot", "y[1] = (zr[0] - zi[0]) * f[1];", "y[1] = (zr[0] + zi[0]) * f[1];", 0),
    ("isrft_no_conj", "cmul(Dr, Di, wr, -wi, &Tr, &Ti);                 /* conj(omega_D^k) */",
     "cmul(Dr, Di, wr, wi, &Tr, &Ti);", 0),
    ("isrft_pairing", "zr[k] = Er - Ti;                                  /* E + i T */", "zr[k] = Er + Ti;", 0),
    ("isrft_dc", "zi[0] = u0 - un;", "zi[0] = u0 + un;", 0),
    ("srft_pair_conj", "x[3] = -Wi;", "x[3] = Wi;", 0),
    ("srft_pair_sub", "float Wr = Er - Tr, Wi = Ei - Ti;", "float Wr = Er + Tr, Wi = Ei - Ti;", 0),
    ("isrft_pair_conj", "zi[N - k] = -Wi;", "zi[N - k] = Wi;", 0),
    ("isrft_pair_sign", "float Wr = Er + Ti, Wi = Ei - Tr;             /* E - i T */",
     "float Wr = Er - Ti, Wi = Ei - Tr;", 0),
    ("attn_gqa_index", "int kv = h / R;", "int kv = h % Hkv;", 0),
    ("attn_no_max_shift", "double p = exp(z[t] - m);", "double p = exp(z[t]);", 0),
    ("attn_len_ignored", "for (int t = 0; t < len; ++t) {\n                double p", "for (int t = 0; t < T; ++t) {\n                double p", 0),
    ("attn_scale_unused", "z[t] = sm_scale * dot;", "z[t] = dot;", 0),
    ("attn_v_uses_k_lambda", "D, G, flags, row);\n                for (int i = 0; i < D; ++i) o[i] += p * row[i];",
     "D, G, flags, row);\n                (void)lv; for (int i = 0; i < D; ++i) o[i] += p * row[i] * lv[i] / lk[i];", 0),
    ("attn_not_normalised", "for (int i = 0; i < D; ++i) o[i] /= l;", "(void)l;", 0),
    ("attn_scale_index", "(double)kvqo_f16_to_f32(scales[i / G]);", "(double)kvqo_f16_to_f32(scales[0]);", 0),
    ("attn_fmt_after_divides_late", "    if (flags & 1)\n        for (int i = 0; i < D; ++i) y[i] /= lam[i];",
     "    if (flags & 1)\n        for (int i = 0; i < D; ++i) y[i] *= 1.0;", 0),
    ("attn_fmt_srft_as_wht", "    if (flags & 2) {\n        kvqo_isrft_f64(y, D, x);", "    if (0) {\n        kvqo_isrft_f64(y, D, x);", 0),
    ("attn_fmt_sign_dropped", "        x[i] *= (double)s[i];\n        if (!(flags & 1)) x[i] /= lam[i];",
     "        if (!(flags & 1)) x[i] /= lam[i];", 0),
]


def _mutate(src: str, old: str, new: str, occ: int) -> str:
    idx = -1
    for _ in range(occ + 1):
        idx = src.index(old, idx + 1)
    return src[:idx] + new + src[idx + len(old):]


@pytest.fixture(scope="module")
def source():
    with open(oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(source, name, old, new, occ):
    mutated = _mutate(source, old, new, occ)
    assert mutated != source
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "mutant.c")
        lib = os.path.join(td, "libmutant.so")
        with open(src, "w") as f:
            f.write(mutated)
        oracle.build(src, lib)
        o = oracle.Oracle(lib)
        failed = []
        for pin in oracle_pins.ALL_PINS:
            try:
                pin(o)
            except AssertionError:
                failed.append(pin.__name__)
            except (ValueError, FloatingPointError):
                failed.append(pin.__name__)
        assert failed, f"no pin caught mutant {name}"
