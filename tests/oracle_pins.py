"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError on failure.  They
check the oracle against what the pages and the mathematics fix:

* brute force: the transform against the dense Sylvester matrix built two
  independent ways (Kronecker powers and the popcount formula);
* the rotation's orthogonality (norm preservation, exact inverse);
* closed forms: zero rows, an impulse (every code +-7 with the Hadamard sign
  pattern), constant rows, a saturating row;
* the quantiser's error bound |y - q S| <= S/2 and the codes' range;
* library routines: fp16 conversion against numpy's IEEE cast;
* hand-worked examples (tests/golden/worked_examples.json) and the pages'
  printed compression figure (tests/golden/accounting.json);
* the SRFT rotation: numpy's rfft (unitary, packed), orthogonality of its
  dense matrix, the fp32 Stockham path within its bound of the float64
  definition, closed forms, and the codec built on it, at power-of-two and
  mixed-radix (three times a power of two) lengths; its twiddle table against
  the correctly rounded exact roots of unity, computed independently in
  80-digit decimal arithmetic, and against the exact symmetries of the roots;
  its complex FFT against numpy's fft, exactly where only the twiddles 1, -1,
  i, -i occur;
* format variants (lambda after the rotation, int8 codes, lambda tables):
  the float64 definition with the dense matrix, the int8 code invariants, the
  table indexing, the round-trip bound and the impulse closed form;
* decode attention: against torch's scaled_dot_product_attention (float64)
  on caches rebuilt with numpy and scipy's Hadamard matrix, and against the
  closed forms one key (o = V_0), zero scale (o = mean V), a huge scale
  (o = V at the arg-max) and masking (entries past the length are ignored).

``tests/test_oracle.py`` runs every pin on the oracle; ``tests/
test_oracle_mutants.py`` plants plausible mistakes in copies of the oracle's
C source and checks that at least one pin fails for each.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

from kv_cache_quantization_02_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
U32 = 2.0 ** -24          # unit roundoff of fp32


def sylvester_kron(D: int) -> np.ndarray:
    H = np.array([[1.0]])
    while H.shape[0] < D:
        H = np.kron(H, np.array([[1.0, 1.0], [1.0, -1.0]]))
    return H


def sylvester_popcount(D: int) -> np.ndarray:
    i = np.arange(D)[:, None]
    j = np.arange(D)[None, :]
    bits = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(bits % 2 == 0, 1.0, -1.0)


def _rand_params(rng, D):
    lam = rng.uniform(0.5, 2.0, D).astype(np.float32)
    s = np.where(rng.random(D) < 0.5, -1, 1).astype(np.int8)
    return lam, s


def _rows(rng, n, D, outliers=4, gain=20.0):
    x = rng.standard_normal((n, D))
    if outliers:
        x[:, rng.permutation(D)[:outliers]] *= gain
    return x.astype(np.float16)


# --------------------------------------------------------------------------
def pin_f16_conversion(o):
    """fp32 -> fp16 (RNE) and fp16 -> fp32 against numpy's IEEE casts."""
    all_bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = all_bits.view(np.float16).astype(np.float32)
    finite = np.isfinite(ref)
    got = np.array([o.f16_bits_to_f32(int(b)) for b in all_bits[finite]],
                   dtype=np.float32)
    assert np.array_equal(got, ref[finite]), "fp16 -> fp32 differs from numpy"
    # midpoints between neighbouring fp16 values are ties: RNE picks the even one
    pos = ref[finite & (ref >= 0)]
    pos = np.unique(pos)
    mids = ((pos[:-1].astype(np.float64) + pos[1:].astype(np.float64)) / 2)
    mids = mids[np.abs(mids) < 65504].astype(np.float32)
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        mids[::37], -mids[::41], rng.standard_normal(2000).astype(np.float32) * 100,
        np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 1e6, -1e6, 2.0 ** -24,
                  2.0 ** -25, 2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26, 2.0 ** -14,
                  6.1e-5, 1.0 / 7.0], dtype=np.float32)])
    for v in vals:
        with np.errstate(over="ignore"):
            want = int(np.float32(v).astype(np.float16).view(np.uint16))
        got = o.f32_to_f16_bits(float(v))
        assert got == want, f"fp32 {v!r} -> fp16 bits {got:#06x}, numpy {want:#06x}"


def pin_norm_const(o):
    """c is the fp32 value nearest 1/sqrt(D) (exact rational check)."""
    assert o.norm_const(64) == 0.125 and o.norm_const(256) == 0.0625
    assert np.float32(o.norm_const(128)).view(np.uint32) == 0x3DB504F3
    for k in range(1, 13):
        D = 1 << k
        c = Fraction(o.norm_const(D))
        ulp = Fraction(float(np.spacing(np.float32(float(c)))))
        lo, hi = c - ulp / 2, c + ulp / 2
        assert lo * lo * D < 1 < hi * hi * D, f"c for D={D} is not the nearest fp32"


def pin_fwht_dense(o):
    """Unnormalised transform == dense Sylvester matrix (two constructions)."""
    rng = np.random.default_rng(1)
    for k in range(1, 9):
        D = 1 << k
        H = sylvester_kron(D)
        assert np.array_equal(H, sylvester_popcount(D))
        v = rng.standard_normal((3, D))
        for row in v:
            got = o.fwht_f64(row)
            np.testing.assert_allclose(got, H @ row, rtol=0, atol=1e-12 * D)
        iv = rng.integers(-50, 50, size=D).astype(np.float64)
        assert np.array_equal(o.fwht_f64(iv), H @ iv)
        assert np.array_equal(o.fwht_f32(iv.astype(np.float32)),
                              (H @ iv).astype(np.float32))


def pin_rotation_dense(o):
    """rotate_f64 == H diag(s) (lambda . x) / sqrt(D); unrotate is its inverse."""
    rng = np.random.default_rng(2)
    for D in (2, 4, 8, 16, 32, 64, 128, 256):
        H = sylvester_kron(D)
        lam, s = _rand_params(rng, D)
        M = H @ np.diag(s.astype(np.float64)) / math.sqrt(D)
        np.testing.assert_allclose(M.T @ M, np.eye(D), atol=1e-12)
        x = rng.standard_normal(D) * 3
        y = o.rotate_f64(x, lam, s)
        np.testing.assert_allclose(y, M @ (lam.astype(np.float64) * x), atol=1e-12)
        xb = o.unrotate_f64(y, lam, s)
        np.testing.assert_allclose(xb, (M.T @ y) / lam.astype(np.float64), atol=1e-12)
        np.testing.assert_allclose(xb, x, atol=1e-12)


def _fwht_err_bound(x64, lam, D):
    """Forward-error bound of the fp32 path against exact arithmetic: one
    rounding at x*lambda, log2(D) roundings per butterfly path, one at *c,
    and the error of c itself."""
    terms = np.abs(x64 * lam.astype(np.float64))
    l1 = terms.sum(axis=-1, keepdims=True)
    return (math.log2(D) + 3) * U32 * l1 / math.sqrt(D) * 1.01


def pin_rotate_f32(o):
    """fp32 forward rotation within its rounding bound of the f64 definition."""
    rng = np.random.default_rng(3)
    for D in (4, 16, 64, 128, 256):
        lam, s = _rand_params(rng, D)
        x = _rows(rng, 16, D)
        y32 = o.rotate_f32(x, lam, s).astype(np.float64)
        x64 = x.astype(np.float64)
        y64 = np.stack([o.rotate_f64(r, lam, s) for r in x64])
        bound = _fwht_err_bound(x64, lam, D)
        assert np.all(np.abs(y32 - y64) <= bound), f"fp32 rotation off at D={D}"


def pin_norm_preservation(o):
    rng = np.random.default_rng(4)
    for D in (8, 64, 128, 256):
        lam, s = _rand_params(rng, D)
        x = _rows(rng, 8, D)
        x64 = x.astype(np.float64)
        ref = np.linalg.norm(x64 * lam.astype(np.float64), axis=1)
        y64 = np.stack([o.rotate_f64(r, lam, s) for r in x64])
        np.testing.assert_allclose(np.linalg.norm(y64, axis=1), ref, rtol=1e-12)
        y32 = o.rotate_f32(x, lam, s).astype(np.float64)
        np.testing.assert_allclose(np.linalg.norm(y32, axis=1), ref, rtol=1e-6)


def pin_roundtrip_unquantized(o):
    """rotate -> inverse recovers x (f64: to 1e-5 absolute and far below;
    fp32: to 1e-5 of the row's largest magnitude)."""
    rng = np.random.default_rng(5)
    for D in (16, 64, 128, 256):
        lam, s = _rand_params(rng, D)
        x = _rows(rng, 8, D)
        x64 = x.astype(np.float64)
        back = np.stack([o.unrotate_f64(o.rotate_f64(r, lam, s), lam, s) for r in x64])
        assert np.max(np.abs(back - x64)) <= 1e-5
        np.testing.assert_allclose(back, x64, atol=1e-12 * np.abs(x64).max())
        b32 = o.unrotate_f32(o.rotate_f32(x, lam, s), lam, s).astype(np.float64)
        scale = np.abs(x64).max(axis=1, keepdims=True)
        assert np.all(np.abs(b32 - x64) <= 1e-5 * scale)


def _scales_f32(scales):
    return np.asarray(scales).astype(np.float32)


def pin_code_invariants(o):
    """Codes lie in [-8, 7]; every group with a normal scale has max|q| = 7;
    the scale is the fp16 rounding of max|y|/7."""
    rng = np.random.default_rng(6)
    cases = []
    for D, G in ((64, 16), (64, 64), (128, 32), (128, 16), (256, 32), (256, 64), (256, 256)):
        lam, s = _rand_params(rng, D)
        cases.append((_rows(rng, 24, D), lam, s, G))
    w = workloads.WORKLOADS["qwen2.5-1.5b"]
    lam, s = workloads.params(w.D, w.seed)
    cases.append((workloads.host_rows(w, 64), lam, s, 32))
    for x, lam, s, G in cases:
        D = x.shape[1]
        q, S = o.quantize_codes(x, lam, s, G)
        assert q.min() >= -8 and q.max() <= 7
        Sf = _scales_f32(S)
        y = o.rotate_f32(x, lam, s)
        a = np.abs(y).reshape(len(x), D // G, G).max(axis=2)
        want = (a / np.float32(7.0)).astype(np.float32).astype(np.float16).astype(np.float32)
        assert np.array_equal(Sf, want), "scale is not fp16(max|y|/7)"
        qm = np.abs(q.astype(np.int32)).reshape(len(x), D // G, G).max(axis=2)
        normal = Sf >= 2.0 ** -14
        assert np.all(qm[normal] == 7), "a group with a normal scale lacks |q| = 7"
        assert not np.any(q.reshape(len(x), D // G, G)[normal] == -8)


def pin_error_bound(o):
    """|y_i - q_i S_j| <= S_j / 2 for every element of a normal-scale group,
    and the reconstruction error obeys the same bound after the inverse:
    ||lambda.(x - x_hat)||_2 <= sqrt(sum_j G S_j^2) / 2 (+ fp32 slack)."""
    rng = np.random.default_rng(8)
    for D, G in ((64, 32), (128, 32), (128, 16), (256, 64)):
        lam, s = _rand_params(rng, D)
        x = _rows(rng, 32, D)
        q, S = o.quantize_codes(x, lam, s, G)
        Sf = _scales_f32(S).astype(np.float64)
        y = o.rotate_f32(x, lam, s).astype(np.float64)
        Se = np.repeat(Sf, G, axis=1)
        err = np.abs(y - q * Se)
        ok = Se >= 2.0 ** -14
        assert np.all(err[ok] <= Se[ok] / 2 * (1 + 1e-6)), "quantiser error above S/2"
        xh = o.dequantize_f32(q, S, lam, s, G).astype(np.float64)
        lhs = np.linalg.norm(lam.astype(np.float64) * (x.astype(np.float64) - xh), axis=1)
        rhs = 0.5 * np.sqrt(G * (Sf ** 2).sum(axis=1))
        slack = (math.log2(D) + 4) * U32 * np.abs(y).sum(axis=1) * 2
        assert np.all(lhs <= rhs + slack), "round trip exceeds the quantiser bound"


def pin_dequant_vs_f64(o):
    """fp32 inverse path within rounding of the f64 inverse rotation of q*S,
    and the fp16 output is the RNE cast of the fp32 output."""
    rng = np.random.default_rng(9)
    for D, G in ((16, 16), (64, 16), (128, 32), (256, 64)):
        lam, s = _rand_params(rng, D)
        q = rng.integers(-8, 8, size=(12, D)).astype(np.int8)
        S = (rng.uniform(0.01, 3.0, size=(12, D // G))).astype(np.float16)
        got = o.dequantize_f32(q, S, lam, s, G).astype(np.float64)
        u = q * np.repeat(S.astype(np.float64), G, axis=1)
        ref = np.stack([o.unrotate_f64(r, lam, s) for r in u])
        bound = (math.log2(D) + 4) * U32 * np.abs(u).sum(axis=1, keepdims=True) \
            / math.sqrt(D) / lam.astype(np.float64).min() * 1.01
        assert np.all(np.abs(got - ref) <= bound), f"inverse path off at D={D}"
        # and against the dense matrix directly
        H = sylvester_kron(D)
        dense = (u @ H.T) / math.sqrt(D) * s.astype(np.float64) / lam.astype(np.float64)
        assert np.all(np.abs(got - dense) <= bound)
        packed = o.pack(q)
        out16 = o.dequantize(packed, S, lam, s, G)
        assert np.array_equal(out16.view(np.uint16),
                              got.astype(np.float32).astype(np.float16).view(np.uint16))


def pin_special_cases(o):
    rng = np.random.default_rng(10)
    for D, G in ((64, 16), (128, 32), (256, 64)):
        lam, s = _rand_params(rng, D)
        # zero rows
        z = np.zeros((2, D), dtype=np.float16)
        q, S = o.quantize_codes(z, lam, s, G)
        assert not q.any() and not S.astype(np.float32).any()
        assert not o.dequantize(o.pack(q), S, lam, s, G).astype(np.float32).any()
        # impulse alpha e_k with lambda = 1: |y_i| = |alpha|/sqrt(D) for all i,
        # every code +-7 with sign = sign(alpha) s_k H[k, i]
        ones = np.ones(D, dtype=np.float32)
        H = sylvester_popcount(D)
        for k, alpha in ((0, 3.0), (D // 3, -1.5), (D - 1, 250.0)):
            x = np.zeros((1, D), dtype=np.float16)
            x[0, k] = alpha
            q, S = o.quantize_codes(x, ones, s, G)
            want = (7 * np.sign(alpha) * s[k] * H[k]).astype(np.int8)
            assert np.array_equal(q[0], want), "impulse codes wrong"
            y = np.float32(alpha) * np.float32(o.norm_const(D))
            sw = (np.abs(y) / np.float32(7)).astype(np.float16)
            assert np.all(S[0] == sw)
        # constant row, lambda = 1, signs = +1: all energy in coefficient 0
        pos = np.ones(D, dtype=np.int8)
        x = np.full((1, D), 0.75, dtype=np.float16)
        q, S = o.quantize_codes(x, ones, pos, G)
        assert q[0, 0] == 7 and not q[0, 1:].any()
        assert np.all(S[0, 1:].astype(np.float32) == 0) and S[0, 0] > 0
        out = o.dequantize(o.pack(q), S, ones, pos, G).astype(np.float32)
        assert np.all(out == out[0, 0]) and abs(out[0, 0] - 0.75) < 0.75 / 7
    # saturating scale: D=256 rows of 65504 with lambda = 2
    D, G = 256, 64
    x = np.full((1, D), 65504.0, dtype=np.float16)
    q, S = o.quantize_codes(x, np.full(D, 2.0, np.float32), np.ones(D, np.int8), G)
    assert S.view(np.uint16)[0, 0] == 0x7BFF and q[0, 0] == 7


def pin_worked_examples(o):
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        ex = json.load(f)
    for e in ex["examples"]:
        x = np.array([e["x"]], dtype=np.float16)
        assert np.array_equal(x.astype(np.float64)[0], np.array(e["x"])), "fixture x not fp16"
        lam = np.array(e["lambda"], dtype=np.float32)
        s = np.array(e["signs"], dtype=np.int8)
        G = e["G"]
        y = o.rotate_f32(x, lam, s)
        assert np.array_equal(y[0].astype(np.float64), np.array(e["y"])), e["name"]
        q, S = o.quantize_codes(x, lam, s, G)
        assert q[0].tolist() == e["codes"], e["name"]
        assert S.view(np.uint16)[0].tolist() == e["scale_bits"], e["name"]
        packed, S2 = o.quantize(x, lam, s, G)
        assert packed[0].tolist() == e["packed"], e["name"]
        out = o.dequantize(packed, S2, lam, s, G)
        assert out[0].astype(np.float64).tolist() == e["dequant"], e["name"]


def pin_divform_near_ties(o):
    """Multiplying by 1/S and dividing by S pick different codes only within
    a few ulp of a rounding tie, and then differ by one."""
    rng = np.random.default_rng(11)
    D, G = 128, 32
    lam, s = _rand_params(rng, D)
    x = _rows(rng, 512, D)
    q, S = o.quantize_codes(x, lam, s, G)
    qd = o.quantize_codes_divform(x, lam, s, G)
    diff = q != qd
    if diff.any():
        assert np.abs(q.astype(int) - qd.astype(int)).max() == 1
        y = o.rotate_f32(x, lam, s).astype(np.float64)
        t = y / np.repeat(S.astype(np.float64), G, axis=1)
        frac = np.abs(np.abs(t - np.floor(t)) - 0.5)
        assert np.all(frac[diff] < 1e-5)
    assert diff.mean() <= 1e-3


def pin_pack_layout(o):
    """Low nibble = even element, two's complement; pack/unpack are inverse."""
    assert o.pack(np.array([1, 2], dtype=np.int8)).tolist() == [0x21]
    assert o.pack(np.array([-1, -8], dtype=np.int8)).tolist() == [0x8F]
    assert o.pack(np.array([7, -7], dtype=np.int8)).tolist() == [0x97]
    allc = np.array([(a, b) for a in range(-8, 8) for b in range(-8, 8)],
                    dtype=np.int8).reshape(-1)
    assert np.array_equal(o.unpack(o.pack(allc)), allc)


def pin_accounting(o):
    """Storage per vector and the pages' printed compression ratio."""
    with open(os.path.join(GOLDEN, "accounting.json")) as f:
        acc = json.load(f)
    G = acc["compression_upper_group"]
    ratio = 16.0 / (4.0 + 16.0 / G)
    assert round(ratio, 2) == acc["compression_upper_printed"]
    assert 16.0 / (4.0 + 16.0 / acc["group_size_in_methodology"]) >= acc["compression_lower_printed"]
    rng = np.random.default_rng(12)
    for D, G in ((64, 16), (128, 32), (256, 64)):
        lam, s = _rand_params(rng, D)
        packed, S = o.quantize(_rows(rng, 3, D), lam, s, G)
        fp16_bytes = 2 * D
        stored = packed.shape[1] + 2 * S.shape[1]
        assert stored == D // 2 + 2 * D // G
        assert abs(fp16_bytes / stored - 16.0 / (4.0 + 16.0 / G)) < 1e-12


# ---- format variants: lambda after the rotation, int8 codes, lambda tables ----

def _y_def(x, lam, s, lambda_after):
    """The rotation's definition in float64 with the dense Sylvester matrix."""
    D = x.shape[1]
    H = sylvester_kron(D)
    x64 = x.astype(np.float64)
    l64 = lam.astype(np.float64)
    s64 = s.astype(np.float64)
    if lambda_after:
        return l64 * ((x64 * s64) @ H.T) / math.sqrt(D)
    return ((x64 * l64 * s64) @ H.T) / math.sqrt(D)


def _codes_ex(o, codes, bits, D):
    if bits == 4:
        return o.unpack(codes).astype(np.int64)
    return codes.view(np.int8).astype(np.int64)


def pin_ex_matches_base(o):
    """bits 4, lambda before, one table: the variant path is the base codec."""
    rng = np.random.default_rng(31)
    for D, G in ((16, 16), (128, 32), (256, 64)):
        lam, s = _rand_params(rng, D)
        x = _rows(rng, 9, D)
        p1, s1 = o.quantize(x, lam, s, G)
        p2, s2 = o.quantize_ex(x, lam, s, G)
        assert np.array_equal(p1, p2) and np.array_equal(s1.view(np.uint16), s2.view(np.uint16))
        assert np.array_equal(o.dequantize(p1, s1, lam, s, G).view(np.uint16),
                              o.dequantize_ex(p2, s2, lam, s, G).view(np.uint16))


def pin_ex_definition(o):
    """Scales and codes against the float64 definition of each order: S within
    one fp16 ulp of fp16(max|y|/qmax) and every code within rounding of y/S."""
    rng = np.random.default_rng(32)
    for D, G in ((16, 16), (64, 32), (128, 32)):
        for bits in (4, 8):
            for after in (False, True):
                lam, s = _rand_params(rng, D)
                x = _rows(rng, 16, D)
                codes, S = o.quantize_ex(x, lam, s, G, bits=bits, lambda_after=after)
                y = _y_def(x, lam, s, after)
                qmax = 7.0 if bits == 4 else 127.0
                a = np.abs(y).reshape(16, D // G, G).max(axis=2)
                Sf = S.astype(np.float64)
                ref = (a / qmax).astype(np.float16).astype(np.float64)
                ulp = np.spacing(ref.astype(np.float16)).astype(np.float64)
                assert np.all(np.abs(Sf - ref) <= ulp), f"scale off bits={bits} after={after}"
                q = _codes_ex(o, codes, bits, D)
                t = y / np.repeat(Sf, G, axis=1)
                lo = -8 if bits == 4 else -128
                assert np.all(np.abs(q - np.clip(t, lo, qmax)) <= 0.5 + 1e-3), \
                    f"codes off bits={bits} after={after}"


def pin_ex_int8_codes(o):
    """8-bit codes lie in [-128, 127], every normal-scale group reaches 127,
    and |y - q S| <= S / 2 (no clamping inside the range)."""
    rng = np.random.default_rng(33)
    D, G = 128, 32
    for after in (False, True):
        lam, s = _rand_params(rng, D)
        x = _rows(rng, 32, D)
        codes, S = o.quantize_ex(x, lam, s, G, bits=8, lambda_after=after)
        q = _codes_ex(o, codes, 8, D).reshape(32, D // G, G)
        Sf = S.astype(np.float64)
        assert q.min() >= -128 and q.max() <= 127
        normal = Sf >= 2.0 ** -14
        assert np.all(np.abs(q).max(axis=2)[normal] == 127)
        y = _y_def(x, lam, s, after).reshape(32, D // G, G)
        err = np.abs(y - q * Sf[..., None])
        assert np.all(err <= Sf[..., None] * (0.5 + 1e-4) + 1e-6)


def pin_ex_tables(o):
    """Row r uses table (r // lambda_rows) % n_lambda."""
    rng = np.random.default_rng(34)
    D, G = 64, 16
    tables = rng.uniform(0.5, 2.0, (3, D)).astype(np.float32)
    s = np.where(rng.random(D) < 0.5, -1, 1).astype(np.int8)
    x = _rows(rng, 11, D)
    for bits in (4, 8):
        for after in (False, True):
            codes, S = o.quantize_ex(x, tables, s, G, bits=bits, lambda_after=after, lambda_rows=2)
            back = o.dequantize_ex(codes, S, tables, s, G, bits=bits, lambda_after=after, lambda_rows=2)
            for r in range(11):
                t = tables[(r // 2) % 3]
                c1, s1 = o.quantize_ex(x[r:r + 1], t, s, G, bits=bits, lambda_after=after)
                assert np.array_equal(codes[r:r + 1], c1)
                assert np.array_equal(S[r:r + 1].view(np.uint16), s1.view(np.uint16))
                b1 = o.dequantize_ex(c1, s1, t, s, G, bits=bits, lambda_after=after)
                assert np.array_equal(back[r:r + 1].view(np.uint16), b1.view(np.uint16))


def pin_ex_roundtrip_bound(o):
    """dequantize(quantize(x)) obeys the quantiser's closed-form bound in the
    space where the scales act: |lambda (x - x^)| (before) or |(x - x^) /
    lambda-weighted| (after) <= 1/2 sqrt(sum S^2), plus output rounding."""
    rng = np.random.default_rng(35)
    for D, G in ((64, 16), (128, 32)):
        for bits in (4, 8):
            for after in (False, True):
                lam, s = _rand_params(rng, D)
                x = _rows(rng, 12, D, outliers=0)
                codes, S = o.quantize_ex(x, lam, s, G, bits=bits, lambda_after=after)
                xh = o.dequantize_ex(codes, S, lam, s, G, bits=bits, lambda_after=after)
                d = x.astype(np.float64) - xh.astype(np.float64)
                Sg = np.repeat(S.astype(np.float64), G, axis=1)
                l64 = lam.astype(np.float64)
                if after:
                    # x - x^ = s H (lambda^-1 (y - y^)) / sqrt(D): an isometry of lambda^-1 (y - y^)
                    bound = 0.5 * np.sqrt((Sg ** 2 / l64 ** 2).sum(axis=1))
                    lhs = np.sqrt((d ** 2).sum(axis=1))
                else:
                    bound = 0.5 * np.sqrt((Sg ** 2).sum(axis=1))
                    lhs = np.sqrt(((d * l64) ** 2).sum(axis=1))
                slack = 2.0 ** -10 * np.sqrt((x.astype(np.float64) ** 2).sum(axis=1)) * (l64.max() if not after else 1.0)
                assert np.all(lhs <= bound * 1.001 + slack), f"bits={bits} after={after}"


def pin_ex_impulse(o):
    """x = alpha e_k, lambda = 1: every code is +-qmax with the Hadamard sign
    pattern of row k, in both orders and both widths."""
    D, G = 32, 8
    s = np.where(np.arange(D) % 3 == 0, -1, 1).astype(np.int8)
    H = sylvester_kron(D)
    for k in (0, 5, 31):
        x = np.zeros((1, D), dtype=np.float16)
        x[0, k] = 3.0
        for bits, qmax in ((4, 7), (8, 127)):
            for after in (False, True):
                codes, S = o.quantize_ex(x, np.ones(D, np.float32), s, G, bits=bits, lambda_after=after)
                q = _codes_ex(o, codes, bits, D)[0]
                assert np.array_equal(q, (qmax * s[k] * H[k]).astype(np.int64))


# ---- the SRFT rotation ---------------------------------------------------

def _rfft_packed(v):
    """numpy's rfft, unitary-scaled and packed (y0 = X_0, y1 = X_N, then
    sqrt(2) (Re, Im) X_k): the pages' pack(F v) read as an orthonormal map."""
    D = v.shape[-1]
    N = D // 2
    X = np.fft.rfft(v, axis=-1) / math.sqrt(D)
    y = np.empty(v.shape, dtype=np.float64)
    y[..., 0] = X[..., 0].real
    y[..., 1] = X[..., N].real
    y[..., 2::2] = 0.0
    for k in range(1, N):
        y[..., 2 * k] = math.sqrt(2.0) * X[..., k].real
        y[..., 2 * k + 1] = math.sqrt(2.0) * X[..., k].imag
    return y


def pin_srft_definition(o):
    """The f64 SRFT equals numpy's rfft packed and scaled; it is orthogonal
    (its dense matrix P has P^T P = I) and the f64 inverse is P^T."""
    rng = np.random.default_rng(41)
    for D in (4, 8, 12, 24, 32, 96, 128, 192, 256):
        v = rng.standard_normal((5, D))
        assert np.abs(o.srft_f64(v) - _rfft_packed(v)).max() < 1e-12 * math.sqrt(D)
        P = o.srft_f64(np.eye(D)).T                    # column j = P e_j
        assert np.abs(P.T @ P - np.eye(D)).max() < 1e-12
        y = rng.standard_normal((5, D))
        assert np.abs(o.isrft_f64(y) - y @ P).max() < 1e-12 * math.sqrt(D)


def pin_srft_f32(o):
    """The fp32 Stockham path lies within its error bound of the f64
    definition, preserves the norm, and its inverse undoes it."""
    rng = np.random.default_rng(42)
    U = 2.0 ** -24
    for D in (8, 12, 48, 64, 96, 128, 256):
        v = rng.standard_normal((16, D)).astype(np.float32)
        v[:, 3] *= 30.0
        y32 = o.srft_f32(v).astype(np.float64)
        y64 = o.srft_f64(v.astype(np.float64))
        bound = 6.0 * math.log2(D) * U * np.abs(v.astype(np.float64)).sum(axis=1, keepdims=True) / math.sqrt(D) * 2
        assert np.all(np.abs(y32 - y64) <= bound)
        nv = np.linalg.norm(v.astype(np.float64), axis=1)
        assert np.all(np.abs(np.linalg.norm(y32, axis=1) - nv) <= 1e-6 * nv)
        b32 = o.isrft_f32(y64.astype(np.float32)).astype(np.float64)
        b64 = o.isrft_f64(y64)
        assert np.all(np.abs(b32 - b64) <= bound * 2)
        assert np.abs(b64 - v).max() <= 1e-12 * np.abs(v).max()


def pin_srft_closed_forms(o):
    """signs +1, lambda 1: a constant row puts everything in y0 (code 7 there,
    0 elsewhere); an impulse at channel 0 gives y = (1, 1, sqrt2, 0, sqrt2, 0,
    ...) / sqrt(D): codes (5, 5, 7, 0, 7, 0, ...) at int4, (90, 90, 127, 0,
    ...) at int8."""
    for D, G in ((32, 8), (96, 32)):
        one = np.ones(D, np.float32)
        s = np.ones(D, np.int8)
        x = np.full((1, D), 0.5, dtype=np.float16)
        codes, S = o.quantize_ex(x, one, s, G, srft=True)
        q = o.unpack(codes)[0]
        assert q[0] == 7 and np.all(q[1:] == 0)
        x = np.zeros((1, D), dtype=np.float16)
        x[0, 0] = 1.0
        for bits, top, edge in ((4, 7, 5), (8, 127, 90)):
            for after in (False, True):
                codes, S = o.quantize_ex(x, one, s, G, bits=bits, lambda_after=after, srft=True)
                q = _codes_ex(o, codes, bits, D)[0]
                want = np.zeros(D, np.int64)
                want[0::2] = top
                want[0] = want[1] = edge
                assert np.array_equal(q, want), (D, bits, after, q)


def pin_srft_codec(o):
    """The codec with the SRFT: scales and codes against the float64 definition
    y = R(lambda . x) or lambda . R(x) with R = P diag(s), and the round trip
    obeys the quantiser bound."""
    rng = np.random.default_rng(43)
    for D, G in ((16, 16), (96, 32), (128, 32), (256, 64)):
        for bits in (4, 8):
            for after in (False, True):
                lam, s = _rand_params(rng, D)
                x = _rows(rng, 12, D, outliers=0)
                codes, S = o.quantize_ex(x, lam, s, G, bits=bits, lambda_after=after, srft=True)
                x64 = x.astype(np.float64)
                l64 = lam.astype(np.float64)
                v = x64 * s.astype(np.float64) * (1.0 if after else l64)
                y = o.srft_f64(v) * (l64 if after else 1.0)
                qmax = 7.0 if bits == 4 else 127.0
                a = np.abs(y).reshape(12, D // G, G).max(axis=2)
                Sf = S.astype(np.float64)
                ref = (a / qmax).astype(np.float16).astype(np.float64)
                ulp = np.spacing(ref.astype(np.float16)).astype(np.float64)
                assert np.all(np.abs(Sf - ref) <= ulp)
                q = _codes_ex(o, codes, bits, D)
                t = y / np.repeat(Sf, G, axis=1)
                assert np.all(np.abs(q - np.clip(t, -qmax - 1, qmax)) <= 0.5 + 1e-3)
                xh = o.dequantize_ex(codes, S, lam, s, G, bits=bits, lambda_after=after, srft=True)
                d = x64 - xh.astype(np.float64)
                Sg = np.repeat(Sf, G, axis=1)
                if after:
                    bound = 0.5 * np.sqrt((Sg ** 2 / l64 ** 2).sum(axis=1))
                    lhs = np.linalg.norm(d, axis=1)
                else:
                    bound = 0.5 * np.sqrt((Sg ** 2).sum(axis=1))
                    lhs = np.linalg.norm(d * l64, axis=1)
                slack = 2.0 ** -10 * np.linalg.norm(x64, axis=1) * (1.0 if after else l64.max())
                assert np.all(lhs <= bound * 1.001 + slack)


# ---- the SRFT's twiddles and complex FFT ----------------------------------

_PI80 = ("3.14159265358979323846264338327950288419716939937510"
         "58209749445923078164062862089986280348253421170679")


def _cos_sin_exact(k: int, M: int):
    """cos and sin of 2 pi k / M to ~75 digits, by Taylor series in decimal
    arithmetic (no libm, no float)."""
    import decimal
    ctx = decimal.Context(prec=90)
    pi = decimal.Decimal(_PI80)
    j = k % M
    x = ctx.divide(ctx.multiply(2 * pi, decimal.Decimal(j)), decimal.Decimal(M))
    if x > pi:
        x = ctx.subtract(x, 2 * pi)                    # |x| <= pi
    x2 = ctx.multiply(x, x)
    c, s = decimal.Decimal(1), x
    tc, ts = decimal.Decimal(1), x
    eps = decimal.Decimal(10) ** -85
    n = 1
    while abs(tc) > eps or abs(ts) > eps:
        tc = ctx.divide(ctx.multiply(-tc, x2), decimal.Decimal((2 * n - 1) * (2 * n)))
        ts = ctx.divide(ctx.multiply(-ts, x2), decimal.Decimal((2 * n) * (2 * n + 1)))
        c, s = ctx.add(c, tc), ctx.add(s, ts)
        n += 1
    return c, s


def _is_nearest_f32(f: np.float32, exact) -> bool:
    """f is the fp32 value nearest `exact` (a Decimal), and not a tie."""
    import decimal
    f = np.float32(f)
    d = abs(decimal.Decimal(float(f)) - exact)
    for nb in (np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))):
        if not d < abs(decimal.Decimal(float(nb)) - exact):
            return False
    return True


def pin_twiddle_exact(o):
    """The twiddle table is the correctly rounded fp32 value of the exact root
    of unity, (cos, -sin)(2 pi k / M), checked against an independent 80-digit
    decimal evaluation; exact zeros are +0."""
    for M in (1, 2, 3, 4, 6, 8, 12, 16, 24, 32, 48, 64, 96, 128, 192, 256):
        for k in range(M):
            wr, wi = o.twiddle(k, M)
            c, s = _cos_sin_exact(k, M)
            cos_zero = (4 * k) % M == 0 and ((4 * k) // M) % 2 == 1     # 2 pi k / M = odd * pi/2
            sin_zero = (2 * k) % M == 0                                 # 2 pi k / M = n pi
            for got, want, zero in ((wr, c, cos_zero), (wi, -s, sin_zero)):
                if zero:
                    assert got == 0.0 and not np.signbit(got), (k, M, got)
                else:
                    assert _is_nearest_f32(got, want), (k, M, float(got), str(want)[:20])


def pin_twiddle_symmetries(o):
    """Exact values and symmetries of the roots, bit for bit: omega^0 = 1,
    omega^(M/4) = -i, omega^(M/2) = -1, omega^(M-k) = conj(omega^k),
    omega^(k+M/4) = -i omega^k and omega^(M/2-k) = -conj(omega^k)."""
    def b(v):
        return np.float32(v).view(np.uint32) if v != 0 else np.uint32(0)
    for M in (4, 8, 12, 16, 24, 32, 48, 64, 96, 128, 256):
        assert o.twiddle(0, M) == (1.0, 0.0)
        assert o.twiddle(M // 4, M) == (0.0, -1.0)
        assert o.twiddle(M // 2, M) == (-1.0, 0.0)
        for k in range(M):
            wr, wi = o.twiddle(k, M)
            cr, ci = o.twiddle(M - k, M)
            assert (b(cr), b(ci)) == (b(wr), b(-wi)), (k, M)
            rr, ri = o.twiddle(k + M // 4, M)
            assert (b(rr), b(ri)) == (b(wi), b(-wr)), (k, M)
            hr, hi = o.twiddle(M // 2 - k, M)
            assert (b(hr), b(hi)) == (b(-wr), b(wi)), (k, M)


def pin_fft_definition(o):
    """The fp32 FFT (forward DIF stages, mixed radix 2 and 3) lies within its
    rounding bound of numpy's fft; its transpose within the bound of N ifft
    (the conjugate DFT)."""
    rng = np.random.default_rng(44)
    for N in (1, 2, 3, 4, 6, 8, 12, 16, 24, 32, 48, 64, 96, 128):
        z = (rng.standard_normal((6, N)) + 1j * rng.standard_normal((6, N))).astype(np.complex64)
        z64 = z.astype(np.complex128)
        stages = max(1, math.ceil(math.log2(N)) + 1)
        bound = 8.0 * stages * U32 * np.abs(z64).sum(axis=1, keepdims=True)
        assert np.all(np.abs(o.fft_f32(z) - np.fft.fft(z64, axis=1)) <= bound), N
        assert np.all(np.abs(o.fft_f32(z, inverse=True) - N * np.fft.ifft(z64, axis=1)) <= bound), N


def pin_fft_exact_trivial_twiddles(o):
    """Where only the twiddles 1, -1, i and -i occur (N = 2 and 4), products by
    them are exact: small-integer inputs give numpy's fft exactly, and a unit
    input at position m gives the row of powers of -i with exact zeros."""
    rng = np.random.default_rng(45)
    for N in (2, 4):
        z = (rng.integers(-9, 10, (20, N)) + 1j * rng.integers(-9, 10, (20, N))).astype(np.complex64)
        want = np.fft.fft(z.astype(np.complex128), axis=1)
        assert np.array_equal(o.fft_f32(z).astype(np.complex128), want), N
        assert np.array_equal(o.fft_f32(z, inverse=True).astype(np.complex128),
                              N * np.fft.ifft(z.astype(np.complex128), axis=1)), N
    for m in range(4):
        e = np.zeros((1, 4), np.complex64)
        e[0, m] = 1.0
        got = o.fft_f32(e)[0]
        want = np.array([(-1j) ** (m * k) for k in range(4)])
        assert np.array_equal(got.astype(np.complex128), want.round()), (m, got)


# ---- decode attention over the int4 cache ------------------------------

def _nibbles(packed):
    """Independent unpack: low nibble first, 4-bit two's complement."""
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    q = np.stack([lo, hi], axis=-1).reshape(p.shape[:-1] + (p.shape[-1] * 2,))
    return np.where(q >= 8, q - 16, q).astype(np.float64)


def _rebuild(packed, scales, lam, s, G):
    """Rows of the cache in float64: (diag(s) H (codes . S) / sqrt D) / lambda,
    with scipy's Sylvester-Hadamard matrix."""
    import scipy.linalg
    q = _nibbles(packed)
    D = q.shape[-1]
    S = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64), G, axis=-1)
    H = scipy.linalg.hadamard(D).astype(np.float64)
    y = q * S
    return (y @ H.T) / math.sqrt(D) * s.astype(np.float64) / lam.astype(np.float64)


def _rebuild_fmt(packed, scales, lam, s, G, lambda_after, srft):
    """Rows of a codec-variant cache in float64: y = codes . S, then
    (diag(s) R^T y) / lambda (lambda before) or diag(s) R^T (y / lambda)
    (after), R^T = H / sqrt D (scipy's Hadamard matrix) or P^T, P the packed
    unitary real DFT built from numpy's rfft of the identity."""
    import scipy.linalg
    q = _nibbles(packed)
    D = q.shape[-1]
    S = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64), G, axis=-1)
    y = q * S
    l64, s64 = lam.astype(np.float64), s.astype(np.float64)
    if lambda_after:
        y = y / l64
    if srft:
        P = _rfft_packed(np.eye(D)).T                   # column j = P e_j
        x = y @ P                                       # rows of P^T y
    else:
        x = (y @ scipy.linalg.hadamard(D).astype(np.float64).T) / math.sqrt(D)
    x = x * s64
    return x if lambda_after else x / l64


def _attn_case(rng, B, Hq, Hkv, T, D, G, smax=2.0):
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    kp = rng.integers(0, 256, (B, Hkv, T, D // 2), dtype=np.uint8)
    vp = rng.integers(0, 256, (B, Hkv, T, D // 2), dtype=np.uint8)
    ks = rng.uniform(0.01, smax, (B, Hkv, T, D // G)).astype(np.float16)
    vs = rng.uniform(0.01, smax, (B, Hkv, T, D // G)).astype(np.float16)
    lk, sk = _rand_params(rng, D)
    lv, sv = _rand_params(rng, D)
    return q, kp, ks, vp, vs, lk, sk, lv, sv


def pin_attention_vs_sdpa(o):
    """The oracle equals torch's SDPA (float64) on independently rebuilt K, V,
    with grouped-query head mapping and per-sequence lengths."""
    import torch
    rng = np.random.default_rng(21)
    for B, Hq, Hkv, T, D, G, scale in ((2, 8, 2, 37, 32, 8, 0.3), (3, 4, 4, 20, 64, 32, 0.125),
                                       (1, 6, 1, 9, 16, 16, 1.7)):
        q, kp, ks, vp, vs, lk, sk, lv, sv = _attn_case(rng, B, Hq, Hkv, T, D, G)
        lens = rng.integers(1, T + 1, B)
        lens[0] = T
        got = o.attention_decode(q, kp, ks, vp, vs, lens, lk, sk, lv, sv, G, scale)
        K = _rebuild(kp, ks, lk, sk, G)
        V = _rebuild(vp, vs, lv, sv, G)
        R = Hq // Hkv
        for b in range(B):
            L = int(lens[b])
            kt = torch.from_numpy(K[b, :, :L]).repeat_interleave(R, dim=0)[None]
            vt = torch.from_numpy(V[b, :, :L]).repeat_interleave(R, dim=0)[None]
            qt = torch.from_numpy(q[b].astype(np.float64))[None, :, None, :]
            ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
            ref = ref[0, :, 0, :].numpy()
            err = np.abs(got[b] - ref).max()
            assert err <= 1e-12 * max(1.0, np.abs(ref).max()), f"attention off by {err}"


def pin_attention_closed_forms(o):
    """One key: o = V_0.  Zero scale: o = mean of V.  Huge scale: o = V at the
    key with the largest score.  Both compared with the fp32 inverse path."""
    rng = np.random.default_rng(22)
    B, Hq, Hkv, T, D, G = 2, 4, 2, 16, 64, 16
    q, kp, ks, vp, vs, lk, sk, lv, sv = _attn_case(rng, B, Hq, Hkv, T, D, G)
    def deq(b, kv, t, packed, scales, lam, s):
        return o.dequantize_f32(o.unpack(packed[b, kv, t]), scales[b, kv, t], lam, s, G)[0]
    one = o.attention_decode(q, kp, ks, vp, vs, [1, 1], lk, sk, lv, sv, G, 0.5)
    for b in range(B):
        for h in range(Hq):
            ref = deq(b, h // 2, 0, vp, vs, lv, sv).astype(np.float64)
            assert np.abs(one[b, h] - ref).max() <= 1e-5 * np.abs(ref).max()
    mean = o.attention_decode(q, kp, ks, vp, vs, [T, 5], lk, sk, lv, sv, G, 0.0)
    for b, L in ((0, T), (1, 5)):
        for h in range(Hq):
            ref = np.mean([deq(b, h // 2, t, vp, vs, lv, sv) for t in range(L)], axis=0)
            assert np.abs(mean[b, h] - ref).max() <= 1e-5 * np.abs(ref).max()
    # huge scale: the softmax is one-hot at the arg-max of the scores
    K = _rebuild(kp, ks, lk, sk, G)
    hard = o.attention_decode(q, kp, ks, vp, vs, [T, T], lk, sk, lv, sv, G, 1e4)
    for b in range(B):
        for h in range(Hq):
            z = K[b, h // 2] @ q[b, h].astype(np.float64)
            top = np.sort(z)[-2:]
            if top[1] - top[0] < 1e-2:
                continue
            ref = deq(b, h // 2, int(np.argmax(z)), vp, vs, lv, sv)
            assert np.all(np.isfinite(hard[b, h]))
            assert np.abs(hard[b, h] - ref).max() <= 1e-5 * np.abs(ref).max()


def pin_attention_formats_vs_sdpa(o):
    """Over caches of every codec-variant format (lambda before or after the
    rotation, Walsh-Hadamard or SRFT rows, the mixed-radix D = 96 included),
    the oracle equals torch's SDPA (float64) on K and V rebuilt independently
    with scipy's Hadamard matrix or numpy's rfft."""
    import torch
    rng = np.random.default_rng(24)
    cases = ((2, 8, 2, 23, 32, 8), (1, 4, 1, 17, 96, 32), (2, 6, 3, 11, 64, 16))
    for B, Hq, Hkv, T, D, G in cases:
        for after in (False, True):
            for srft in (False, True):
                if D == 96 and not srft:
                    continue
                q, kp, ks, vp, vs, lk, sk, lv, sv = _attn_case(rng, B, Hq, Hkv, T, D, G)
                lens = rng.integers(1, T + 1, B)
                got = o.attention_decode(q, kp, ks, vp, vs, lens, lk, sk, lv, sv, G, 0.45,
                                         lambda_after=after, srft=srft)
                K = _rebuild_fmt(kp, ks, lk, sk, G, after, srft)
                V = _rebuild_fmt(vp, vs, lv, sv, G, after, srft)
                R = Hq // Hkv
                for b in range(B):
                    L = int(lens[b])
                    kt = torch.from_numpy(K[b, :, :L]).repeat_interleave(R, dim=0)[None]
                    vt = torch.from_numpy(V[b, :, :L]).repeat_interleave(R, dim=0)[None]
                    qt = torch.from_numpy(q[b].astype(np.float64))[None, :, None, :]
                    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=0.45)
                    ref = ref[0, :, 0, :].numpy()
                    err = np.abs(got[b] - ref).max()
                    assert err <= 1e-11 * max(1.0, np.abs(ref).max()), (D, after, srft, err)


def pin_attention_formats_closed_forms(o):
    """SRFT and lambda-after caches: one key gives that key's value row (the
    codec's own fp32 dequantisation of it, within its rounding), a zero score
    scale gives the mean of the value rows."""
    rng = np.random.default_rng(25)
    B, Hq, Hkv, T, D, G = 1, 2, 1, 6, 64, 16
    for after, srft in ((True, False), (False, True), (True, True)):
        q, kp, ks, vp, vs, lk, sk, lv, sv = _attn_case(rng, B, Hq, Hkv, T, D, G)
        rows = o.dequantize_ex(vp[0, 0], vs[0, 0], lv, sv, G, lambda_after=after,
                               srft=srft).astype(np.float64)
        one = o.attention_decode(q, kp, ks, vp, vs, [1], lk, sk, lv, sv, G, 0.5,
                                 lambda_after=after, srft=srft)
        for h in range(Hq):
            assert np.abs(one[0, h] - rows[0]).max() <= 2e-3 * np.abs(rows[0]).max()
        mean = o.attention_decode(q, kp, ks, vp, vs, [T], lk, sk, lv, sv, G, 0.0,
                                  lambda_after=after, srft=srft)
        for h in range(Hq):
            ref = rows.mean(axis=0)
            assert np.abs(mean[0, h] - ref).max() <= 2e-3 * np.abs(rows).max()


def pin_attention_masking(o):
    """Entries past a sequence's length do not matter; length 0 gives 0."""
    rng = np.random.default_rng(23)
    B, Hq, Hkv, T, D, G = 2, 2, 1, 12, 32, 32
    q, kp, ks, vp, vs, lk, sk, lv, sv = _attn_case(rng, B, Hq, Hkv, T, D, G)
    a = o.attention_decode(q, kp, ks, vp, vs, [7, 0], lk, sk, lv, sv, G, 0.4)
    kp2, vp2, ks2 = kp.copy(), vp.copy(), ks.copy()
    kp2[:, :, 7:] ^= 0x5A
    vp2[:, :, 7:] ^= 0xA5
    ks2[:, :, 7:] = np.float16(60000.0)
    b = o.attention_decode(q, kp2, ks2, vp2, vs, [7, 0], lk, sk, lv, sv, G, 0.4)
    assert np.array_equal(a, b)
    assert np.all(a[1] == 0.0)


ALL_PINS = [
    pin_f16_conversion, pin_norm_const, pin_fwht_dense, pin_rotation_dense,
    pin_rotate_f32, pin_norm_preservation, pin_roundtrip_unquantized,
    pin_code_invariants, pin_error_bound, pin_dequant_vs_f64,
    pin_special_cases, pin_worked_examples, pin_divform_near_ties,
    pin_pack_layout, pin_accounting,
    pin_attention_vs_sdpa, pin_attention_closed_forms, pin_attention_masking,
    pin_attention_formats_vs_sdpa, pin_attention_formats_closed_forms,
    pin_ex_matches_base, pin_ex_definition, pin_ex_int8_codes, pin_ex_tables,
    pin_ex_roundtrip_bound, pin_ex_impulse,
    pin_srft_definition, pin_srft_f32, pin_srft_closed_forms, pin_srft_codec,
    pin_twiddle_exact, pin_twiddle_symmetries, pin_fft_definition,
    pin_fft_exact_trivial_twiddles,
]
