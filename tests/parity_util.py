"""Comparison helpers for the GPU-vs-oracle parity tests.

The bar (from the method's target): int4 codes and fp16 scales bit-exact,
except that a code whose oracle value y*r lies within 1e-6 of a rounding tie
may differ by +-1, on at most 1e-5 of the elements; dequantised fp16 output
within 1e-3 absolute of the oracle.  Because the GPU kernels mirror the
oracle's rounding points one for one, the expected number of exempted codes
is zero and the dequantised output is expected to be bit-identical; the
helpers report both counts.
"""
from __future__ import annotations

import numpy as np

TIE_EPS = 1e-6
TIE_FRACTION = 1e-5
DEQUANT_ATOL = 1e-3


def check_quant(o, x16, lam, signs, G, gpu_packed, gpu_scales, label=""):
    """Returns the number of tie-exempted code differences (asserts the bar)."""
    packed_o, scales_o = o.quantize(x16, lam, signs, G)
    gs = np.ascontiguousarray(gpu_scales).view(np.uint16)
    os_ = scales_o.view(np.uint16)
    if not np.array_equal(gs, os_):
        bad = np.argwhere(gs != os_)
        r, j = bad[0]
        raise AssertionError(
            f"{label}: {len(bad)} scale(s) differ; first at row {r} group {j}: "
            f"gpu {gs[r, j]:#06x} oracle {os_[r, j]:#06x}")
    if np.array_equal(gpu_packed, packed_o):
        return 0
    qg = o.unpack(np.ascontiguousarray(gpu_packed)).astype(np.int32)
    qo = o.unpack(packed_o).astype(np.int32)
    mism = qg != qo
    n_mism = int(mism.sum())
    assert np.abs(qg - qo)[mism].max() == 1, f"{label}: a code differs by more than 1"
    y = o.rotate_f32(x16, lam, signs)
    Sf = scales_o.astype(np.float32)
    r = np.where(Sf == 0, np.float32(0), np.float32(1) / np.where(Sf == 0, 1, Sf)).astype(np.float32)
    t = (y * np.repeat(r, G, axis=1)).astype(np.float64)
    dist = np.abs(np.abs(t - np.floor(t)) - 0.5)
    assert np.all(dist[mism] <= TIE_EPS * np.maximum(1.0, np.abs(t[mism]))), \
        f"{label}: {n_mism} code(s) differ away from a rounding tie"
    assert n_mism <= TIE_FRACTION * qg.size, f"{label}: {n_mism} tie differences exceed 1e-5"
    return n_mism


def check_dequant(o, packed, scales, lam, signs, G, gpu_out, label=""):
    """Returns the number of fp16 outputs not bit-identical (asserts 1e-3)."""
    ref = o.dequantize(np.ascontiguousarray(packed), np.ascontiguousarray(scales), lam, signs, G)
    g = np.ascontiguousarray(gpu_out)
    same = g.view(np.uint16) == ref.view(np.uint16)
    if same.all():
        return 0
    gf = g.astype(np.float64)
    rf = ref.astype(np.float64)
    both_inf = np.isinf(gf) & np.isinf(rf) & (np.sign(gf) == np.sign(rf))
    diff = np.where(both_inf, 0.0, np.abs(gf - rf))
    worst = np.unravel_index(np.argmax(diff), diff.shape)
    assert diff.max() <= DEQUANT_ATOL, (
        f"{label}: dequant differs by {diff.max():.3g} at {worst}: gpu {gf[worst]} "
        f"oracle {rf[worst]}")
    return int((~same).sum())
