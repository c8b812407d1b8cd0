"""Seeded synthetic KV-cache inputs shaped like the caches the method was
measured on (Qwen2.5-1.5B, Gemma-3-1B, Qwen3-8B).

This module only draws random inputs -- the fp16 KV rows, the per-channel
lambda and the random +-1 signs.  It holds none of the method's arithmetic and
is the one module that both the CUDA path's callers and the oracle's tests
import.  There are no model weights or activations here: every input is
synthetic, with the shape and value statistics described for each workload.

A "vector" is one (layer, K|V, kv-head, token) row of length D; a cache
[layers][2][heads][tokens][D] is flattened row-major to [n_vec, D].
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_vec: int
    D: int
    groups: tuple
    dist: str                      # "normal" | "student_t3"
    outlier_channels: int          # channels (per row) multiplied by outlier_gain
    outlier_gain: float
    channel_scale_logu: tuple | None   # per-channel scale ~ LogUniform[lo, hi]
    seed: int
    shape: dict                    # the cache shape that n_vec flattens
    note: str = ""


def _n(shape: dict) -> int:
    return int(math.prod(shape.values()))


_TINY = dict(vectors=256)
_QWEN25 = dict(layers=28, kv=2, heads=2, tokens=4096)
_GEMMA3 = dict(layers=26, kv=2, heads=1, tokens=4096)
_QWEN3 = dict(layers=36, kv=2, heads=8, tokens=32768)
_DECODE_NEW = dict(seqs=64, layers=36, kv=2, heads=8, tokens=1)
_DECODE_CACHE = dict(seqs=64, layers=36, kv=2, heads=8, tokens=4096)

WORKLOADS = {
    "tiny": Workload(
        "tiny", _n(_TINY), 128, (32,), "normal", 4, 20.0, None, 0, _TINY,
        "256 vectors, one head, N(0,1) with 4 seeded outlier channels x20"),
    "qwen2.5-1.5b": Workload(
        "qwen2.5-1.5b", _n(_QWEN25), 128, (32,), "student_t3", 0, 1.0,
        (0.1, 10.0), 1, _QWEN25,
        "28 layers x 2 KV heads x 4096 tokens, K and V; Student-t(3) with a "
        "per-channel LogU[0.1, 10] scale"),
    "gemma-3-1b": Workload(
        "gemma-3-1b", _n(_GEMMA3), 256, (32, 64), "normal", 8, 30.0, None, 2,
        _GEMMA3,
        "26 layers x 1 KV head x 4096 tokens, K and V; N(0,1) with 8 outlier "
        "channels x30"),
    "qwen3-8b-prefill": Workload(
        "qwen3-8b-prefill", _n(_QWEN3), 128, (32,), "student_t3", 4, 20.0,
        None, 3, _QWEN3,
        "36 layers x 8 KV heads x 32768 tokens, K and V; Student-t(3) with 4 "
        "outlier channels x20"),
    "decode-append": Workload(
        "decode-append", _n(_DECODE_NEW), 128, (32,), "normal", 0, 1.0, None,
        4, _DECODE_NEW,
        "one new token for 64 sequences x 36 layers x 8 KV heads, K and V; "
        "N(0,1)"),
    "decode-cache": Workload(
        "decode-cache", _n(_DECODE_CACHE), 128, (32,), "normal", 0, 1.0, None,
        5, _DECODE_CACHE,
        "the int4 cache the decode step reads back: 64 sequences x 36 layers x "
        "8 KV heads x 4096 tokens, K and V; N(0,1)"),
}

FP16_CLIP = 60000.0   # magnitudes are clipped below the fp16 maximum


def params(D: int, seed: int):
    """lambda ~ U[0.5, 2] (float32[D]) and Rademacher signs (int8[D])."""
    rng = np.random.default_rng([seed, 0x1A3B])
    lam = rng.uniform(0.5, 2.0, size=D).astype(np.float32)
    signs = np.where(rng.random(D) < 0.5, -1, 1).astype(np.int8)
    return lam, signs


def channel_gain(w: Workload) -> np.ndarray:
    """Per-channel multiplier: outlier channels (seeded permutation) times the
    optional LogUniform per-channel scale.  float32[D]."""
    rng = np.random.default_rng([w.seed, 0x5EED])
    gain = np.ones(w.D, dtype=np.float64)
    if w.outlier_channels:
        idx = rng.permutation(w.D)[: w.outlier_channels]
        gain[idx] *= w.outlier_gain
    if w.channel_scale_logu is not None:
        lo, hi = w.channel_scale_logu
        gain *= np.exp(rng.uniform(math.log(lo), math.log(hi), size=w.D))
    return gain.astype(np.float32)


def host_rows(w: Workload, n: int, seed_offset: int = 0) -> np.ndarray:
    """n rows of the workload's distribution drawn on the host (numpy PCG64).
    float16[n, D]."""
    rng = np.random.default_rng([w.seed, 0xC0DE, seed_offset])
    if w.dist == "normal":
        z = rng.standard_normal((n, w.D))
    elif w.dist == "student_t3":
        z = rng.standard_t(3, size=(n, w.D))
    else:
        raise ValueError(w.dist)
    z *= channel_gain(w).astype(np.float64)
    np.clip(z, -FP16_CLIP, FP16_CLIP, out=z)
    return z.astype(np.float16)


def device_rows(w: Workload, n: int, device, seed_offset: int = 0,
                chunk_rows: int = 1 << 19, out=None):
    """n rows of the workload's distribution drawn on a CUDA device with torch's
    Philox generator, in chunks, straight into an fp16 [n, D] tensor."""
    import torch

    if out is None:
        out = torch.empty((n, w.D), dtype=torch.float16, device=device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed * 1_000_003 + seed_offset)
    gain = torch.from_numpy(channel_gain(w)).to(device)
    for r0 in range(0, n, chunk_rows):
        r1 = min(n, r0 + chunk_rows)
        z = torch.randn((r1 - r0, w.D), generator=gen, device=device,
                        dtype=torch.float32)
        if w.dist == "student_t3":
            chi = torch.randn((3, r1 - r0, w.D), generator=gen, device=device,
                              dtype=torch.float32)
            chi2 = (chi * chi).sum(0)
            z = z / torch.sqrt(chi2 / 3.0)
            del chi, chi2
        elif w.dist != "normal":
            raise ValueError(w.dist)
        z = z * gain
        z.clamp_(-FP16_CLIP, FP16_CLIP)
        out[r0:r1].copy_(z)
    return out


def adversarial_rows(D: int) -> np.ndarray:
    """Hand-picked edge rows: all zero, one spike, constant, powers of two that
    make exact ties, fp16 extremes and subnormals.  float16[k, D]."""
    rows = []
    rows.append(np.zeros(D))
    spike = np.zeros(D); spike[D // 3] = 1000.0; rows.append(spike)
    rows.append(np.full(D, 0.75))
    rows.append(np.full(D, -3.0))
    alt = np.array([(-1.0) ** i * 2.0 ** (i % 5 - 2) for i in range(D)]); rows.append(alt)
    rows.append(np.full(D, 65504.0))
    big = np.zeros(D); big[0] = -65504.0; big[1] = 65504.0; rows.append(big)
    rows.append(np.full(D, 2.0 ** -24))                  # smallest subnormal
    sub = np.array([(i % 7 - 3) * 2.0 ** -20 for i in range(D)]); rows.append(sub)
    ramp = np.linspace(-8.0, 8.0, D); rows.append(ramp)
    half = np.array([0.5 * (i % 16) - 4.0 for i in range(D)]); rows.append(half)
    return np.stack(rows).astype(np.float16)
