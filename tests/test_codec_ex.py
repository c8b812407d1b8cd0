"""Format variants of the codec (kvq_quantize_ex / kvq_dequantize_ex) against
the oracle's kvqo_quantize_ex / kvqo_dequantize_ex: codes, scales and
dequantised fp16 output bit-identical, for every group size, both code widths,
both lambda positions and both rotations (WHT, SRFT), with one lambda table or
several, on ragged sizes, the edge rows and a large sampled batch; the SRFT at
every length it supports (D = 64, 128, 256 and the mixed-radix D = 96)."""
import itertools

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_02_b200 import kvq, workloads

pytestmark = pytest.mark.gpu

D = 128
COMBOS = list(itertools.product((16, 32, 64), (4, 8), (False, True), (False, True)))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(x16, lam, s, G, bits, after, rows=None, srft=False):
    codes, scales = kvq.quantize_ex(_dev(x16), _dev(lam), _dev(s), G, bits=bits,
                                    lambda_after=after, lambda_rows=rows, srft=srft)
    back = kvq.dequantize_ex(codes, scales, _dev(lam), _dev(s), G, bits=bits,
                             lambda_after=after, lambda_rows=rows, srft=srft)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), back.cpu().numpy()


def _compare(o, x16, lam, s, G, bits, after, rows=None, label="", srft=False):
    codes, scales, back = _run(x16, lam, s, G, bits, after, rows, srft)
    oc, os_ = o.quantize_ex(x16, lam, s, G, bits=bits, lambda_after=after, lambda_rows=rows, srft=srft)
    ob = o.dequantize_ex(oc, os_, lam, s, G, bits=bits, lambda_after=after, lambda_rows=rows, srft=srft)
    assert np.array_equal(scales.view(np.uint16), os_.view(np.uint16)), f"{label}: scales differ"
    assert np.array_equal(codes, oc), f"{label}: {int((codes != oc).sum())} code bytes differ"
    assert np.array_equal(back.view(np.uint16), ob.view(np.uint16)), f"{label}: dequant differs"


@pytest.mark.parametrize("G,bits,after,srft", COMBOS)
def test_variant_matches_oracle(G, bits, after, srft):
    o = oracle.get()
    w = workloads.WORKLOADS["qwen3-8b-prefill"]
    x16 = workloads.host_rows(w, 1000, seed_offset=G + bits + int(after))   # ragged: 31 tiles + 8
    lam, s = workloads.params(D, 7)
    _compare(o, x16, lam, s, G, bits, after, srft=srft,
             label=f"G{G} b{bits} after{int(after)} srft{int(srft)}")


@pytest.mark.parametrize("G,bits,after,srft", [(32, 4, False, False), (32, 8, True, False),
                                               (16, 4, True, True), (64, 8, False, True)])
def test_variant_lambda_tables(G, bits, after, srft):
    """Three tables over 64-row ranges: row r uses table (r // 64) % 3."""
    o = oracle.get()
    w = workloads.WORKLOADS["qwen2.5-1.5b"]
    x16 = workloads.host_rows(w, 777, seed_offset=3)
    rng = np.random.default_rng(11)
    tables = rng.uniform(0.5, 2.0, (3, D)).astype(np.float32)
    _, s = workloads.params(D, 8)
    _compare(o, x16, tables, s, G, bits, after, rows=64, label="tables", srft=srft)


@pytest.mark.parametrize("bits,after,srft", list(itertools.product((4, 8), (False, True), (False, True))))
def test_variant_edge_rows(bits, after, srft):
    o = oracle.get()
    x16 = workloads.adversarial_rows(D)
    lam, s = workloads.params(D, 9)
    _compare(o, x16, lam, s, 32, bits, after, label="edge", srft=srft)


def test_base_options_equal_base_codec():
    """bits 4, lambda before, one table: the same bytes as kvq_quantize."""
    w = workloads.WORKLOADS["qwen3-8b-prefill"]
    x = workloads.device_rows(w, 100_000, torch.device("cuda"))
    lam, s = workloads.params(D, w.seed)
    lt, st = _dev(lam), _dev(s)
    p1, s1 = kvq.quantize(x, lt, st, 32)
    p2, s2 = kvq.quantize_ex(x, lt, st, 32)
    d1 = kvq.dequantize(p1, s1, lt, st, 32)
    d2 = kvq.dequantize_ex(p2, s2, lt, st, 32)
    torch.cuda.synchronize()
    assert torch.equal(p1, p2) and torch.equal(s1.view(torch.int16), s2.view(torch.int16))
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


@pytest.mark.parametrize("bits,after,srft", [(8, True, False), (4, True, True), (4, False, True)])
def test_variant_large_sampled(bits, after, srft):
    """2^21 device-drawn rows with per-(layer, head) tables: sampled rows against
    the oracle, every row's scales consistent with its codes."""
    o = oracle.get()
    w = workloads.WORKLOADS["qwen3-8b-prefill"]
    n, G, rows_per = 1 << 21, 32, 4096
    x = workloads.device_rows(w, n, torch.device("cuda"))
    rng = np.random.default_rng(12)
    tables = rng.uniform(0.5, 2.0, (16, D)).astype(np.float32)
    _, s = workloads.params(D, 13)
    codes, scales = kvq.quantize_ex(x, _dev(tables), _dev(s), G, bits=bits, lambda_after=after,
                                    lambda_rows=rows_per, srft=srft)
    back = kvq.dequantize_ex(codes, scales, _dev(tables), _dev(s), G, bits=bits,
                             lambda_after=after, lambda_rows=rows_per, srft=srft)
    torch.cuda.synchronize()
    idx = np.sort(rng.choice(n, 4096, replace=False))
    it = torch.from_numpy(idx).cuda()
    xs = x[it].cpu().numpy()
    for k, r in enumerate(idx):
        t = tables[(r // rows_per) % 16]
        oc, os_ = o.quantize_ex(xs[k:k + 1], t, s, G, bits=bits, lambda_after=after, srft=srft)
        assert np.array_equal(codes[r].cpu().numpy()[None], oc), f"row {r}"
        assert np.array_equal(scales[r].cpu().numpy().view(np.uint16)[None], os_.view(np.uint16))
        ob = o.dequantize_ex(oc, os_, t, s, G, bits=bits, lambda_after=after, srft=srft)
        assert np.array_equal(back[r].cpu().numpy().view(np.uint16)[None], ob.view(np.uint16))
        if k >= 255:
            break


# ---- the SRFT at every supported length ------------------------------------

SRFT_DG = [(64, 16), (64, 32), (64, 64), (96, 16), (96, 32), (128, 16), (128, 32), (128, 64),
           (256, 16), (256, 32), (256, 64)]


def _rows(D, n, seed, outliers=4, gain=20.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, D))
    ch = rng.permutation(D)[:outliers]
    x[:, ch] *= gain
    return x.astype(np.float16)


@pytest.mark.parametrize("bits,after", [(4, False), (4, True), (8, False), (8, True)])
@pytest.mark.parametrize("D,G", SRFT_DG)
def test_srft_lengths_match_oracle(D, G, bits, after):
    """Ragged batches: 1000 rows span 31 full warp tiles and a partial one (62
    and a partial one at D = 256, where a warp tile is 16 rows)."""
    o = oracle.get()
    x16 = _rows(D, 1000, seed=D + G + bits + int(after))
    lam, s = workloads.params(D, 17 + D)
    _compare(o, x16, lam, s, G, bits, after, srft=True, label=f"D{D} G{G} b{bits} after{int(after)}")


@pytest.mark.parametrize("bits,after", [(4, False), (4, True), (8, False), (8, True)])
@pytest.mark.parametrize("D", [64, 96, 256])
def test_srft_lengths_edge_rows(D, bits, after):
    """Zero, spike, constant, tie-making, fp16-extreme and subnormal rows: zero
    signs of exact-zero outputs included, bit for bit."""
    o = oracle.get()
    x16 = workloads.adversarial_rows(D)
    lam, s = workloads.params(D, 19)
    _compare(o, x16, lam, s, 32, bits, after, srft=True, label=f"edge D{D}")


@pytest.mark.parametrize("D,G,bits,after", [(96, 16, 4, True), (256, 32, 4, True), (256, 64, 8, False),
                                            (64, 32, 8, True)])
def test_srft_lengths_lambda_tables(D, G, bits, after):
    """Five tables over 96-row ranges: row r uses table (r // 96) % 5."""
    o = oracle.get()
    x16 = _rows(D, 1111, seed=5)
    rng = np.random.default_rng(23)
    tables = rng.uniform(0.5, 2.0, (5, D)).astype(np.float32)
    _, s = workloads.params(D, 24)
    _compare(o, x16, tables, s, G, bits, after, rows=96, srft=True, label=f"tables D{D}")


@pytest.mark.parametrize("D,bits,after", [(256, 4, True), (96, 4, True), (256, 8, False)])
def test_srft_lengths_large_sampled(D, bits, after):
    """2^20 device-drawn rows with per-(layer, head) tables: 256 sampled rows
    against the oracle, codes, scales and dequantised output."""
    o = oracle.get()
    n, G, rows_per = 1 << 20, 32, 4096
    gen = torch.Generator(device="cuda").manual_seed(D)
    x = (torch.randn((n, D), generator=gen, device="cuda") * 3.0).to(torch.float16)
    rng = np.random.default_rng(29)
    tables = rng.uniform(0.5, 2.0, (8, D)).astype(np.float32)
    _, s = workloads.params(D, 31)
    codes, scales = kvq.quantize_ex(x, _dev(tables), _dev(s), G, bits=bits, lambda_after=after,
                                    lambda_rows=rows_per, srft=True)
    back = kvq.dequantize_ex(codes, scales, _dev(tables), _dev(s), G, bits=bits,
                             lambda_after=after, lambda_rows=rows_per, srft=True)
    torch.cuda.synchronize()
    idx = np.sort(rng.choice(n, 256, replace=False))
    it = torch.from_numpy(idx).cuda()
    xs, cs, ss, bs = (t[it].cpu().numpy() for t in (x, codes, scales, back))
    for k, r in enumerate(idx):
        t = tables[(r // rows_per) % 8]
        oc, os_ = o.quantize_ex(xs[k:k + 1], t, s, G, bits=bits, lambda_after=after, srft=True)
        assert np.array_equal(cs[k:k + 1], oc), f"row {r}"
        assert np.array_equal(ss[k:k + 1].view(np.uint16), os_.view(np.uint16)), f"row {r}"
        ob = o.dequantize_ex(oc, os_, t, s, G, bits=bits, lambda_after=after, srft=True)
        assert np.array_equal(bs[k:k + 1].view(np.uint16), ob.view(np.uint16)), f"row {r}"


def test_srft_rejects_bad_lengths():
    x = torch.zeros((4, 96), dtype=torch.float16, device="cuda")
    lam, s = workloads.params(96, 1)
    with pytest.raises(kvq.KvqError):
        kvq.quantize_ex(x, _dev(lam), _dev(s), 64, srft=True)        # 64 does not divide 96
    with pytest.raises(kvq.KvqError):
        kvq.quantize_ex(x, _dev(lam), _dev(s), 32, srft=False)       # no Walsh-Hadamard at 96
