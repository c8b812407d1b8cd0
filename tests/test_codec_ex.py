"""Format variants of the codec (kvq_quantize_ex / kvq_dequantize_ex) against
the oracle's kvqo_quantize_ex / kvqo_dequantize_ex: codes, scales and
dequantised fp16 output bit-identical, for every group size, both code widths,
both lambda positions and both rotations (WHT, SRFT), with one lambda table or
several, on ragged sizes, the edge rows and a large sampled batch."""
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
