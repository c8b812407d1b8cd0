"""The tensor-core dequantizer (kvq_dequantize_tc: the Walsh-Hadamard
transform's in-group factor as m16n8k16 tensor-core products on the integer
codes, the cross-group stages as fp32 butterflies) against the oracle and the
butterfly dequantizer: fp16 output bit-identical, for every group size it
takes, on ragged sizes, the edge rows and a large sampled batch."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_02_b200 import kvq, workloads

pytestmark = pytest.mark.gpu

D = 128


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("G", [16, 32, 64])
@pytest.mark.parametrize("n", [1, 31, 1000, 77777])
def test_tc_matches_oracle(G, n):
    o = oracle.get()
    w = workloads.WORKLOADS["qwen3-8b-prefill"]
    x16 = workloads.host_rows(w, n, seed_offset=G + n)
    lam, s = workloads.params(D, 3)
    pk, sc = o.quantize(x16, lam, s, G)
    ref = o.dequantize(pk, sc, lam, s, G)
    got = kvq.dequantize(_dev(pk), _dev(sc), _dev(lam), _dev(s), G, tensor_cores=True)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy().view(np.uint16), ref.view(np.uint16)), \
        f"{int((got.cpu().numpy().view(np.uint16) != ref.view(np.uint16)).sum())} outputs differ"


@pytest.mark.parametrize("G", [16, 32, 64])
def test_tc_edge_rows_and_random_codes(G):
    """Zero, spike, constant, fp16-extreme and subnormal rows, and codes drawn
    uniformly over all nibbles with scales over six orders of magnitude
    (subnormal scales included): exact-zero outputs keep their signs."""
    o = oracle.get()
    lam, s = workloads.params(D, 5)
    x16 = workloads.adversarial_rows(D)
    pk, sc = o.quantize(x16, lam, s, G)
    rng = np.random.default_rng(G)
    pk2 = rng.integers(0, 256, (333, D // 2), dtype=np.uint8)
    sc2 = (10.0 ** rng.uniform(-6, 0, (333, D // G))).astype(np.float16)
    pk = np.concatenate([pk, pk2])
    sc = np.concatenate([sc, sc2])
    ref = o.dequantize(pk, sc, lam, s, G)
    got = kvq.dequantize(_dev(pk), _dev(sc), _dev(lam), _dev(s), G, tensor_cores=True)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy().view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("G", [32, 64])
def test_tc_equals_butterfly_kernel_large(G):
    """2^21 device-drawn rows: the tensor-core and butterfly dequantizers give
    the same bytes; 4-byte-misaligned scales take the direct-load path."""
    w = workloads.WORKLOADS["qwen3-8b-prefill"]
    n = (1 << 21) + 13
    x = workloads.device_rows(w, n, torch.device("cuda"))
    lam, s = workloads.params(D, w.seed)
    lt, st = _dev(lam), _dev(s)
    pk, sc = kvq.quantize(x, lt, st, G)
    a = kvq.dequantize(pk, sc, lt, st, G)
    b = kvq.dequantize(pk, sc, lt, st, G, tensor_cores=True)
    sc_off = torch.empty(n * (D // G) + 1, dtype=torch.float16, device="cuda")[1:].view(n, D // G)
    sc_off.copy_(sc)
    c = kvq.dequantize(pk, sc_off, lt, st, G, tensor_cores=True)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))
