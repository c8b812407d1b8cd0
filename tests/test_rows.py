"""kvq_quantize_rows: encode new vectors straight into chosen rows of a cache
(the decode-time append), checked against the oracle row by row; rows not
named stay untouched, out-of-range indices are skipped and reported."""
import numpy as np
import pytest

import oracle
from kv_cache_quantization_02_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D,G", [(128, 32), (64, 16), (256, 64)])
def test_scatter_into_cache(D, G):
    import torch
    from kv_cache_quantization_02_b200 import kvq
    o = oracle.get()
    dev = torch.device("cuda")
    N, n = 3001, 777
    lam, s = workloads.params(D, seed=31)
    rng = np.random.default_rng(D + G)
    x16 = (rng.standard_normal((n, D)) * 4).astype(np.float16)
    idx = rng.permutation(N)[:n].astype(np.int64)
    packed = torch.full((N, D // 2), 0x5A, dtype=torch.uint8, device=dev)
    scales = torch.full((N, D // G), 77.0, dtype=torch.float16, device=dev)
    kvq.quantize_rows(torch.from_numpy(x16).to(dev), torch.from_numpy(lam).to(dev),
                      torch.from_numpy(s).to(dev), G, torch.from_numpy(idx).to(dev),
                      packed, scales)
    torch.cuda.synchronize()
    pk, sc = packed.cpu().numpy(), scales.cpu().numpy()
    p_ref, s_ref = o.quantize(x16, lam, s, G)
    assert np.array_equal(pk[idx], p_ref)
    assert np.array_equal(sc[idx].view(np.uint16), s_ref.view(np.uint16))
    rest = np.setdiff1d(np.arange(N), idx)
    assert np.all(pk[rest] == 0x5A) and np.all(sc[rest] == np.float16(77.0))


def test_out_of_range_indices_are_skipped():
    import torch
    from kv_cache_quantization_02_b200 import kvq
    o = oracle.get()
    dev = torch.device("cuda")
    D, G, N = 128, 32, 64
    lam, s = workloads.params(D, seed=32)
    x16 = (np.random.default_rng(5).standard_normal((6, D))).astype(np.float16)
    idx = np.array([3, -1, 10, N, 40, 1 << 40], dtype=np.int64)
    packed = torch.zeros((N, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.zeros((N, D // G), dtype=torch.float16, device=dev)
    kvq.kvq_fault_status(clear=True)
    kvq.quantize_rows(torch.from_numpy(x16).to(dev), torch.from_numpy(lam).to(dev),
                      torch.from_numpy(s).to(dev), G, torch.from_numpy(idx).to(dev),
                      packed, scales)
    torch.cuda.synchronize()
    assert kvq.kvq_fault_status(clear=True) & 4
    good = [0, 2, 4]
    p_ref, _ = o.quantize(x16[good], lam, s, G)
    pk = packed.cpu().numpy()
    assert np.array_equal(pk[idx[good]], p_ref)
    untouched = np.setdiff1d(np.arange(N), idx[good])
    assert not pk[untouched].any()


def test_decode_append_shape():
    """One new K and V token for 64 sequences x 36 layers x 8 KV heads,
    appended at token 100 of a 128-token slot per (sequence, layer, head)."""
    import torch
    from kv_cache_quantization_02_b200 import kvq
    o = oracle.get()
    dev = torch.device("cuda")
    w = workloads.WORKLOADS["decode-append"]
    D, G, n = w.D, 32, w.n_vec
    T = 128
    lam, s = workloads.params(D, w.seed)
    x = workloads.device_rows(w, n, dev)
    idx = torch.arange(n, device=dev, dtype=torch.int64) * T + 100
    packed = torch.zeros((n * T, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.zeros((n * T, D // G), dtype=torch.float16, device=dev)
    kvq.quantize_rows(x, torch.from_numpy(lam).to(dev), torch.from_numpy(s).to(dev), G, idx,
                      packed, scales)
    torch.cuda.synchronize()
    p_ref, s_ref = o.quantize(x.cpu().numpy(), lam, s, G)
    assert np.array_equal(packed[idx].cpu().numpy(), p_ref)
    assert np.array_equal(scales[idx].cpu().numpy().view(np.uint16), s_ref.view(np.uint16))
