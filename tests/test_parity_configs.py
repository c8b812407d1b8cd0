"""Full-size parity on the workloads shaped like the pages' caches, in the
launch configuration the benchmark times (same entry points, same grids).

Inputs are drawn on the device.  The oracle checks sampled rows one by one
(the head, the tail and a seeded random set, 65,536 rows per tensor); the
whole tensor is checked on the device for properties that hold at any size:
every code in [-8, 7], every group with a normal fp16 scale reaching |q| = 7,
and dequantised values finite where the input was.
"""
import numpy as np
import pytest

import oracle
from kv_cache_quantization_02_b200 import workloads
from parity_util import check_dequant, check_quant

pytestmark = pytest.mark.gpu

CASES = [("qwen2.5-1.5b", 32), ("gemma-3-1b", 32), ("gemma-3-1b", 64),
         ("qwen3-8b-prefill", 32), ("decode-append", 32), ("decode-cache", 32)]
SAMPLE = 65_536


def _sample_rows(n, seed):
    rng = np.random.default_rng(seed)
    k = min(n, SAMPLE)
    if n <= SAMPLE:
        return np.arange(n)
    head = np.arange(4096)
    tail = np.arange(n - 4096, n)
    rest = rng.choice(np.arange(4096, n - 4096), size=k - 8192, replace=False)
    return np.unique(np.concatenate([head, tail, rest]))


def _device_invariants(torch, packed, scales, G, chunk=1 << 20):
    """Codes in range and max|q| = 7 in every normal-scale group, whole tensor."""
    n, half = packed.shape
    D = half * 2
    for r0 in range(0, n, chunk):
        p = packed[r0:r0 + chunk].to(torch.int16)
        lo = ((p & 0xF) ^ 8) - 8
        hi = ((p >> 4) ^ 8) - 8
        q = torch.stack([lo, hi], dim=-1).reshape(p.shape[0], D)
        assert int(q.min()) >= -8 and int(q.max()) <= 7
        qm = q.abs().reshape(p.shape[0], D // G, G).amax(dim=2)
        sc = scales[r0:r0 + chunk].float()
        normal = sc >= 2.0 ** -14
        assert bool((qm[normal] == 7).all()), "a normal-scale group lacks |q| = 7"
        zero = sc == 0
        assert bool((qm[zero] == 0).all())


@pytest.mark.parametrize("name,G", CASES, ids=[f"{c}-g{g}" for c, g in CASES])
def test_full_size(name, G):
    import torch
    from kv_cache_quantization_02_b200 import kvq
    o = oracle.get()
    w = workloads.WORKLOADS[name]
    dev = torch.device("cuda")
    n, D = w.n_vec, w.D
    lam, s = workloads.params(D, w.seed)
    lam_t, s_t = torch.from_numpy(lam).to(dev), torch.from_numpy(s).to(dev)
    x = workloads.device_rows(w, n, dev)
    packed, scales = kvq.quantize(x, lam_t, s_t, G)
    torch.cuda.synchronize()
    rows = _sample_rows(n, w.seed)
    idx = torch.from_numpy(rows).to(dev)
    x16 = x.index_select(0, idx).cpu().numpy()
    pk = packed.index_select(0, idx).cpu().numpy()
    sc = scales.index_select(0, idx).cpu().numpy()
    assert check_quant(o, x16, lam, s, G, pk, sc, name) == 0
    _device_invariants(torch, packed, scales, G)
    out = kvq.dequantize(packed, scales, lam_t, s_t, G, out=x)   # x is no longer needed
    torch.cuda.synchronize()
    assert check_dequant(o, pk, sc, lam, s, G, out.index_select(0, idx).cpu().numpy(), name) == 0
    assert bool(torch.isfinite(out).all())
    del x, packed, scales, out
    torch.cuda.empty_cache()
