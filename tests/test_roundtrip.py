"""kvq_roundtrip (quantize then dequantize in one kernel) against the oracle's
quantize -> dequantize, bit for bit, with and without the codes written."""
import numpy as np
import pytest

import oracle
from kv_cache_quantization_02_b200 import workloads
from parity_util import check_dequant, check_quant

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D,G", [(64, 16), (64, 64), (128, 32), (128, 16), (128, 128),
                                 (256, 32), (256, 64), (256, 256)])
@pytest.mark.parametrize("n", [1, 129, 5003])
def test_roundtrip_matches_oracle(D, G, n):
    import torch
    from kv_cache_quantization_02_b200 import kvq
    o = oracle.get()
    dev = torch.device("cuda")
    lam, s = workloads.params(D, seed=D + G)
    rng = np.random.default_rng(n + D)
    x = rng.standard_normal((n, D))
    x[:, rng.permutation(D)[:4]] *= 25
    x16 = x.astype(np.float16)
    xt = torch.from_numpy(x16).to(dev)
    lam_t, s_t = torch.from_numpy(lam).to(dev), torch.from_numpy(s).to(dev)
    out = kvq.roundtrip(xt, lam_t, s_t, G)
    packed = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, D // G), dtype=torch.float16, device=dev)
    out2 = kvq.roundtrip(xt, lam_t, s_t, G, packed=packed, scales=scales)
    torch.cuda.synchronize()
    p_ref, s_ref = o.quantize(x16, lam, s, G)
    assert check_quant(o, x16, lam, s, G, packed.cpu().numpy(), scales.cpu().numpy(), "rt") == 0
    assert check_dequant(o, p_ref, s_ref, lam, s, G, out.cpu().numpy(), "rt") == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint16), out2.cpu().numpy().view(np.uint16))


def test_roundtrip_adversarial():
    import torch
    from kv_cache_quantization_02_b200 import kvq
    o = oracle.get()
    dev = torch.device("cuda")
    for D, G in ((128, 32), (256, 64)):
        x16 = workloads.adversarial_rows(D)
        lam, s = workloads.params(D, seed=4)
        out = kvq.roundtrip(torch.from_numpy(x16).to(dev), torch.from_numpy(lam).to(dev),
                            torch.from_numpy(s).to(dev), G)
        torch.cuda.synchronize()
        p_ref, s_ref = o.quantize(x16, lam, s, G)
        assert check_dequant(o, p_ref, s_ref, lam, s, G, out.cpu().numpy(), "rt-adv") == 0


@pytest.mark.parametrize("D,G", [(128, 32), (256, 64)])
def test_roundtrip_many_tiles(D, G):
    """A ragged batch with several warp tiles per warp (the tile-claim loop),
    codes written: every row against the oracle."""
    import torch
    from kv_cache_quantization_02_b200 import kvq
    o = oracle.get()
    dev = torch.device("cuda")
    n = 300_007
    lam, s = workloads.params(D, seed=5)
    x16 = workloads.host_rows(workloads.WORKLOADS["qwen3-8b-prefill" if D == 128 else "gemma-3-1b"],
                              n, seed_offset=D)
    xt = torch.from_numpy(x16).to(dev)
    packed = torch.empty((n, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, D // G), dtype=torch.float16, device=dev)
    out = kvq.roundtrip(xt, torch.from_numpy(lam).to(dev), torch.from_numpy(s).to(dev), G,
                        packed=packed, scales=scales)
    torch.cuda.synchronize()
    p_ref, s_ref = o.quantize(x16, lam, s, G)
    assert np.array_equal(packed.cpu().numpy(), p_ref)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), s_ref.view(np.uint16))
    assert check_dequant(o, p_ref, s_ref, lam, s, G, out.cpu().numpy(), "rt-many") == 0
