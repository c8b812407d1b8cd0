"""kvq_attention_decode_static (the allocation-free entry point, its key-split
scratch in a static device array) against kvq_attention_decode with a
caller-provided workspace: identical outputs on two calls in a row with
different inputs, and a refusal when the shapes need more scratch than the
static array holds.  Collected last so its static scratch outlives every
other test's use of the library."""
import math

import numpy as np
import pytest
import torch

from kv_cache_quantization_02_b200 import kvq, workloads

pytestmark = pytest.mark.gpu


def _inputs(B, Hq, Hkv, T, D, G, seed):
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    kp = torch.randint(0, 256, (B, Hkv, T, D // 2), dtype=torch.uint8, device=dev, generator=gen)
    vp = torch.randint(0, 256, (B, Hkv, T, D // 2), dtype=torch.uint8, device=dev, generator=gen)
    ks = (torch.rand((B, Hkv, T, D // G), device=dev, generator=gen) * 0.4 + 0.02).half()
    vs = (torch.rand((B, Hkv, T, D // G), device=dev, generator=gen) * 0.4 + 0.02).half()
    q = torch.randn((B, Hq, D), device=dev, generator=gen).half()
    lens = torch.randint(1, T + 1, (B,), dtype=torch.int32, device=dev, generator=gen)
    lk, sk = workloads.params(D, seed)
    lv, sv = workloads.params(D, seed + 1)
    t = lambda a: torch.from_numpy(a).to(dev)
    return q, kp, ks, vp, vs, lens, t(lk), t(sk), t(lv), t(sv)


def _static(args, B, Hq, Hkv, T, D, G, scale, out):
    q, kp, ks, vp, vs, lens, lk, sk, lv, sv = args
    return kvq.kvq_attention_decode_static(
        q.data_ptr(), kp.data_ptr(), ks.data_ptr(), vp.data_ptr(), vs.data_ptr(), lens.data_ptr(),
        lk.data_ptr(), sk.data_ptr(), lv.data_ptr(), sv.data_ptr(), B, Hq, Hkv, T, D, G, scale,
        out.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("B,Hq,Hkv,T,D,G", [(1, 8, 2, 4096, 128, 32), (3, 4, 1, 2048, 64, 64)])
def test_static_matches_workspace_entry_twice(B, Hq, Hkv, T, D, G):
    need = kvq.kvq_attention_workspace_bytes(B, Hq, Hkv, T, D, G)
    assert 0 < need <= 8 << 20                   # the shapes do split
    scale = 1.0 / math.sqrt(D)
    for seed in (1, 2):                          # two calls in a row, different inputs
        args = _inputs(B, Hq, Hkv, T, D, G, seed)
        ref = kvq.attention_decode(*args, G, scale, workspace=True)
        out = torch.empty_like(ref)
        assert _static(args, B, Hq, Hkv, T, D, G, scale, out) == kvq.KVQ_OK
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_static_rejects_oversize():
    # 1183 (sequence, KV head) pairs x 2 key splits x 8 heads x 132 floats > 8 MiB
    B, Hq, Hkv, T, D, G = 1183, 8, 1, 512, 128, 32
    need = kvq.kvq_attention_workspace_bytes(B, Hq, Hkv, T, D, G)
    if need <= 8 << 20:
        pytest.skip(f"this device splits these shapes into {need} bytes")
    args = _inputs(B, Hq, Hkv, T, D, G, 3)
    out = torch.zeros((B, Hq, D), dtype=torch.float16, device="cuda")
    assert _static(args, B, Hq, Hkv, T, D, G, 0.1, out) == kvq.KVQ_ERR_COUNT
    torch.cuda.synchronize()
    assert int(out.abs().max()) == 0              # nothing was launched
