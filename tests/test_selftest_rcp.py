"""The quantisers' reciprocal of a group scale, r = 1/S (an approximate
reciprocal refined by one Newton step in the kernels), against the IEEE fp32
quotient 1/S, bit for bit, at every positive finite fp16 value S: every scale
the codec can store.  The library's self-test entry point evaluates the same
device function the kernels call."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_rcp_of_every_fp16_scale_is_ieee():
    import torch
    from kv_cache_quantization_02_b200 import kvq
    n = 0x7BFF
    out = torch.full((n,), float("nan"), dtype=torch.float32, device="cuda")
    assert kvq.kvq_selftest_rcp_f16(out.data_ptr(), 0) == kvq.KVQ_OK
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    s = np.arange(1, n + 1, dtype=np.uint16).view(np.float16).astype(np.float32)
    want = np.float32(1.0) / s
    bad = np.flatnonzero(got.view(np.uint32) != want.view(np.uint32))
    assert bad.size == 0, (f"{bad.size} scales differ, first S bits 0x{bad[0] + 1:04x}: "
                           f"{got[bad[0]]!r} != {want[bad[0]]!r}")


def test_rcp_selftest_checks_its_arguments():
    import torch
    from kv_cache_quantization_02_b200 import kvq
    assert kvq.kvq_selftest_rcp_f16(0, 0) == kvq.KVQ_ERR_NULL
    buf = torch.empty(0x7C00, dtype=torch.float32, device="cuda")
    assert kvq.kvq_selftest_rcp_f16(buf.data_ptr() + 2, 0) == kvq.KVQ_ERR_ALIGN
