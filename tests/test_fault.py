"""Failure detection of the bounded shared-memory-barrier waits, on the GPU.

The kernels wait for their bulk copies with bounded polls; a block that gives
up sets the device fault word instead of hanging.  The self-test kernel waits
on a barrier that nothing completes, with a short poll limit, so the give-up
path runs for real: the word must report it, clear, and leave the context
usable (the next quantize/dequantize still matches the oracle).
"""
import numpy as np
import pytest

import oracle
from kv_cache_quantization_02_b200 import workloads
from parity_util import check_dequant, check_quant

pytestmark = pytest.mark.gpu


def _roundtrip(torch, kvq, o):
    D, G, n = 128, 32, 777
    lam, s = workloads.params(D, seed=21)
    rng = np.random.default_rng(21)
    x16 = (rng.standard_normal((n, D)) * 3).astype(np.float16)
    dev = torch.device("cuda")
    lam_t, s_t = torch.from_numpy(lam).to(dev), torch.from_numpy(s).to(dev)
    packed, scales = kvq.quantize(torch.from_numpy(x16).to(dev), lam_t, s_t, G)
    out = kvq.dequantize(packed, scales, lam_t, s_t, G)
    torch.cuda.synchronize()
    pk, sc = packed.cpu().numpy(), scales.cpu().numpy()
    assert check_quant(o, x16, lam, s, G, pk, sc, "after") == 0
    assert check_dequant(o, pk, sc, lam, s, G, out.cpu().numpy(), "after") == 0


def test_wait_timeout_is_reported_and_recoverable():
    import torch
    from kv_cache_quantization_02_b200 import kvq
    o = oracle.get()
    assert kvq.kvq_fault_status(clear=True) in (0, 1, 2, 3)
    _roundtrip(torch, kvq, o)
    assert kvq.kvq_fault_status() == 0, "a real kernel gave up a bounded wait"
    assert kvq.kvq_selftest_wait_timeout(2000) == kvq.KVQ_OK
    torch.cuda.synchronize()
    assert kvq.kvq_fault_status() & 2, "the give-up path did not set the fault word"
    assert kvq.kvq_fault_status(clear=True) & 2
    assert kvq.kvq_fault_status() == 0
    _roundtrip(torch, kvq, o)
    assert kvq.kvq_fault_status() == 0
