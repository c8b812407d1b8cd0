"""GPU kernels against the CPU oracle, element by element, through the C ABI.

Sizes: small enough for the oracle to finish in seconds, but spanning many
warps and blocks, ragged tails (n not a multiple of the vectors per warp or
per block) and, for the largest case, several passes of the grid-stride loop.
"""
import numpy as np
import pytest

import oracle
from kv_cache_quantization_02_b200 import workloads
from parity_util import check_dequant, check_quant

pytestmark = pytest.mark.gpu

SHAPES = [(64, 16), (64, 32), (64, 64),
          (128, 16), (128, 32), (128, 64), (128, 128),
          (256, 16), (256, 32), (256, 64), (256, 128), (256, 256)]


@pytest.fixture(scope="module")
def env():
    import torch
    from kv_cache_quantization_02_b200 import kvq
    assert torch.cuda.is_available()
    return torch, kvq, oracle.get()


def _rows(seed, n, D, outliers=4, gain=20.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, D))
    x[:, rng.permutation(D)[:outliers]] *= gain
    return x.astype(np.float16)


def _run(torch, kvq, x16, lam, s, G, stream=None):
    dev = torch.device("cuda")
    x = torch.from_numpy(x16).to(dev)
    lam_t = torch.from_numpy(lam).to(dev)
    s_t = torch.from_numpy(s).to(dev)
    packed, scales = kvq.quantize(x, lam_t, s_t, G, stream=stream)
    out = kvq.dequantize(packed, scales, lam_t, s_t, G, stream=stream)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), scales.cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("D,G", SHAPES)
@pytest.mark.parametrize("n", [1, 7, 255, 257, 1031])
def test_random_rows(env, D, G, n):
    torch, kvq, o = env
    lam, s = workloads.params(D, seed=D * 7 + G)
    x16 = _rows(D + G + n, n, D)
    packed, scales, out = _run(torch, kvq, x16, lam, s, G)
    assert check_quant(o, x16, lam, s, G, packed, scales, f"D={D} G={G} n={n}") == 0
    assert check_dequant(o, packed, scales, lam, s, G, out, f"D={D} G={G} n={n}") == 0


@pytest.mark.parametrize("D,G", SHAPES)
def test_adversarial_rows(env, D, G):
    """Zero rows, spikes, constants, exact ties, fp16 extremes, subnormals."""
    torch, kvq, o = env
    x16 = workloads.adversarial_rows(D)
    for lam, s in (workloads.params(D, seed=3),
                   (np.ones(D, np.float32), np.ones(D, np.int8)),
                   (np.full(D, 2.0, np.float32), -np.ones(D, np.int8))):
        packed, scales, out = _run(torch, kvq, x16, lam, s, G)
        assert check_quant(o, x16, lam, s, G, packed, scales, f"adv D={D} G={G}") == 0
        assert check_dequant(o, packed, scales, lam, s, G, out, f"adv D={D} G={G}") == 0


def test_tiny_workload(env):
    """256 vectors, one head, D=128, N(0,1) with 4 outlier channels x20."""
    torch, kvq, o = env
    w = workloads.WORKLOADS["tiny"]
    lam, s = workloads.params(w.D, w.seed)
    x16 = workloads.host_rows(w, w.n_vec)
    packed, scales, out = _run(torch, kvq, x16, lam, s, 32)
    assert check_quant(o, x16, lam, s, 32, packed, scales, "tiny") == 0
    assert check_dequant(o, packed, scales, lam, s, 32, out, "tiny") == 0


@pytest.mark.parametrize("D,G", [(128, 32), (256, 64), (64, 16)])
def test_grid_stride_wraps(env, D, G):
    """More vectors than one pass of the persistent grid covers, ragged tail."""
    torch, kvq, o = env
    n = 200_003
    lam, s = workloads.params(D, seed=11)
    x16 = workloads.host_rows(
        workloads.Workload("t", n, D, (G,), "student_t3", 4, 20.0, (0.1, 10.0), 9, {}), n)
    packed, scales, out = _run(torch, kvq, x16, lam, s, G)
    assert check_quant(o, x16, lam, s, G, packed, scales, "wrap") == 0
    assert check_dequant(o, packed, scales, lam, s, G, out, "wrap") == 0


def test_guard_bands_and_offsets(env):
    """Outputs written exactly in place: canary rows around them stay intact;
    inputs and outputs may start at any row of a larger buffer."""
    torch, kvq, o = env
    D, G, n = 128, 32, 333
    dev = torch.device("cuda")
    lam, s = workloads.params(D, seed=5)
    x16 = _rows(1, n + 3, D)
    x_all = torch.from_numpy(x16).to(dev)
    x = x_all[1:n + 1]
    lam_t, s_t = torch.from_numpy(lam).to(dev), torch.from_numpy(s).to(dev)
    packed_all = torch.full((n + 2, D // 2), 0xAB, dtype=torch.uint8, device=dev)
    scales_all = torch.full((n + 2, D // G), 1234.0, dtype=torch.float16, device=dev)
    out_all = torch.full((n + 2, D), -777.0, dtype=torch.float16, device=dev)
    kvq.quantize(x, lam_t, s_t, G, packed=packed_all[1:n + 1], scales=scales_all[1:n + 1])
    kvq.dequantize(packed_all[1:n + 1], scales_all[1:n + 1], lam_t, s_t, G, out=out_all[1:n + 1])
    torch.cuda.synchronize()
    for t, fill in ((packed_all, 0xAB), (scales_all, 1234.0), (out_all, -777.0)):
        assert bool((t[0] == fill).all()) and bool((t[-1] == fill).all())
    pk = packed_all[1:n + 1].cpu().numpy()
    sc = scales_all[1:n + 1].cpu().numpy()
    assert check_quant(o, x16[1:n + 1], lam, s, G, pk, sc, "offset") == 0
    assert check_dequant(o, pk, sc, lam, s, G, out_all[1:n + 1].cpu().numpy(), "offset") == 0


def test_deterministic_and_stream_independent(env):
    torch, kvq, o = env
    D, G = 256, 32
    lam, s = workloads.params(D, seed=8)
    x16 = _rows(2, 4097, D)
    a = _run(torch, kvq, x16, lam, s, G)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        b = _run(torch, kvq, x16, lam, s, G, stream=st)
    for u, v in zip(a, b):
        assert np.array_equal(np.ascontiguousarray(u).view(np.uint8),
                              np.ascontiguousarray(v).view(np.uint8))


def test_misaligned_input_is_rejected(env):
    torch, kvq, o = env
    D, G, n = 128, 32, 4
    dev = torch.device("cuda")
    flat = torch.zeros(n * D + 64, dtype=torch.float16, device=dev)
    x = flat[4:4 + n * D].view(n, D)            # 8-byte offset: not 16-aligned
    lam = torch.ones(D, dtype=torch.float32, device=dev)
    s = torch.ones(D, dtype=torch.int8, device=dev)
    with pytest.raises(kvq.KvqError) as ei:
        kvq.quantize(x, lam, s, G)
    assert ei.value.status == kvq.KVQ_ERR_ALIGN


def test_zero_vectors(env):
    torch, kvq, o = env
    dev = torch.device("cuda")
    x = torch.empty((0, 128), dtype=torch.float16, device=dev)
    lam = torch.ones(128, dtype=torch.float32, device=dev)
    s = torch.ones(128, dtype=torch.int8, device=dev)
    packed, scales = kvq.quantize(x, lam, s, 32)
    out = kvq.dequantize(packed, scales, lam, s, 32)
    torch.cuda.synchronize()
    assert packed.shape == (0, 64) and out.shape == (0, 128)
