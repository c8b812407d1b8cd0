"""Fused decode attention over the int4 cache (kvq_attention_decode) against
the oracle's double-precision definition.

Tolerance.  The kernel computes the same attention in fp32 with tensor-core
products: the rotated query is split into fp16 hi + lo parts (relative error
~2^-22), codes are exact, the scores and the weighted value sums accumulate in
fp32, p * S_V is split hi + lo again, and the result is rounded once to fp16
(half an fp16 ulp, 2^-11 relative).  The value product runs on biased codes
n = q + 8 in [0, 15] and removes the bias 8 sum p S_V by a second product per
16 keys, so the fp32 rounding of the accumulated sums is not relative to the
result: each of the ~L/8 tensor-core accumulations of a value entry (codes
and bias, 16 keys each) rounds an accumulator of at most 15 sum_t p_t S_V,t 2^-24,
which after the division by l = sum_t p_t is at most 2 u 15 (L/8 + 8) max S_V
in the rotated domain (u = 2^-24, eight more for the online rescalings), and
the inverse rotation (orthonormal) and 1/lambda_V carry that into each output
as at most sqrt(D) / min lambda_V times it.  Every output must lie within
    |out - o| <= 2^-10 |o| + 1e-4 max|o_row| + 2 u 15 (L/8 + 8) max S_V sqrt(D) / min lambda_V,
one fp16 ulp, a small absolute floor for near-zero outputs, and that
accumulation bound (L the sequence's length, max S_V over its attended rows).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_02_b200 import kvq, workloads

pytestmark = pytest.mark.gpu


def _case(B, Hq, Hkv, T, D, G, seed, lens=None, dist="uniform"):
    """Random caches: codes uniform over all nibbles, scales in a realistic
    range; or, with dist="quantized", rows that are the codes of real
    quantize calls on Gaussian K/V with outliers."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    lk, sk = workloads.params(D, seed)
    lv, sv = workloads.params(D, seed + 1)
    if dist == "uniform":
        kp = rng.integers(0, 256, (B, Hkv, T, D // 2), dtype=np.uint8)
        vp = rng.integers(0, 256, (B, Hkv, T, D // 2), dtype=np.uint8)
        ks = rng.uniform(0.02, 0.5, (B, Hkv, T, D // G)).astype(np.float16)
        vs = rng.uniform(0.02, 0.5, (B, Hkv, T, D // G)).astype(np.float16)
    else:
        o = oracle.get()
        x = rng.standard_normal((2, B * Hkv * T, D))
        x[:, :, rng.permutation(D)[:4]] *= 20.0
        x = x.astype(np.float16)
        kp, ks = o.quantize(x[0], lk, sk, G)
        vp, vs = o.quantize(x[1], lv, sv, G)
        kp = kp.reshape(B, Hkv, T, D // 2)
        vp = vp.reshape(B, Hkv, T, D // 2)
        ks = ks.reshape(B, Hkv, T, D // G)
        vs = vs.reshape(B, Hkv, T, D // G)
    if lens is None:
        lens = rng.integers(0, T + 1, B)
    lens = np.asarray(lens, dtype=np.int32)
    return dict(q=q, kp=kp, ks=ks, vp=vp, vs=vs, lens=lens, lk=lk, sk=sk, lv=lv, sv=sv, G=G)


def _gpu(c, scale, workspace=True):
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    out = kvq.attention_decode(t(c["q"]), t(c["kp"]), t(c["ks"]), t(c["vp"]), t(c["vs"]),
                               t(c["lens"]), t(c["lk"]), t(c["sk"]), t(c["lv"]), t(c["sv"]),
                               c["G"], scale, workspace=workspace)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _oracle(c, scale):
    return oracle.get().attention_decode(c["q"], c["kp"], c["ks"], c["vp"], c["vs"], c["lens"],
                                         c["lk"], c["sk"], c["lv"], c["sv"], c["G"], scale)


def _accum_floor(c):
    """The value product's accumulation bound per sequence, [B, 1, 1]."""
    vs = np.asarray(c["vs"], dtype=np.float16).astype(np.float64)
    lens = np.asarray(c["lens"])
    D = np.asarray(c["q"]).shape[-1]
    lam_min = float(np.abs(np.asarray(c["lv"], dtype=np.float64)).min())
    out = np.zeros((len(lens), 1, 1))
    for b, L in enumerate(lens):
        if L > 0:
            smax = float(vs[b, :, :L].max())
            out[b] = 2.0 * 2.0 ** -24 * 15.0 * (L / 8.0 + 8.0) * smax * math.sqrt(D) / lam_min
    return out


def _check(got, ref, c=None):
    row = np.abs(ref).max(axis=-1, keepdims=True)
    bound = 2.0 ** -10 * np.abs(ref) + 1e-4 * row
    if c is not None:
        bound = bound + _accum_floor(c)
    err = np.abs(got - ref)
    worst = float((err - bound).max())
    assert np.all(err <= bound), f"max excess {worst}, max err {err.max()}"
    return float(err.max())


CASES = [
    # B, Hq, Hkv, T, D, G, lens
    (2, 8, 2, 64, 128, 32, [64, 37]),
    (3, 4, 4, 160, 64, 32, [0, 1, 160]),
    (2, 16, 2, 96, 128, 64, [17, 96]),
    (1, 6, 1, 48, 128, 128, [48]),
    (4, 8, 8, 16, 64, 64, [15, 16, 1, 0]),
    (2, 32, 8, 208, 128, 32, [65, 208]),
    (1, 2, 2, 1024, 128, 32, [1000]),          # few pairs: the key axis splits
    (1, 8, 1, 4096, 64, 32, [4095]),
    (2, 8, 2, 96, 128, 16, [96, 50]),           # groups of 16 (the paper's)
    (1, 4, 4, 64, 64, 16, [64]),
    (2, 8, 2, 64, 256, 32, [64, 23]),           # D = 256 (Gemma-3-1B)
    (1, 4, 1, 128, 256, 16, [128]),
    (2, 16, 2, 48, 256, 64, [48, 31]),
    (1, 8, 1, 64, 256, 128, [60]),
    (1, 8, 1, 256, 256, 16, [256]),             # D = 256, 8 heads per KV head: two head tiles per warp pair
    (2, 16, 2, 512, 256, 32, [512, 300]),       # many blocks per pair, a ragged last block
    (1, 4, 1, 4096, 256, 32, [4000]),           # one pair: the key axis splits
]


@pytest.mark.parametrize("B,Hq,Hkv,T,D,G,lens", CASES)
def test_attention_matches_oracle(B, Hq, Hkv, T, D, G, lens):
    c = _case(B, Hq, Hkv, T, D, G, seed=B * 7 + T, lens=lens)
    scale = 1.0 / math.sqrt(D)
    _check(_gpu(c, scale), _oracle(c, scale), c)


@pytest.mark.parametrize("dist", ["quantized"])
def test_attention_on_quantized_rows(dist):
    """Rows that are real quantize outputs (peaked softmax from outliers)."""
    c = _case(2, 8, 2, 256, 128, 32, seed=5, lens=[256, 131], dist=dist)
    for scale in (1.0 / math.sqrt(128), 0.3):
        _check(_gpu(c, scale), _oracle(c, scale), c)


def test_split_and_unsplit_agree():
    """With and without workspace (split key axis vs one pass): both match
    the oracle; they differ only in fp32 summation order."""
    c = _case(1, 4, 2, 2048, 128, 32, seed=11, lens=[1999])
    assert kvq.kvq_attention_workspace_bytes(1, 4, 2, 2048, 128, 32) > 0
    ref = _oracle(c, 0.1)
    a = _gpu(c, 0.1, workspace=True)
    b = _gpu(c, 0.1, workspace=False)
    _check(a, ref, c)
    _check(b, ref, c)


def test_extreme_scales_and_zero_length():
    c = _case(3, 4, 1, 64, 128, 32, seed=13, lens=[64, 0, 9])
    for scale in (0.0, 1e-3, 5.0):
        got = _gpu(c, scale)
        _check(got, _oracle(c, scale), c)
    assert np.all(got[1] == 0.0)


def test_bad_length_is_clamped_and_flagged():
    kvq.kvq_fault_status(True)
    c = _case(2, 4, 2, 32, 128, 32, seed=17, lens=[40, 32])
    got = _gpu(c, 0.2)
    assert kvq.kvq_fault_status(True) & 8
    c["lens"] = np.array([32, 32], dtype=np.int32)
    _check(got, _oracle(c, 0.2), c)
    assert kvq.kvq_fault_status(False) == 0


def test_decode_config_sampled():
    """The bench's decode shape (a 64-sequence batch x 36 layers folded into
    B, 8 KV heads, 32 query heads, 4096 positions) on a slice of sequences,
    sampled rows checked against the oracle one (sequence, KV head) at a time."""
    B, Hq, Hkv, T, D, G = 48, 32, 8, 4096, 128, 32
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(4)
    kp = torch.randint(0, 256, (B, Hkv, T, D // 2), dtype=torch.uint8, device=dev, generator=gen)
    vp = torch.randint(0, 256, (B, Hkv, T, D // 2), dtype=torch.uint8, device=dev, generator=gen)
    ks = (torch.rand((B, Hkv, T, D // G), device=dev, generator=gen) * 0.4 + 0.02).half()
    vs = (torch.rand((B, Hkv, T, D // G), device=dev, generator=gen) * 0.4 + 0.02).half()
    q = torch.randn((B, Hq, D), device=dev, generator=gen).half()
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    lens[::5] = 1234
    lk, sk = workloads.params(D, 4)
    lv, sv = workloads.params(D, 5)
    t = lambda a: torch.from_numpy(a).to(dev)
    out = kvq.attention_decode(q, kp, ks, vp, vs, lens, t(lk), t(sk), t(lv), t(sv), G,
                               1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    R = Hq // Hkv
    for b, kvh in ((0, 0), (5, 7), (47, 3)):
        L = int(lens[b])
        sub = dict(q=q[b:b + 1, kvh * R:(kvh + 1) * R].cpu().numpy(),
                   kp=kp[b:b + 1, kvh:kvh + 1].cpu().numpy(), ks=ks[b:b + 1, kvh:kvh + 1].cpu().numpy(),
                   vp=vp[b:b + 1, kvh:kvh + 1].cpu().numpy(), vs=vs[b:b + 1, kvh:kvh + 1].cpu().numpy(),
                   lens=np.array([L], dtype=np.int32), lk=lk, sk=sk, lv=lv, sv=sv, G=G)
        ref = _oracle(sub, 1.0 / math.sqrt(D))[0]
        got = out[b, kvh * R:(kvh + 1) * R].cpu().numpy().astype(np.float64)
        _check(got[None], ref[None], sub)


def test_decode_config_sampled_paper_format():
    """The paper's own cache format (SRFT, lambda after, groups of 16) at the
    bench's decode shape on a slice of sequences: the cache written on the
    GPU by kvq_quantize_ex from device-drawn rows, sampled (sequence, KV head)
    pairs checked against the oracle on the same codes."""
    B, Hq, Hkv, T, D, G = 12, 32, 8, 4096, 128, 16
    dev = torch.device("cuda")
    c = workloads.WORKLOADS["decode-cache"]
    rows = 2 * B * Hkv * T
    lam, sgn = workloads.params(D, 21)
    lt, st = torch.from_numpy(lam).to(dev), torch.from_numpy(sgn).to(dev)
    x = workloads.device_rows(c, rows, dev, seed_offset=3)
    codes, scales = kvq.quantize_ex(x, lt, st, G, lambda_after=True, srft=True)
    del x
    pk = codes.view(2, B, Hkv, T, D // 2)
    sc = scales.view(2, B, Hkv, T, D // G)
    gen = torch.Generator(device=dev)
    gen.manual_seed(6)
    q = torch.randn((B, Hq, D), device=dev, generator=gen).half()
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    lens[::3] = 2000
    scale = 1.0 / math.sqrt(D)
    out = kvq.attention_decode(q, pk[0], sc[0], pk[1], sc[1], lens, lt, st, lt, st, G, scale,
                               lambda_after=True, srft=True)
    torch.cuda.synchronize()
    R = Hq // Hkv
    for b, kvh in ((0, 0), (5, 7), (11, 3)):
        L = int(lens[b])
        sub = dict(q=q[b:b + 1, kvh * R:(kvh + 1) * R].cpu().numpy(),
                   kp=pk[0, b:b + 1, kvh:kvh + 1].cpu().numpy(), ks=sc[0, b:b + 1, kvh:kvh + 1].cpu().numpy(),
                   vp=pk[1, b:b + 1, kvh:kvh + 1].cpu().numpy(), vs=sc[1, b:b + 1, kvh:kvh + 1].cpu().numpy(),
                   lens=np.array([L], dtype=np.int32), lk=lam, sk=sgn, lv=lam, sv=sgn, G=G)
        ref = oracle.get().attention_decode(sub["q"], sub["kp"], sub["ks"], sub["vp"], sub["vs"],
                                            sub["lens"], lam, sgn, lam, sgn, G, scale,
                                            lambda_after=True, srft=True)[0]
        got = out[b, kvh * R:(kvh + 1) * R].cpu().numpy().astype(np.float64)
        _check(got[None], ref[None], sub)


# ---- caches of the codec variants' formats -----------------------------------

def _case_fmt(B, Hq, Hkv, T, D, G, seed, after, srft, lens=None):
    """K and V rows that are real kvq_quantize_ex codes (int4) of Gaussian rows
    with outlier channels, in the given format."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    lk, sk = workloads.params(D, seed)
    lv, sv = workloads.params(D, seed + 1)
    o = oracle.get()
    x = rng.standard_normal((2, B * Hkv * T, D))
    x[:, :, rng.permutation(D)[:4]] *= 20.0
    x = x.astype(np.float16)
    kp, ks = o.quantize_ex(x[0], lk, sk, G, lambda_after=after, srft=srft)
    vp, vs = o.quantize_ex(x[1], lv, sv, G, lambda_after=after, srft=srft)
    if lens is None:
        lens = rng.integers(0, T + 1, B)
    return dict(q=q, kp=kp.reshape(B, Hkv, T, D // 2), ks=ks.reshape(B, Hkv, T, D // G),
                vp=vp.reshape(B, Hkv, T, D // 2), vs=vs.reshape(B, Hkv, T, D // G),
                lens=np.asarray(lens, dtype=np.int32), lk=lk, sk=sk, lv=lv, sv=sv, G=G)


FMT_CASES = [
    # B, Hq, Hkv, T, D, G, lens
    (3, 8, 2, 256, 128, 32, None),
    (2, 4, 4, 96, 64, 32, [96, 17]),
    (4, 32, 8, 80, 128, 64, [0, 1, 80, 33]),
    (1, 2, 1, 400, 128, 128, [400]),
    (2, 4, 2, 64, 128, 16, [64, 21]),           # the paper's groups of 16
    (2, 8, 2, 96, 256, 32, [96, 40]),           # D = 256
    (1, 8, 1, 64, 256, 16, [64]),
]


@pytest.mark.parametrize("after,srft", [(True, False), (False, True), (True, True)])
@pytest.mark.parametrize("case", FMT_CASES)
def test_attention_formats_match_oracle(case, after, srft):
    """The paper's cache format (SRFT, lambda after) and the other variants:
    the query rotated to the cache's domain once, the output rotated back once
    per head, against the oracle's double-precision definition on the same
    rows; with and without the key-axis split."""
    B, Hq, Hkv, T, D, G, lens = case
    c = _case_fmt(B, Hq, Hkv, T, D, G, seed=B * T + D + int(after) + 2 * int(srft),
                  after=after, srft=srft, lens=lens)
    ref = oracle.get().attention_decode(c["q"], c["kp"], c["ks"], c["vp"], c["vs"], c["lens"],
                                        c["lk"], c["sk"], c["lv"], c["sv"], G, 0.0883,
                                        lambda_after=after, srft=srft)
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    for ws in (True, False):
        out = kvq.attention_decode(t(c["q"]), t(c["kp"]), t(c["ks"]), t(c["vp"]), t(c["vs"]),
                                   t(c["lens"]), t(c["lk"]), t(c["sk"]), t(c["lv"]), t(c["sv"]),
                                   G, 0.0883, workspace=ws, lambda_after=after, srft=srft)
        torch.cuda.synchronize()
        _check(out.cpu().numpy().astype(np.float64), ref, c)


def test_attention_formats_reject_bad_flags():
    c = _case(1, 2, 1, 16, 128, 32, seed=3)
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    args = [t(c[k]).data_ptr() for k in ("q", "kp", "ks", "vp", "vs", "lens", "lk", "sk", "lv", "sv")]
    out = torch.empty((1, 2, 128), dtype=torch.float16, device=dev)
    assert kvq.kvq_attention_decode_ex(*args, 1, 2, 1, 16, 128, 32, 4, 0.1, out.data_ptr()) == kvq.KVQ_ERR_GROUP


def test_paper_format_inside_cuda_graph():
    """The SRFT rotations run inside the kernels (no host-side table), so the
    paper-format call can be captured in a CUDA graph: its replay gives the
    eager call's bytes, with and without the key-axis split."""
    B, Hq, Hkv, T, D, G = 2, 8, 2, 512, 128, 16
    c = _case_fmt(B, Hq, Hkv, T, D, G, seed=77, after=True, srft=True, lens=[512, 301])
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    args = [t(c[k]) for k in ("q", "kp", "ks", "vp", "vs", "lens", "lk", "sk", "lv", "sv")]
    need = kvq.kvq_attention_workspace_bytes(B, Hq, Hkv, T, D, G)
    for ws in (torch.empty(max(need, 16), dtype=torch.uint8, device=dev), False):
        eager = kvq.attention_decode(*args, G, 0.0883, workspace=ws, lambda_after=True, srft=True)
        out = torch.empty_like(eager)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s), torch.cuda.graph(graph, stream=s):
            kvq.attention_decode(*args, G, 0.0883, out=out, workspace=ws, lambda_after=True,
                                 srft=True, stream=s)
        torch.cuda.current_stream().wait_stream(s)
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
        del graph
