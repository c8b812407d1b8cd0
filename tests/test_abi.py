"""The C-ABI library loads, exports every symbol include/kvq.h declares, and
rejects bad arguments with a status before touching the GPU (no GPU needed:
every call here returns before any CUDA runtime call)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def _declared():
    with open(HEADER) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_02_b200 import kvq
    return kvq


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("kvq_quantize", "kvq_dequantize", "kvq_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(kvq):
    lib = ctypes.CDLL(kvq.LIBRARY)
    for name in _declared():
        assert hasattr(lib, name), f"{name} declared in kvq.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", kvq.LIBRARY],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (kvq_[a-z0-9_]+)\b", out))
    assert exported == set(_declared()), f"exports {exported} != header {_declared()}"


def test_version_and_status_strings(kvq):
    assert kvq.kvq_version() >> 16 == 1
    for st in range(-6, 1):
        s = kvq.kvq_status_string(st)
        assert s.startswith("KVQ_")
    assert "unknown" in kvq.kvq_status_string(-99)
    assert kvq.kvq_last_cuda_error() == 0


# Fake, never-dereferenced device addresses: every case below fails a
# precondition, so the library returns before any CUDA call.
A = 0x7F0000000000          # 256-byte aligned


@pytest.mark.parametrize("D,G,n,want", [
    (96, 32, 10, -3), (32, 32, 10, -3), (512, 32, 10, -3),
    (128, 8, 10, -4), (128, 24, 10, -4), (128, 256, 10, -4), (64, 128, 10, -4),
    (128, 32, -1, -5), (128, 32, 1 << 31, -5), (64, 16, (1 << 40), -5),
])
def test_shape_errors(kvq, D, G, n, want):
    assert kvq.kvq_quantize(A, A, A, n, D, G, A, A, 0) == want
    assert kvq.kvq_dequantize(A, A, A, A, n, D, G, A, 0) == want


def test_zero_vectors_is_a_noop(kvq):
    assert kvq.kvq_quantize(0, 0, 0, 0, 128, 32, 0, 0, 0) == 0
    assert kvq.kvq_dequantize(0, 0, 0, 0, 0, 128, 32, 0, 0) == 0


@pytest.mark.parametrize("which", range(5))
def test_null_pointers(kvq, which):
    q = [A, A, A, A, A]
    q[which] = 0
    x, lam, s, packed, scales = q
    assert kvq.kvq_quantize(x, lam, s, 4, 128, 32, packed, scales, 0) == -1
    packed, scales, lam, s, out = q
    assert kvq.kvq_dequantize(packed, scales, lam, s, 4, 128, 32, out, 0) == -1


def test_alignment(kvq):
    assert kvq.kvq_quantize(A + 8, A, A, 4, 128, 32, A, A, 0) == -2       # x needs 16
    assert kvq.kvq_quantize(A, A + 2, A, 4, 128, 32, A, A, 0) == -2       # lambda needs 4
    assert kvq.kvq_quantize(A, A, A, 4, 128, 32, A + 8, A, 0) == -2       # packed needs 16
    assert kvq.kvq_quantize(A, A, A, 4, 128, 32, A, A + 1, 0) == -2       # scales need 2
    assert kvq.kvq_dequantize(A + 8, A, A, A, 4, 128, 32, A, 0) == -2
    assert kvq.kvq_dequantize(A, A + 1, A, A, 4, 128, 32, A, 0) == -2
    assert kvq.kvq_dequantize(A, A, A + 1, A, 4, 128, 32, A, 0) == -2
    assert kvq.kvq_dequantize(A, A, A, A, 4, 128, 32, A + 8, 0) == -2     # x_out needs 16


def test_binding_fails_loudly_without_the_library(tmp_path):
    """The product path has no fallback: a missing library is an ImportError."""
    import importlib.util
    import shutil
    pkg = tmp_path / "kv_cache_quantization_02_b200"
    pkg.mkdir()
    src = os.path.join(ROOT, "kv_cache_quantization_02_b200", "kvq.py")
    shutil.copy(src, pkg / "kvq.py")
    spec = importlib.util.spec_from_file_location("kvq_nolib", pkg / "kvq.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_quantize_rows_errors(kvq):
    assert kvq.kvq_quantize_rows(A, A, A, 4, 128, 32, 0, 100, A, A, 0) == -1     # row_idx NULL
    assert kvq.kvq_quantize_rows(A, A, A, 4, 128, 32, A + 4, 100, A, A, 0) == -2  # row_idx needs 8
    assert kvq.kvq_quantize_rows(A, A, A, 4, 128, 32, A, -1, A, A, 0) == -5       # cache_rows < 0
    assert kvq.kvq_quantize_rows(A, A, A, 4, 96, 32, A, 100, A, A, 0) == -3
    assert kvq.kvq_quantize_rows(0, 0, 0, 0, 128, 32, 0, 0, 0, 0, 0) == 0


def test_roundtrip_errors(kvq):
    assert kvq.kvq_roundtrip(A, A, A, 4, 128, 32, 0, 0, 0, 0) == -1       # x_hat NULL
    assert kvq.kvq_roundtrip(A, A, A, 4, 128, 32, A, A, 0, 0) == -1       # packed without scales
    assert kvq.kvq_roundtrip(A, A, A, 4, 128, 32, A + 8, 0, 0, 0) == -2   # x_hat needs 16
    assert kvq.kvq_roundtrip(A, A, A, 4, 128, 8, A, 0, 0, 0) == -4
    assert kvq.kvq_roundtrip(0, 0, 0, 0, 128, 32, 0, 0, 0, 0) == 0


def test_attention_errors(kvq):
    A_ = A
    args = lambda **kw: dict(dict(B=1, Hq=32, Hkv=8, T=4096, D=128, G=32), **kw)
    def call(q=A_, B=1, Hq=32, Hkv=8, T=4096, D=128, G=32, out=A_, lens=A_):
        return kvq.kvq_attention_decode(q, A_, A_, A_, A_, lens, A_, A_, A_, A_,
                                        B, Hq, Hkv, T, D, G, 0.1, out)
    assert call(D=512) == -3 and call(D=96) == -3 and call(D=32) == -3
    assert call(G=8) == -4 and call(G=256) == -4 and call(D=64, G=128) == -4
    assert call(Hq=40, Hkv=4) == -5          # 10 query heads per KV head
    assert call(Hq=30) == -5                 # not a multiple of Hkv
    assert call(T=4000 + 8) == -5            # T % 16 != 0
    assert call(B=-1) == -5
    assert call(q=0) == -1 and call(out=0) == -1 and call(lens=0) == -1
    assert call(q=A_ + 8) == -2 and call(out=A_ + 8) == -2 and call(lens=A_ + 2) == -2
    assert call(B=0, q=0, out=0, lens=0) == 0
    assert kvq.kvq_attention_workspace_bytes(1, 32, 8, 4096, 96, 32) == -1
    assert kvq.kvq_attention_workspace_bytes(1, 32, 8, 4096, 256, 16) > 0
    assert kvq.kvq_attention_workspace_bytes(4096, 32, 8, 4096, 128, 32) == 0


def test_dequantize_tc_errors(kvq):
    d = lambda **kw: kvq.kvq_dequantize_tc(kw.get("p", A), A, A, A, kw.get("n", 64), kw.get("D", 128),
                                           kw.get("G", 32), kw.get("out", A))
    assert d(D=64) == -3 and d(D=256) == -3 and d(D=96) == -3
    assert d(G=128) == -4 and d(G=8) == -4
    assert d(n=-1) == -5 and d(n=0) == 0
    assert d(p=0) == -1 and d(out=0) == -1 and d(out=A + 8) == -2


def test_codec_ex_errors(kvq):
    q = lambda **kw: kvq.kvq_quantize_ex(kw.get("x", A), kw.get("lam", A), A, kw.get("n", 64),
                                         kw.get("D", 128), kw.get("G", 32), kw.get("bits", 4),
                                         0, kw.get("rows", 64), kw.get("nl", 1), kw.get("codes", A), A)
    d = lambda **kw: kvq.kvq_dequantize_ex(kw.get("codes", A), A, A, A, kw.get("n", 64),
                                           kw.get("D", 128), kw.get("G", 32), kw.get("bits", 4),
                                           1, kw.get("rows", 64), kw.get("nl", 1), kw.get("out", A))
    flag = lambda **kw: kvq.kvq_quantize_ex(A, A, A, 64, 128, 32, 4, kw["flags"], 64, 1, A, A)
    assert flag(flags=4) == -4 and flag(flags=-1) == -4
    for f in (q, d):
        assert f(D=64) == -3 and f(D=256) == -3
        assert f(G=128) == -4 and f(G=8) == -4 and f(bits=5) == -4
        assert f(n=-1) == -5 and f(nl=0) == -5 and f(rows=0) == -5
        assert f(nl=3, rows=48) == -5            # several tables: rows a multiple of 32
        assert f(n=0) == 0
    assert q(x=0) == -1 and q(codes=0) == -1 and d(codes=0) == -1 and d(out=0) == -1
    assert q(x=A + 8) == -2 and q(lam=A + 2) == -2 and d(codes=A + 8) == -2 and d(out=A + 8) == -2
    # the SRFT (flags bit 1) takes D = 64, 96, 128 or 256 and a group dividing D
    sq = lambda **kw: kvq.kvq_quantize_ex(A, A, A, kw.get("n", 64), kw["D"], kw.get("G", 32), 4,
                                          2 | kw.get("after", 0), 64, 1, A, A)
    sd = lambda **kw: kvq.kvq_dequantize_ex(A, A, A, A, kw.get("n", 64), kw["D"], kw.get("G", 32), 8,
                                            2 | kw.get("after", 0), 64, 1, A)
    for f in (sq, sd):
        assert f(D=96, G=64) == -4 and f(D=80) == -3 and f(D=512) == -3 and f(D=32) == -3
        assert f(D=192) == -3 and f(D=256, G=128) == -4
        for D in (64, 96, 128, 256):
            assert f(D=D, n=0) == 0 and f(D=D, n=0, after=1) == 0
