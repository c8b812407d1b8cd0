"""CPU oracle for the fused KV-cache rotate-and-quantize path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's ``smoke()`` check
and the benchmark's CPU-baseline / reference legs may import this module.  The
product path (the CUDA library and its binding) never imports, loads or
calls it, and it shares no code with that path.

The arithmetic lives in ``kvq_oracle.c`` (plain C99, compiled with
``-O2 -ffp-contract=off``, no fast-math).  This module only compiles it,
loads it with ctypes and marshals numpy arrays.  ctypes releases the GIL
during each foreign call, so callers may run row slices in Python threads.

Functions pinned by the ``-m "not gpu"`` tests: every public function here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "kvq_oracle.c")
LIBRARY = os.path.join(_HERE, "libkvq_oracle.so")

CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall", "-Wextra"]

_lock = threading.Lock()


def build(source: str = SOURCE, output: str = LIBRARY) -> str:
    """Compile the C oracle into a shared library (gcc).  Returns its path."""
    cmd = ["gcc", *CFLAGS, source, "-o", output, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return output


def _needs_build(output: str, source: str) -> bool:
    return (not os.path.exists(output)
            or os.path.getmtime(output) < os.path.getmtime(source))


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


class Oracle:
    """ctypes handle on one compiled copy of the C oracle."""

    def __init__(self, library: str | None = None):
        if library is None:
            with _lock:
                if _needs_build(LIBRARY, SOURCE):
                    build()
            library = LIBRARY
        self.path = library
        lib = ctypes.CDLL(library)
        sig = {
            "kvqo_f32_to_f16": (ctypes.c_uint16, [ctypes.c_float]),
            "kvqo_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
            "kvqo_norm_const": (ctypes.c_float, [_I]),
            "kvqo_fwht_f64": (None, [_P, _I]),
            "kvqo_fwht_f32": (None, [_P, _I]),
            "kvqo_rotate_f64": (None, [_P, _P, _P, _I, _P]),
            "kvqo_unrotate_f64": (None, [_P, _P, _P, _I, _P]),
            "kvqo_rotate_f32": (_I, [_P, _P, _P, _I64, _I, _P]),
            "kvqo_unrotate_f32": (_I, [_P, _P, _P, _I64, _I, _P]),
            "kvqo_quantize_codes": (_I, [_P, _P, _P, _I64, _I, _I, _P, _P]),
            "kvqo_quantize_codes_divform": (_I, [_P, _P, _P, _I64, _I, _I, _P]),
            "kvqo_quantize": (_I, [_P, _P, _P, _I64, _I, _I, _P, _P]),
            "kvqo_dequantize": (_I, [_P, _P, _P, _P, _I64, _I, _I, _P]),
            "kvqo_dequantize_f32": (_I, [_P, _P, _P, _P, _I64, _I, _I, _P]),
            "kvqo_pack": (None, [_P, _I64, _P]),
            "kvqo_unpack": (None, [_P, _I64, _P]),
            "kvqo_quantize_ex": (_I, [_P, _P, _P, _I64, _I, _I, _I, _I, _I64, _I, _P, _P]),
            "kvqo_dequantize_ex": (_I, [_P, _P, _P, _P, _I64, _I, _I, _I, _I, _I64, _I, _P]),
            "kvqo_srft_f32": (_I, [_P, _I, _P]),
            "kvqo_isrft_f32": (_I, [_P, _I, _P]),
            "kvqo_twiddle": (None, [_I, _I, _P, _P]),
            "kvqo_fft_f32": (_I, [_P, _P, _I, _I]),
            "kvqo_srft_f64": (None, [_P, _I, _P]),
            "kvqo_isrft_f64": (None, [_P, _I, _P]),
            "kvqo_attention_decode": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                           _I, _I, _I, _I, _I, _I, ctypes.c_double, _P]),
            "kvqo_attention_decode_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                              _I, _I, _I, _I, _I, _I, _I, ctypes.c_double, _P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        self._lib = lib

    # ---- scalar helpers -------------------------------------------------
    def f32_to_f16_bits(self, f: float) -> int:
        return int(self._lib.kvqo_f32_to_f16(float(f)))

    def f16_bits_to_f32(self, bits: int) -> float:
        return float(self._lib.kvqo_f16_to_f32(int(bits)))

    def norm_const(self, D: int) -> float:
        return float(self._lib.kvqo_norm_const(int(D)))

    # ---- transforms -----------------------------------------------------
    def fwht_f64(self, v: np.ndarray) -> np.ndarray:
        out = np.ascontiguousarray(v, dtype=np.float64).copy()
        self._lib.kvqo_fwht_f64(_ptr(out), out.shape[-1])
        return out

    def fwht_f32(self, v: np.ndarray) -> np.ndarray:
        out = np.ascontiguousarray(v, dtype=np.float32).copy()
        self._lib.kvqo_fwht_f32(_ptr(out), out.shape[-1])
        return out

    def rotate_f64(self, x, lam, signs) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float64)
        lam = np.ascontiguousarray(lam, dtype=np.float64)
        s = np.ascontiguousarray(signs, dtype=np.int8)
        y = np.empty_like(x)
        self._lib.kvqo_rotate_f64(_ptr(x), _ptr(lam), _ptr(s), x.shape[-1], _ptr(y))
        return y

    def unrotate_f64(self, y, lam, signs) -> np.ndarray:
        y = np.ascontiguousarray(y, dtype=np.float64)
        lam = np.ascontiguousarray(lam, dtype=np.float64)
        s = np.ascontiguousarray(signs, dtype=np.int8)
        x = np.empty_like(y)
        self._lib.kvqo_unrotate_f64(_ptr(y), _ptr(lam), _ptr(s), y.shape[-1], _ptr(x))
        return x

    def rotate_f32(self, x_f16, lam, signs) -> np.ndarray:
        x = _rows_f16(x_f16)
        lam, s = _params(lam, signs)
        y = np.empty(x.shape, dtype=np.float32)
        _check(self._lib.kvqo_rotate_f32(_ptr(x), _ptr(lam), _ptr(s),
                                         x.shape[0], x.shape[1], _ptr(y)))
        return y

    def unrotate_f32(self, y, lam, signs) -> np.ndarray:
        y = np.ascontiguousarray(np.atleast_2d(y), dtype=np.float32)
        lam, s = _params(lam, signs)
        x = np.empty_like(y)
        _check(self._lib.kvqo_unrotate_f32(_ptr(y), _ptr(lam), _ptr(s),
                                           y.shape[0], y.shape[1], _ptr(x)))
        return x

    # ---- the quantiser ----------------------------------------------------
    def quantize_codes(self, x_f16, lam, signs, group: int):
        """Unpacked codes int8[n, D] and fp16 scales [n, D/group]."""
        x = _rows_f16(x_f16)
        lam, s = _params(lam, signs)
        n, D = x.shape
        codes = np.empty((n, D), dtype=np.int8)
        scales = np.empty((n, D // group), dtype=np.uint16)
        _check(self._lib.kvqo_quantize_codes(_ptr(x), _ptr(lam), _ptr(s), n, D,
                                             group, _ptr(codes), _ptr(scales)))
        return codes, scales.view(np.float16)

    def quantize_codes_divform(self, x_f16, lam, signs, group: int):
        x = _rows_f16(x_f16)
        lam, s = _params(lam, signs)
        n, D = x.shape
        codes = np.empty((n, D), dtype=np.int8)
        _check(self._lib.kvqo_quantize_codes_divform(_ptr(x), _ptr(lam), _ptr(s),
                                                     n, D, group, _ptr(codes)))
        return codes

    def quantize(self, x_f16, lam, signs, group: int):
        """Packed codes uint8[n, D/2] and fp16 scales [n, D/group]."""
        x = _rows_f16(x_f16)
        lam, s = _params(lam, signs)
        n, D = x.shape
        packed = np.empty((n, D // 2), dtype=np.uint8)
        scales = np.empty((n, D // group), dtype=np.uint16)
        _check(self._lib.kvqo_quantize(_ptr(x), _ptr(lam), _ptr(s), n, D, group,
                                       _ptr(packed), _ptr(scales)))
        return packed, scales.view(np.float16)

    def dequantize(self, packed, scales, lam, signs, group: int) -> np.ndarray:
        """fp16 [n, D] from packed codes and fp16 scales."""
        packed = np.ascontiguousarray(np.atleast_2d(packed), dtype=np.uint8)
        sc = np.ascontiguousarray(np.atleast_2d(scales)).view(np.uint16)
        lam, s = _params(lam, signs)
        n, D = packed.shape[0], packed.shape[1] * 2
        out = np.empty((n, D), dtype=np.uint16)
        _check(self._lib.kvqo_dequantize(_ptr(packed), _ptr(sc), _ptr(lam), _ptr(s),
                                         n, D, group, _ptr(out)))
        return out.view(np.float16)

    def dequantize_f32(self, codes, scales, lam, signs, group: int) -> np.ndarray:
        """fp32 [n, D] (no final fp16 rounding) from unpacked codes."""
        codes = np.ascontiguousarray(np.atleast_2d(codes), dtype=np.int8)
        sc = np.ascontiguousarray(np.atleast_2d(scales)).view(np.uint16)
        lam, s = _params(lam, signs)
        n, D = codes.shape
        out = np.empty((n, D), dtype=np.float32)
        _check(self._lib.kvqo_dequantize_f32(_ptr(codes), _ptr(sc), _ptr(lam), _ptr(s),
                                             n, D, group, _ptr(out)))
        return out

    def pack(self, codes) -> np.ndarray:
        codes = np.ascontiguousarray(codes, dtype=np.int8)
        out = np.empty(codes.shape[:-1] + (codes.shape[-1] // 2,), dtype=np.uint8)
        self._lib.kvqo_pack(_ptr(codes), codes.size, _ptr(out))
        return out

    def unpack(self, packed) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int8)
        self._lib.kvqo_unpack(_ptr(packed), packed.size * 2, _ptr(out))
        return out


    def twiddle(self, k: int, M: int) -> tuple[np.float32, np.float32]:
        """The oracle's fp32 omega_M^k = (cos, -sin)(2 pi k / M)."""
        wr, wi = ctypes.c_float(), ctypes.c_float()
        self._lib.kvqo_twiddle(k, M, ctypes.byref(wr), ctypes.byref(wi))
        return np.float32(wr.value), np.float32(wi.value)

    def fft_f32(self, z, inverse: bool = False) -> np.ndarray:
        """The oracle's fp32 complex FFT of rows z [n, N] (forward DIF stages,
        or with inverse=True their transpose: the unnormalised conjugate DFT)."""
        z = np.atleast_2d(np.asarray(z, dtype=np.complex64))
        out = np.empty_like(z)
        for r in range(z.shape[0]):
            re = np.ascontiguousarray(z[r].real, dtype=np.float32)
            im = np.ascontiguousarray(z[r].imag, dtype=np.float32)
            _check(self._lib.kvqo_fft_f32(_ptr(re), _ptr(im), z.shape[1], 1 if inverse else 0))
            out[r] = re + 1j * im
        return out

    def srft_f32(self, v) -> np.ndarray:
        """fp32 SRFT (packed unitary real DFT) of rows v [n, D]."""
        v = np.ascontiguousarray(np.atleast_2d(v), dtype=np.float32)
        out = np.empty_like(v)
        for r in range(v.shape[0]):
            _check(self._lib.kvqo_srft_f32(_ptr(v[r]), v.shape[1], _ptr(out[r])))
        return out

    def isrft_f32(self, y) -> np.ndarray:
        y = np.ascontiguousarray(np.atleast_2d(y), dtype=np.float32)
        out = np.empty_like(y)
        for r in range(y.shape[0]):
            _check(self._lib.kvqo_isrft_f32(_ptr(y[r]), y.shape[1], _ptr(out[r])))
        return out

    def srft_f64(self, v) -> np.ndarray:
        v = np.ascontiguousarray(np.atleast_2d(v), dtype=np.float64)
        out = np.empty_like(v)
        for r in range(v.shape[0]):
            self._lib.kvqo_srft_f64(_ptr(v[r]), v.shape[1], _ptr(out[r]))
        return out

    def isrft_f64(self, y) -> np.ndarray:
        y = np.ascontiguousarray(np.atleast_2d(y), dtype=np.float64)
        out = np.empty_like(y)
        for r in range(y.shape[0]):
            self._lib.kvqo_isrft_f64(_ptr(y[r]), y.shape[1], _ptr(out[r]))
        return out

    def quantize_ex(self, x_f16, lam, signs, group: int, bits: int = 4, lambda_after: bool = False,
                    lambda_rows: int | None = None, srft: bool = False):
        """Format variants: lam is [n_lambda, D] (or [D]); row r uses table
        (r // lambda_rows) % n_lambda.  Returns (codes uint8 [n, D/2 or D],
        scales fp16 [n, D/group])."""
        x = _rows_f16(x_f16)
        n, D = x.shape
        lam = np.ascontiguousarray(np.atleast_2d(lam), dtype=np.float32)
        s = np.ascontiguousarray(signs, dtype=np.int8)
        nl = lam.shape[0]
        rows = lambda_rows if lambda_rows is not None else max(n, 1)
        codes = np.empty((n, D // 2 if bits == 4 else D), dtype=np.uint8)
        scales = np.empty((n, D // group), dtype=np.uint16)
        _check(self._lib.kvqo_quantize_ex(_ptr(x), _ptr(lam), _ptr(s), n, D, group, bits,
                                          _flags(lambda_after, srft), rows, nl,
                                          _ptr(codes), _ptr(scales)))
        return codes, scales.view(np.float16)

    def dequantize_ex(self, codes, scales, lam, signs, group: int, bits: int = 4,
                      lambda_after: bool = False, lambda_rows: int | None = None,
                      srft: bool = False) -> np.ndarray:
        codes = np.ascontiguousarray(np.atleast_2d(codes), dtype=np.uint8)
        sc = np.ascontiguousarray(np.atleast_2d(scales)).view(np.uint16)
        lam = np.ascontiguousarray(np.atleast_2d(lam), dtype=np.float32)
        s = np.ascontiguousarray(signs, dtype=np.int8)
        n = codes.shape[0]
        D = codes.shape[1] * (2 if bits == 4 else 1)
        rows = lambda_rows if lambda_rows is not None else max(n, 1)
        out = np.empty((n, D), dtype=np.uint16)
        _check(self._lib.kvqo_dequantize_ex(_ptr(codes), _ptr(sc), _ptr(lam), _ptr(s), n, D,
                                            group, bits, _flags(lambda_after, srft), rows,
                                            lam.shape[0], _ptr(out)))
        return out.view(np.float16)

    def attention_decode(self, q, k_packed, k_scales, v_packed, v_scales, seq_len,
                         lam_k, s_k, lam_v, s_v, group: int, sm_scale: float,
                         lambda_after: bool = False, srft: bool = False) -> np.ndarray:
        """Decode attention over the int4 cache, float64 [B, Hq, D].

        q fp16 [B, Hq, D]; packed u8 [B, Hkv, T, D/2]; scales fp16
        [B, Hkv, T, D/group]; seq_len int [B].  lambda_after / srft: the
        cache's rows are codec-variant rows of that format."""
        q = np.ascontiguousarray(q)
        if q.dtype != np.float16 or q.ndim != 3:
            raise TypeError("q must be float16 [B, Hq, D]")
        B, Hq, D = q.shape
        kp = np.ascontiguousarray(k_packed, dtype=np.uint8)
        vp = np.ascontiguousarray(v_packed, dtype=np.uint8)
        ks = np.ascontiguousarray(k_scales).view(np.uint16)
        vs = np.ascontiguousarray(v_scales).view(np.uint16)
        if kp.ndim != 4 or kp.shape[0] != B or kp.shape[3] * 2 != D or vp.shape != kp.shape:
            raise ValueError("packed caches must be [B, Hkv, T, D/2]")
        Hkv, T = kp.shape[1], kp.shape[2]
        sl = np.ascontiguousarray(seq_len, dtype=np.int32)
        lk, sk = _params(lam_k, s_k)
        lv, sv = _params(lam_v, s_v)
        out = np.empty((B, Hq, D), dtype=np.float64)
        _check(self._lib.kvqo_attention_decode_ex(
            _ptr(q.view(np.uint16)), _ptr(kp), _ptr(ks), _ptr(vp), _ptr(vs), _ptr(sl),
            _ptr(lk), _ptr(sk), _ptr(lv), _ptr(sv), B, Hq, Hkv, T, D, group,
            _flags(lambda_after, srft), float(sm_scale), _ptr(out)))
        return out


def _flags(lambda_after: bool, srft: bool) -> int:
    return (1 if lambda_after else 0) | (2 if srft else 0)


def _rows_f16(x) -> np.ndarray:
    x = np.atleast_2d(np.asarray(x))
    if x.dtype != np.float16:
        raise TypeError("oracle input rows must be float16")
    return np.ascontiguousarray(x).view(np.uint16)


def _params(lam, signs):
    lam = np.ascontiguousarray(lam, dtype=np.float32)
    s = np.ascontiguousarray(signs, dtype=np.int8)
    return lam, s


def _check(rc: int) -> None:
    if rc != 0:
        raise ValueError(f"oracle rejected the shape (status {rc})")


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle compiled from this directory's source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
