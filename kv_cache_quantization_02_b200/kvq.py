"""Thin Python binding of libkvq.so (include/kvq.h), argument marshalling only.

The raw entry points keep the C names and take integer device addresses:

    kvq_quantize(x, lam, signs, n_vec, D, group, packed, scales, stream) -> status
    kvq_dequantize(packed, scales, lam, signs, n_vec, D, group, x_out, stream) -> status
    kvq_attention_decode(q, k_packed, k_scales, v_packed, v_scales, seq_len,
                         lam_k, s_k, lam_v, s_v, B, Hq, Hkv, T, D, group,
                         sm_scale, out, workspace, workspace_bytes, stream) -> status

``quantize`` / ``dequantize`` accept torch CUDA tensors, allocate outputs
with torch when none are given, call the C entry point on the current (or
given) stream and raise ``KvqError`` on a non-zero status.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback.  If the
library is missing, importing this module raises ImportError.
"""
from __future__ import annotations

import ctypes
import os

import torch  # loads libcudart first, so the library shares torch's runtime

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_PKG, "libkvq.so")

if not os.path.exists(LIBRARY):
    raise ImportError(
        f"{LIBRARY} is not built; run `python -m kv_cache_quantization_02_b200.build`")

_lib = ctypes.CDLL(LIBRARY)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int

_lib.kvq_quantize.restype = _I
_lib.kvq_quantize.argtypes = [_P, _P, _P, _I64, _I, _I, _P, _P, _P]
_lib.kvq_quantize_rows.restype = _I
_lib.kvq_quantize_rows.argtypes = [_P, _P, _P, _I64, _I, _I, _P, _I64, _P, _P, _P]
_lib.kvq_roundtrip.restype = _I
_lib.kvq_roundtrip.argtypes = [_P, _P, _P, _I64, _I, _I, _P, _P, _P, _P]
_lib.kvq_dequantize.restype = _I
_lib.kvq_dequantize.argtypes = [_P, _P, _P, _P, _I64, _I, _I, _P, _P]
_lib.kvq_dequantize_tc.restype = _I
_lib.kvq_dequantize_tc.argtypes = [_P, _P, _P, _P, _I64, _I, _I, _P, _P]
_lib.kvq_quantize_ex.restype = _I
_lib.kvq_quantize_ex.argtypes = [_P, _P, _P, _I64, _I, _I, _I, _I, _I64, _I, _P, _P, _P]
_lib.kvq_dequantize_ex.restype = _I
_lib.kvq_dequantize_ex.argtypes = [_P, _P, _P, _P, _I64, _I, _I, _I, _I, _I64, _I, _P, _P]
_lib.kvq_attention_decode.restype = _I
_lib.kvq_attention_decode.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                      _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P, _I64, _P]
_lib.kvq_attention_decode_ex.restype = _I
_lib.kvq_attention_decode_ex.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                         _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P, _I64, _P]
_lib.kvq_attention_decode_static.restype = _I
_lib.kvq_attention_decode_static.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                             _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P]
_lib.kvq_attention_workspace_bytes.restype = _I64
_lib.kvq_attention_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
_lib.kvq_status_string.restype = ctypes.c_char_p
_lib.kvq_status_string.argtypes = [_I]
_lib.kvq_last_cuda_error.restype = _I
_lib.kvq_last_cuda_error.argtypes = []
_lib.kvq_version.restype = _I
_lib.kvq_version.argtypes = []
_lib.kvq_fault_status.restype = _I
_lib.kvq_fault_status.argtypes = [_I]
_lib.kvq_selftest_wait_timeout.restype = _I
_lib.kvq_selftest_wait_timeout.argtypes = [ctypes.c_uint32, _P]
_lib.kvq_selftest_rcp_f16.restype = _I
_lib.kvq_selftest_rcp_f16.argtypes = [_P, _P]

KVQ_OK = 0
KVQ_ERR_NULL = -1
KVQ_ERR_ALIGN = -2
KVQ_ERR_DIM = -3
KVQ_ERR_GROUP = -4
KVQ_ERR_COUNT = -5
KVQ_ERR_LAUNCH = -6


class KvqError(RuntimeError):
    def __init__(self, status: int):
        msg = kvq_status_string(status)
        if status == KVQ_ERR_LAUNCH:
            msg += f" (cudaError {kvq_last_cuda_error()})"
        super().__init__(msg)
        self.status = status


# ---- raw C entry points -------------------------------------------------

def kvq_quantize(x: int, lam: int, signs: int, n_vec: int, D: int, group: int,
                 packed: int, scales: int, stream: int = 0) -> int:
    return _lib.kvq_quantize(x, lam, signs, n_vec, D, group, packed, scales, stream)


def kvq_quantize_rows(x: int, lam: int, signs: int, n_vec: int, D: int, group: int,
                      row_idx: int, cache_rows: int, packed: int, scales: int,
                      stream: int = 0) -> int:
    return _lib.kvq_quantize_rows(x, lam, signs, n_vec, D, group, row_idx, cache_rows,
                                  packed, scales, stream)


def kvq_roundtrip(x: int, lam: int, signs: int, n_vec: int, D: int, group: int,
                  x_hat: int, packed: int = 0, scales: int = 0, stream: int = 0) -> int:
    return _lib.kvq_roundtrip(x, lam, signs, n_vec, D, group, x_hat, packed, scales, stream)


def kvq_dequantize(packed: int, scales: int, lam: int, signs: int, n_vec: int,
                   D: int, group: int, x_out: int, stream: int = 0) -> int:
    return _lib.kvq_dequantize(packed, scales, lam, signs, n_vec, D, group, x_out, stream)


KVQ_LAMBDA_AFTER = 1
KVQ_SRFT = 2


def kvq_dequantize_tc(packed: int, scales: int, lam: int, signs: int, n_vec: int,
                      D: int, group: int, x_out: int, stream: int = 0) -> int:
    return _lib.kvq_dequantize_tc(packed, scales, lam, signs, n_vec, D, group, x_out, stream)


def kvq_quantize_ex(x: int, lam: int, signs: int, n_vec: int, D: int, group: int, bits: int,
                    flags: int, lambda_rows: int, n_lambda: int, codes: int, scales: int,
                    stream: int = 0) -> int:
    return _lib.kvq_quantize_ex(x, lam, signs, n_vec, D, group, bits, flags, lambda_rows,
                                n_lambda, codes, scales, stream)


def kvq_dequantize_ex(codes: int, scales: int, lam: int, signs: int, n_vec: int, D: int,
                      group: int, bits: int, flags: int, lambda_rows: int, n_lambda: int,
                      x_out: int, stream: int = 0) -> int:
    return _lib.kvq_dequantize_ex(codes, scales, lam, signs, n_vec, D, group, bits, flags,
                                  lambda_rows, n_lambda, x_out, stream)


def _ex_flags(lambda_after: bool, srft: bool) -> int:
    return (KVQ_LAMBDA_AFTER if lambda_after else 0) | (KVQ_SRFT if srft else 0)


def kvq_attention_decode(q: int, k_packed: int, k_scales: int, v_packed: int, v_scales: int,
                         seq_len: int, lam_k: int, s_k: int, lam_v: int, s_v: int,
                         B: int, Hq: int, Hkv: int, T: int, D: int, group: int,
                         sm_scale: float, out: int, workspace: int = 0,
                         workspace_bytes: int = 0, stream: int = 0) -> int:
    return _lib.kvq_attention_decode(q, k_packed, k_scales, v_packed, v_scales, seq_len,
                                     lam_k, s_k, lam_v, s_v, B, Hq, Hkv, T, D, group,
                                     sm_scale, out, workspace, workspace_bytes, stream)


def kvq_attention_decode_ex(q: int, k_packed: int, k_scales: int, v_packed: int, v_scales: int,
                            seq_len: int, lam_k: int, s_k: int, lam_v: int, s_v: int,
                            B: int, Hq: int, Hkv: int, T: int, D: int, group: int, flags: int,
                            sm_scale: float, out: int, workspace: int = 0,
                            workspace_bytes: int = 0, stream: int = 0) -> int:
    return _lib.kvq_attention_decode_ex(q, k_packed, k_scales, v_packed, v_scales, seq_len,
                                        lam_k, s_k, lam_v, s_v, B, Hq, Hkv, T, D, group, flags,
                                        sm_scale, out, workspace, workspace_bytes, stream)


def kvq_attention_decode_static(q: int, k_packed: int, k_scales: int, v_packed: int,
                                v_scales: int, seq_len: int, lam_k: int, s_k: int, lam_v: int,
                                s_v: int, B: int, Hq: int, Hkv: int, T: int, D: int, group: int,
                                sm_scale: float, out: int, stream: int = 0) -> int:
    return _lib.kvq_attention_decode_static(q, k_packed, k_scales, v_packed, v_scales, seq_len,
                                            lam_k, s_k, lam_v, s_v, B, Hq, Hkv, T, D, group,
                                            sm_scale, out, stream)


def kvq_attention_workspace_bytes(B: int, Hq: int, Hkv: int, T: int, D: int, group: int) -> int:
    return _lib.kvq_attention_workspace_bytes(B, Hq, Hkv, T, D, group)


def kvq_status_string(status: int) -> str:
    return _lib.kvq_status_string(status).decode()


def kvq_last_cuda_error() -> int:
    return _lib.kvq_last_cuda_error()


def kvq_version() -> int:
    return _lib.kvq_version()


def kvq_fault_status(clear: bool = False) -> int:
    return _lib.kvq_fault_status(1 if clear else 0)


def kvq_selftest_wait_timeout(limit: int, stream: int = 0) -> int:
    return _lib.kvq_selftest_wait_timeout(limit, stream)


def kvq_selftest_rcp_f16(out: int, stream: int = 0) -> int:
    return _lib.kvq_selftest_rcp_f16(out, stream)


# ---- torch-tensor convenience --------------------------------------------

def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _need(t: torch.Tensor, dtype, shape, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def quantize(x: torch.Tensor, lam: torch.Tensor, signs: torch.Tensor, group: int,
             packed: torch.Tensor | None = None, scales: torch.Tensor | None = None,
             stream=None):
    """x: fp16 [n, D] -> (packed uint8 [n, D/2], scales fp16 [n, D/group])."""
    if x.dim() != 2:
        raise ValueError("x must be [n_vec, D]")
    n, D = x.shape
    _need(x, torch.float16, (n, D), "x")
    _need(lam, torch.float32, (D,), "lambda")
    _need(signs, torch.int8, (D,), "signs")
    if packed is None:
        packed = torch.empty((n, D // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((n, max(D // group, 1)), dtype=torch.float16, device=x.device)
    _need(packed, torch.uint8, (n, D // 2), "packed")
    _need(scales, torch.float16, (n, max(D // group, 1)), "scales")
    rc = kvq_quantize(x.data_ptr(), lam.data_ptr(), signs.data_ptr(), n, D, group,
                      packed.data_ptr(), scales.data_ptr(), _stream_handle(stream))
    if rc != KVQ_OK:
        raise KvqError(rc)
    return packed, scales


def quantize_rows(x: torch.Tensor, lam: torch.Tensor, signs: torch.Tensor, group: int,
                  row_idx: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                  stream=None):
    """Encode x: fp16 [n, D] into rows row_idx (int64 [n]) of the cache
    (packed uint8 [N, D/2], scales fp16 [N, D/group]); other rows untouched."""
    if x.dim() != 2:
        raise ValueError("x must be [n_vec, D]")
    n, D = x.shape
    _need(x, torch.float16, (n, D), "x")
    _need(lam, torch.float32, (D,), "lambda")
    _need(signs, torch.int8, (D,), "signs")
    _need(row_idx, torch.int64, (n,), "row_idx")
    N = packed.shape[0]
    _need(packed, torch.uint8, (N, D // 2), "packed")
    _need(scales, torch.float16, (N, max(D // group, 1)), "scales")
    rc = kvq_quantize_rows(x.data_ptr(), lam.data_ptr(), signs.data_ptr(), n, D, group,
                           row_idx.data_ptr(), N, packed.data_ptr(), scales.data_ptr(),
                           _stream_handle(stream))
    if rc != KVQ_OK:
        raise KvqError(rc)
    return packed, scales


def roundtrip(x: torch.Tensor, lam: torch.Tensor, signs: torch.Tensor, group: int,
              out: torch.Tensor | None = None, packed: torch.Tensor | None = None,
              scales: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """x_hat = dequantize(quantize(x)) in one kernel; codes/scales optional."""
    if x.dim() != 2:
        raise ValueError("x must be [n_vec, D]")
    n, D = x.shape
    _need(x, torch.float16, (n, D), "x")
    _need(lam, torch.float32, (D,), "lambda")
    _need(signs, torch.int8, (D,), "signs")
    if out is None:
        out = torch.empty((n, D), dtype=torch.float16, device=x.device)
    _need(out, torch.float16, (n, D), "out")
    if (packed is None) != (scales is None):
        raise ValueError("pass both packed and scales, or neither")
    pk = sc = 0
    if packed is not None:
        _need(packed, torch.uint8, (n, D // 2), "packed")
        _need(scales, torch.float16, (n, max(D // group, 1)), "scales")
        pk, sc = packed.data_ptr(), scales.data_ptr()
    rc = kvq_roundtrip(x.data_ptr(), lam.data_ptr(), signs.data_ptr(), n, D, group,
                       out.data_ptr(), pk, sc, _stream_handle(stream))
    if rc != KVQ_OK:
        raise KvqError(rc)
    return out


def quantize_ex(x: torch.Tensor, lam: torch.Tensor, signs: torch.Tensor, group: int,
                bits: int = 4, lambda_after: bool = False, lambda_rows: int | None = None,
                codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                stream=None, srft: bool = False):
    """Format variants.  x fp16 [n, D]; lam fp32 [n_lambda, D] (or [D]); row r
    uses table (r // lambda_rows) % n_lambda.  -> (codes uint8 [n, D/2 or D],
    scales fp16 [n, D/group]).  D = 128, or 64, 96, 128, 256 with srft=True."""
    if x.dim() != 2:
        raise ValueError("x must be [n_vec, D]")
    n, D = x.shape
    _need(x, torch.float16, (n, D), "x")
    lam2 = lam.reshape(-1, D)
    _need(lam2, torch.float32, (lam2.shape[0], D), "lambda")
    _need(signs, torch.int8, (D,), "signs")
    cb = D // 2 if bits == 4 else D
    if codes is None:
        codes = torch.empty((n, cb), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((n, D // group), dtype=torch.float16, device=x.device)
    _need(codes, torch.uint8, (n, cb), "codes")
    _need(scales, torch.float16, (n, D // group), "scales")
    rows = lambda_rows if lambda_rows is not None else max(n, 1)
    rc = kvq_quantize_ex(x.data_ptr(), lam2.data_ptr(), signs.data_ptr(), n, D, group, bits,
                         _ex_flags(lambda_after, srft), rows, lam2.shape[0], codes.data_ptr(),
                         scales.data_ptr(), _stream_handle(stream))
    if rc != KVQ_OK:
        raise KvqError(rc)
    return codes, scales


def dequantize_ex(codes: torch.Tensor, scales: torch.Tensor, lam: torch.Tensor,
                  signs: torch.Tensor, group: int, bits: int = 4, lambda_after: bool = False,
                  lambda_rows: int | None = None, out: torch.Tensor | None = None,
                  stream=None, srft: bool = False) -> torch.Tensor:
    """Inverse of quantize_ex -> fp16 [n, D]."""
    if codes.dim() != 2:
        raise ValueError("codes must be [n_vec, bytes]")
    n = codes.shape[0]
    D = codes.shape[1] * (2 if bits == 4 else 1)
    _need(codes, torch.uint8, (n, codes.shape[1]), "codes")
    _need(scales, torch.float16, (n, D // group), "scales")
    lam2 = lam.reshape(-1, D)
    _need(lam2, torch.float32, (lam2.shape[0], D), "lambda")
    _need(signs, torch.int8, (D,), "signs")
    if out is None:
        out = torch.empty((n, D), dtype=torch.float16, device=codes.device)
    _need(out, torch.float16, (n, D), "out")
    rows = lambda_rows if lambda_rows is not None else max(n, 1)
    rc = kvq_dequantize_ex(codes.data_ptr(), scales.data_ptr(), lam2.data_ptr(), signs.data_ptr(),
                           n, D, group, bits, _ex_flags(lambda_after, srft), rows, lam2.shape[0],
                           out.data_ptr(), _stream_handle(stream))
    if rc != KVQ_OK:
        raise KvqError(rc)
    return out


def attention_decode(q: torch.Tensor, k_packed: torch.Tensor, k_scales: torch.Tensor,
                     v_packed: torch.Tensor, v_scales: torch.Tensor, seq_len: torch.Tensor,
                     lam_k: torch.Tensor, s_k: torch.Tensor, lam_v: torch.Tensor,
                     s_v: torch.Tensor, group: int, sm_scale: float,
                     out: torch.Tensor | None = None, workspace: torch.Tensor | bool = True,
                     stream=None, lambda_after: bool = False, srft: bool = False) -> torch.Tensor:
    """Decode attention over the int4 cache.  q fp16 [B, Hq, D]; packed uint8
    [B, Hkv, T, D/2]; scales fp16 [B, Hkv, T, D/group]; seq_len int32 [B]
    -> fp16 [B, Hq, D].  ``workspace``: a uint8 CUDA tensor, True to allocate
    the size the library asks for, or False to run without splitting.
    ``lambda_after`` / ``srft``: the cache's rows are quantize_ex rows of that
    format (int4)."""
    if q.dim() != 3 or k_packed.dim() != 4:
        raise ValueError("q must be [B, Hq, D] and the caches [B, Hkv, T, D/2]")
    B, Hq, D = q.shape
    Hkv, T = k_packed.shape[1], k_packed.shape[2]
    _need(q, torch.float16, (B, Hq, D), "q")
    for name, t in (("k_packed", k_packed), ("v_packed", v_packed)):
        _need(t, torch.uint8, (B, Hkv, T, D // 2), name)
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _need(t, torch.float16, (B, Hkv, T, max(D // group, 1)), name)
    _need(seq_len, torch.int32, (B,), "seq_len")
    for name, t in (("lambda_k", lam_k), ("lambda_v", lam_v)):
        _need(t, torch.float32, (D,), name)
    for name, t in (("signs_k", s_k), ("signs_v", s_v)):
        _need(t, torch.int8, (D,), name)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, torch.float16, (B, Hq, D), "out")
    ws, wsb = 0, 0
    if workspace is True:
        need = kvq_attention_workspace_bytes(B, Hq, Hkv, T, D, group)
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        else:
            workspace = None
    if isinstance(workspace, torch.Tensor):
        if not workspace.is_cuda or workspace.dtype != torch.uint8:
            raise ValueError("workspace must be a uint8 CUDA tensor")
        ws, wsb = workspace.data_ptr(), workspace.numel()
    rc = kvq_attention_decode_ex(q.data_ptr(), k_packed.data_ptr(), k_scales.data_ptr(),
                                 v_packed.data_ptr(), v_scales.data_ptr(), seq_len.data_ptr(),
                                 lam_k.data_ptr(), s_k.data_ptr(), lam_v.data_ptr(), s_v.data_ptr(),
                                 B, Hq, Hkv, T, D, group, _ex_flags(lambda_after, srft),
                                 float(sm_scale), out.data_ptr(), ws, wsb, _stream_handle(stream))
    if rc != KVQ_OK:
        raise KvqError(rc)
    return out


def dequantize(packed: torch.Tensor, scales: torch.Tensor, lam: torch.Tensor,
               signs: torch.Tensor, group: int, out: torch.Tensor | None = None,
               stream=None, tensor_cores: bool = False) -> torch.Tensor:
    """(packed uint8 [n, D/2], scales fp16 [n, D/group]) -> fp16 [n, D].
    ``tensor_cores``: run kvq_dequantize_tc (the in-group Hadamard on the
    tensor cores; D = 128, group 16/32/64), bit-identical."""
    if packed.dim() != 2:
        raise ValueError("packed must be [n_vec, D/2]")
    n, D = packed.shape[0], packed.shape[1] * 2
    _need(packed, torch.uint8, (n, D // 2), "packed")
    _need(scales, torch.float16, (n, max(D // group, 1)), "scales")
    _need(lam, torch.float32, (D,), "lambda")
    _need(signs, torch.int8, (D,), "signs")
    if out is None:
        out = torch.empty((n, D), dtype=torch.float16, device=packed.device)
    _need(out, torch.float16, (n, D), "out")
    fn = kvq_dequantize_tc if tensor_cores else kvq_dequantize
    rc = fn(packed.data_ptr(), scales.data_ptr(), lam.data_ptr(),
            signs.data_ptr(), n, D, group, out.data_ptr(),
            _stream_handle(stream))
    if rc != KVQ_OK:
        raise KvqError(rc)
    return out
