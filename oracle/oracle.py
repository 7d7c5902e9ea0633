"""ctypes wrapper over the C oracle (oracle/ck_oracle.c) -- test infrastructure only.

Arguments are CPU torch tensors (strided views allowed for x) or numpy arrays;
results are numpy arrays, with 16-bit outputs returned as torch tensors of that dtype.
"""
from __future__ import annotations

import ctypes
import threading

import numpy as np
import torch

from . import build as _build

__all__ = ["lib", "round_to", "decode", "rotate", "quantize", "rotate_quant", "pack_w4",
           "unpack_w4", "gemm_s32", "epilogue", "linear", "quantize_int8", "rotate_quant_int8",
           "linear_w8a8", "philox4x32_10", "quantize_packed", "DT"]

DT = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
DT_NAME = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}

_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_U64 = ctypes.c_uint64

_SIGS = {
    "ck_oracle_round": [_P, _I64, _I],
    "ck_oracle_decode": [_P, _I, _I64, _P],
    "ck_oracle_encode": [_P, _I, _I64, _P],
    "ck_oracle_rotate": [_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _I64, _P],
    "ck_oracle_quantize": [_P, _I64, _I64, _P, _P, _P],
    "ck_oracle_rotate_quant": [_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _P, _I64, _P, _P],
    "ck_oracle_pack_w4": [_P, _I64, _I64, _P],
    "ck_oracle_unpack_w4": [_P, _I64, _I64, _I64, _P],
    "ck_oracle_gemm_s32": [_P, _I64, _P, _I64, _I64, _P],
    "ck_oracle_epilogue": [_P, _I64, _I64, _P, _P, _P, _I, _P, _I],
    "ck_oracle_linear": [_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _I64, _I64, _P, _P, _I, _I,
                         _P, _I64, _P, _I64, _P, _P, _P],
    "ck_oracle_quantize_int8": [_P, _I64, _I64, _P, _P, _P],
    "ck_oracle_rotate_quant_int8": [_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _P, _I64, _P, _P],
    "ck_oracle_linear_w8a8": [_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _I64, _I64, _P, _P, _I,
                              _I, _P, _I64, _P, _I64, _P, _P, _P],
    "ck_oracle_philox4x32_10": [_P, _P, _P],
    "ck_oracle_quantize_packed": [_P, _I64, _I64, _P, _I, _U64, _U64, _P, _P, _P],
}


class OracleError(RuntimeError):
    pass


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            for name, args in _SIGS.items():
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = ctypes.c_int
            _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with {rc}")


def _ptr(a) -> int | None:
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        return a.data_ptr()
    return a.ctypes.data


def _dtcode(t: torch.Tensor) -> int:
    return DT[t.dtype]


def _rows(rows, M: int) -> np.ndarray:
    if rows is None:
        return np.arange(M, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def round_to(v, dtype: torch.dtype) -> np.ndarray:
    """Round float64 values to the nearest value of ``dtype`` (returned as float64)."""
    a = np.array(v, dtype=np.float64, copy=True).reshape(-1)
    _check(lib().ck_oracle_round(_ptr(a), a.size, DT[dtype]), "round")
    return a.reshape(np.shape(v))


def decode(t: torch.Tensor) -> np.ndarray:
    t = t.contiguous()
    out = np.empty(t.numel(), dtype=np.float64)
    _check(lib().ck_oracle_decode(_ptr(t), _dtcode(t), t.numel(), _ptr(out)), "decode")
    return out.reshape(tuple(t.shape))


def rotate(x: torch.Tensor, R: torch.Tensor, g: int, rows=None) -> np.ndarray:
    M, K = x.shape
    r = _rows(rows, M)
    y = np.empty((r.size, K), dtype=np.float64)
    Rc = R.contiguous()
    _check(lib().ck_oracle_rotate(_ptr(x), _dtcode(x), M, K, x.stride(0), x.stride(1), _ptr(Rc),
                                  g, _ptr(r), r.size, _ptr(y)), "rotate")
    return y


def quantize(y: np.ndarray, scale_in: float | None = None):
    y = np.ascontiguousarray(y, dtype=np.float64)
    n, K = y.shape
    codes = np.empty((n, K), dtype=np.int8)
    scales = np.empty(n, dtype=np.float32)
    s_in = None if scale_in is None else np.array([scale_in], dtype=np.float32)
    _check(lib().ck_oracle_quantize(_ptr(y), n, K, _ptr(s_in), _ptr(codes), _ptr(scales)),
           "quantize")
    return codes, scales


def rotate_quant(x: torch.Tensor, R: torch.Tensor, g: int, scale_in: float | None = None,
                 rows=None):
    M, K = x.shape
    r = _rows(rows, M)
    codes = np.empty((r.size, K), dtype=np.int8)
    scales = np.empty(r.size, dtype=np.float32)
    s_in = None if scale_in is None else np.array([scale_in], dtype=np.float32)
    Rc = R.contiguous()
    _check(lib().ck_oracle_rotate_quant(_ptr(x), _dtcode(x), M, K, x.stride(0), x.stride(1),
                                        _ptr(Rc), g, _ptr(s_in), _ptr(r), r.size, _ptr(codes),
                                        _ptr(scales)), "rotate_quant")
    return codes, scales


def pack_w4(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.int8)
    N, K = w.shape
    out = np.empty((N, K // 2), dtype=np.int8)
    _check(lib().ck_oracle_pack_w4(_ptr(w), N, K, _ptr(out)), "pack_w4")
    return out


def unpack_w4(packed, K: int) -> np.ndarray:
    p = packed.numpy() if isinstance(packed, torch.Tensor) else np.asarray(packed)
    N = p.shape[0]
    ld = p.strides[0] if p.ndim == 2 else K // 2
    out = np.empty((N, K), dtype=np.int8)
    _check(lib().ck_oracle_unpack_w4(_ptr(p), N, K, ld, _ptr(out)), "unpack_w4")
    return out


def gemm_s32(q: np.ndarray, w: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    w = np.ascontiguousarray(w, dtype=np.int8)
    M, K = q.shape
    N = w.shape[0]
    acc = np.empty((M, N), dtype=np.int32)
    _check(lib().ck_oracle_gemm_s32(_ptr(q), M, _ptr(w), N, K, _ptr(acc)), "gemm_s32")
    return acc


def _out_tensor(shape, dtype: torch.dtype) -> torch.Tensor:
    return torch.empty(shape, dtype=dtype)


def epilogue(acc: np.ndarray, a_scale: np.ndarray, w_scale: torch.Tensor,
             bias: torch.Tensor | None, out_dtype: torch.dtype) -> torch.Tensor:
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    a_scale = np.ascontiguousarray(a_scale, dtype=np.float32)
    M, N = acc.shape
    ws = w_scale.contiguous()
    b = None if bias is None else bias.contiguous()
    out = _out_tensor((M, N), out_dtype)
    _check(lib().ck_oracle_epilogue(_ptr(acc), M, N, _ptr(a_scale), _ptr(ws), _ptr(b),
                                    _dtcode(ws), _ptr(out), DT[out_dtype]), "epilogue")
    return out


def linear(x: torch.Tensor, R: torch.Tensor, g: int, w_packed: torch.Tensor,
           w_scale: torch.Tensor, bias: torch.Tensor | None, rows=None, cols=None,
           out_dtype: torch.dtype | None = None):
    """Whole linear on the listed rows/cols; returns (out, codes, scales)."""
    M, K = x.shape
    N = w_packed.shape[0]
    r = _rows(rows, M)
    c = _rows(cols, N)
    out_dtype = out_dtype or x.dtype
    out = _out_tensor((r.size, c.size), out_dtype)
    codes = np.empty((r.size, K), dtype=np.int8)
    scales = np.empty(r.size, dtype=np.float32)
    ws = w_scale.contiguous()
    b = None if bias is None else bias.contiguous()
    Rc = R.contiguous()
    _check(lib().ck_oracle_linear(_ptr(x), _dtcode(x), M, K, x.stride(0), x.stride(1), _ptr(Rc),
                                  g, _ptr(w_packed), N, w_packed.stride(0), _ptr(ws), _ptr(b),
                                  _dtcode(ws), DT[out_dtype], _ptr(r), r.size, _ptr(c), c.size,
                                  _ptr(out), _ptr(codes), _ptr(scales)), "linear")
    return out, codes, scales


# ---------------------------------------------------------------- W8A8 variant

def quantize_int8(y: np.ndarray, scale_in: float | None = None):
    y = np.ascontiguousarray(y, dtype=np.float64)
    n, K = y.shape
    codes = np.empty((n, K), dtype=np.int8)
    scales = np.empty(n, dtype=np.float32)
    s_in = None if scale_in is None else np.array([scale_in], dtype=np.float32)
    _check(lib().ck_oracle_quantize_int8(_ptr(y), n, K, _ptr(s_in), _ptr(codes), _ptr(scales)),
           "quantize_int8")
    return codes, scales


def rotate_quant_int8(x: torch.Tensor, R: torch.Tensor, g: int, scale_in: float | None = None,
                      rows=None):
    M, K = x.shape
    r = _rows(rows, M)
    codes = np.empty((r.size, K), dtype=np.int8)
    scales = np.empty(r.size, dtype=np.float32)
    s_in = None if scale_in is None else np.array([scale_in], dtype=np.float32)
    Rc = R.contiguous()
    _check(lib().ck_oracle_rotate_quant_int8(_ptr(x), _dtcode(x), M, K, x.stride(0), x.stride(1),
                                             _ptr(Rc), g, _ptr(s_in), _ptr(r), r.size,
                                             _ptr(codes), _ptr(scales)), "rotate_quant_int8")
    return codes, scales


def linear_w8a8(x: torch.Tensor, R: torch.Tensor, g: int, w: torch.Tensor, w_scale: torch.Tensor,
                bias: torch.Tensor | None, rows=None, cols=None, out_dtype=None):
    """W8A8 linear (INT8 codes, INT8 weights (N, K)); returns (out, codes, scales)."""
    M, K = x.shape
    N = w.shape[0]
    r = _rows(rows, M)
    c = _rows(cols, N)
    out_dtype = out_dtype or x.dtype
    out = _out_tensor((r.size, c.size), out_dtype)
    codes = np.empty((r.size, K), dtype=np.int8)
    scales = np.empty(r.size, dtype=np.float32)
    ws = w_scale.contiguous()
    b = None if bias is None else bias.contiguous()
    Rc = R.contiguous()
    _check(lib().ck_oracle_linear_w8a8(_ptr(x), _dtcode(x), M, K, x.stride(0), x.stride(1),
                                       _ptr(Rc), g, _ptr(w), N, w.stride(0), _ptr(ws), _ptr(b),
                                       _dtcode(ws), DT[out_dtype], _ptr(r), r.size, _ptr(c),
                                       c.size, _ptr(out), _ptr(codes), _ptr(scales)),
           "linear_w8a8")
    return out, codes, scales


# ---------------------------------------------------------------- packed quantizer

def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.empty(4, dtype=np.uint32)
    _check(lib().ck_oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out)), "philox4x32_10")
    return out


def quantize_packed(y: np.ndarray, rows, K: int, scale_in: float | None = None,
                    stochastic: bool = False, seed: int = 0, offset: int = 0):
    """Nibble-packed signed-INT4 codes of the rotated rows y (listed by their row index in the
    (M, K) tensor, which the stochastic rounding's counter uses); returns (packed, scales)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    n = y.shape[0]
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    packed = np.empty((n, K // 2), dtype=np.uint8)
    scales = np.empty(n, dtype=np.float32)
    s_in = None if scale_in is None else np.array([scale_in], dtype=np.float32)
    _check(lib().ck_oracle_quantize_packed(_ptr(y), n, K, _ptr(s_in), 1 if stochastic else 0,
                                           seed, offset, _ptr(r), _ptr(packed), _ptr(scales)),
           "quantize_packed")
    return packed, scales
