"""Thin Python binding over libck.so (include/ck.h): argument marshalling only.

Each function takes CUDA torch tensors, passes their device pointers, sizes and
strides to the C entry point of the same name, and raises CkError on a non-OK
status.  Every step of the computation runs in the library's CUDA kernels; there is
no CPU path.  Loading fails loudly if libck.so has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libck.so")

CK_OK, CK_ERR_INVALID_ARG, CK_ERR_UNSUPPORTED, CK_ERR_OVERFLOW = 0, 1, 2, 3
CK_ERR_WORKSPACE, CK_ERR_CUDA, CK_ERR_TIMEOUT = 4, 5, 6
CK_F32, CK_F16, CK_BF16, CK_I8 = 0, 1, 2, 3

DTYPE_CODE = {torch.float32: CK_F32, torch.float16: CK_F16, torch.bfloat16: CK_BF16,
              torch.int8: CK_I8}
CODE_DTYPE = {v: k for k, v in DTYPE_CODE.items()}

# every entry point include/ck.h declares, with its ctypes signature
_P, _I64, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "ck_rotate_quant": ([_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _P, _I64, _P, _P, _P], _I),
    "ck_w4a4_linear": ([_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _P, _I64, _I64, _P, _I, _P,
                        _P, _I, _I64, _P, _SZ, _P, _P], _I),
    "ck_w4a4_linear_workspace_bytes": ([_I64, _I64, _I64, _I64], _SZ),
    "ck_workspace_codes_pitch": ([_I64], _I64),
    "ck_workspace_scales_offset": ([_I64, _I64], _SZ),
    "ck_w4a4_linear_noalloc": ([_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _P, _I64, _I64, _P,
                                _I, _P, _P, _I, _I64, _P, _P], _I),
    "ck_w4a4_grouped_linear": ([_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _P, _I64, _P, _I, _P,
                                _I, _P, _P, _P, _I, _P, _SZ, _P, _P], _I),
    "ck_unpack_w4": ([_P, _I64, _I64, _I64, _P, _I64, _P], _I),
    "ck_rotate_quant_int8": ([_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _P, _I64, _P, _P, _P],
                             _I),
    "ck_w8a8_linear": ([_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _P, _I64, _I64, _P, _I, _P,
                        _P, _I, _I64, _P, _SZ, _P, _P], _I),
    "ck_w8a8_linear_workspace_bytes": ([_I64, _I64, _I64, _I64], _SZ),
    "ck_rotate_quant_packed": ([_P, _I, _I64, _I64, _I64, _I64, _P, _I, _P, _I, ctypes.c_uint64,
                                ctypes.c_uint64, _P, _I64, _P, _P], _I),
    "ck_status_string": ([_I], ctypes.c_char_p),
}


class CkError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def load_library(path: str) -> ctypes.CDLL:
    """Load a build of the library at `path` with every entry point's ctypes signature set."""
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not found at {path}; run "
                          "`python -m rotated_w4a4_quantized_group_b200.build`")
    L = ctypes.CDLL(path)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


def lib() -> ctypes.CDLL:
    """Load libck.so (raises if it is missing: build it with the package's build module)."""
    global _lib
    if _lib is None:
        _lib = load_library(LIB_PATH)
    return _lib


def status_string(status: int) -> str:
    return lib().ck_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != CK_OK:
        raise CkError(status, where)


def _stream(stream) -> int | None:
    """The caller's stream, or torch's current stream of the current device (every entry
    point makes its tensors' device current before asking)."""
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t) -> int | None:
    """Device address of a tensor argument (None stays NULL, an int is taken as an address).
    A tensor outside GPU memory is refused here: the library would hand its host address to
    the device."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError(f"ck: tensor arguments must live on a CUDA device, got one on {t.device}")
    return t.data_ptr()


def workspace_bytes(M: int, N: int, K: int, w_ld: int) -> int:
    return int(lib().ck_w4a4_linear_workspace_bytes(M, N, K, w_ld))


def workspace_codes_pitch(K: int) -> int:
    return int(lib().ck_workspace_codes_pitch(K))


def workspace_scales_offset(M: int, K: int) -> int:
    return int(lib().ck_workspace_scales_offset(M, K))


def _check_rotation(x: torch.Tensor, R: torch.Tensor, g: int):
    # the C ABI reads R as g*g row-major elements of x's dtype
    if tuple(R.shape) != (g, g) or R.dtype != x.dtype or not R.is_contiguous():
        raise ValueError(f"R must be a contiguous ({g}, {g}) tensor of {x.dtype}; got "
                         f"{tuple(R.shape)} {R.dtype} strides {R.stride()}")


def ck_rotate_quant(x: torch.Tensor, R: torch.Tensor, g: int, scale_in: torch.Tensor | None = None,
                    codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None, stream=None):
    """Stage 1 on a 2-D (M, K) CUDA view; returns (codes int8 (M, K), scales fp32 (M,))."""
    M, K = x.shape
    _check_rotation(x, R, g)
    _same_device(x, R, scale_in, codes, scales, dev_status)
    if codes is None:
        codes = torch.empty(M, K, dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(M, dtype=torch.float32, device=x.device)
    if codes.dtype != torch.int8 or tuple(codes.shape) != (M, K) or codes.stride(1) != 1:
        raise ValueError(f"codes must be an int8 ({M}, {K}) view with unit inner stride")
    if scales.dtype != torch.float32 or scales.numel() < M or not scales.is_contiguous():
        raise ValueError(f"scales must be a contiguous fp32 tensor of at least {M} values")
    with torch.cuda.device(x.device):
        st = lib().ck_rotate_quant(_ptr(x), DTYPE_CODE[x.dtype], M, K, x.stride(0), x.stride(1),
                                   _ptr(R), g, _ptr(scale_in), _ptr(codes), codes.stride(0),
                                   _ptr(scales), _ptr(dev_status), _stream(stream))
    _check(st, "ck_rotate_quant")
    return codes, scales


def _check_weights(w_packed: torch.Tensor, N: int, K: int):
    # the library reads N rows of K/2 bytes through the row pitch w_packed.stride(0)
    if w_packed.dtype != torch.int8 or w_packed.dim() != 2 or w_packed.stride(1) != 1 or \
            tuple(w_packed.shape) != (N, K // 2):
        raise ValueError(f"w_packed must be an int8 (N, K/2) = ({N}, {K // 2}) view with unit inner "
                         f"stride; got {tuple(w_packed.shape)} {w_packed.dtype} strides "
                         f"{w_packed.stride()}")


def _check_out(out: torch.Tensor, M: int, N: int, x: torch.Tensor):
    # the library writes M rows of N values through the row pitch out.stride(0)
    if tuple(out.shape) != (M, N) or out.stride(1) != 1 or out.device != x.device:
        raise ValueError(f"out must be an (M, N) = ({M}, {N}) view with unit inner stride on "
                         f"{x.device}; got {tuple(out.shape)} strides {out.stride()} on {out.device}")


def _same_device(x: torch.Tensor, *ts):
    """Every tensor argument on x's CUDA device (a host tensor's address would be read by the
    device; a tensor on another GPU would be read through the wrong device's memory)."""
    _ptr(x)
    for t in ts:
        if t is not None and not isinstance(t, int) and t.device != x.device:
            raise ValueError(f"every tensor must be on {x.device}; got one on {t.device}")


def ck_w4a4_linear(x: torch.Tensor, R: torch.Tensor | None, g: int, w_packed: torch.Tensor,
                   w_scale: torch.Tensor, bias: torch.Tensor | None = None, *,
                   a_scale: torch.Tensor | None = None, out: torch.Tensor | None = None,
                   out_dtype: torch.dtype | None = None, workspace: torch.Tensor | None = None,
                   dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The whole W4A4 linear.  x is (M, K) activations (fp32/fp16/bf16) or int8 codes (with
    a_scale); w_packed is (N, K/2) int8.  Returns out (M, N)."""
    M, K = x.shape
    N = w_packed.shape[0]
    if x.dtype != torch.int8:
        _check_rotation(x, R, g)
    _check_weights(w_packed, N, K)
    _same_device(x, R, w_packed, w_scale, bias, a_scale, workspace, dev_status)
    if out is None:
        odt = out_dtype or (x.dtype if x.dtype != torch.int8 else w_scale.dtype)
        out = torch.empty(M, N, dtype=odt, device=x.device)
    _check_out(out, M, N, x)
    with torch.cuda.device(x.device):
        if workspace is None:
            nbytes = workspace_bytes(M, N, K, w_packed.stride(0))
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
        st = lib().ck_w4a4_linear(
            _ptr(x), DTYPE_CODE[x.dtype], M, K, x.stride(0), x.stride(1), _ptr(R), int(g),
            _ptr(a_scale), _ptr(w_packed), N, w_packed.stride(0), _ptr(w_scale),
            DTYPE_CODE[w_scale.dtype], _ptr(bias), _ptr(out), DTYPE_CODE[out.dtype],
            out.stride(0), _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream))
    _check(st, "ck_w4a4_linear")
    return out


def ck_w4a4_linear_noalloc(x: torch.Tensor, R: torch.Tensor | None, g: int,
                           w_packed: torch.Tensor, w_scale: torch.Tensor,
                           bias: torch.Tensor | None = None, *, out: torch.Tensor,
                           a_scale: torch.Tensor | None = None,
                           dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """ck_w4a4_linear with the library's built-in 32 MiB scratch instead of a workspace, for
    callers that cannot allocate device memory; `out` must be given (nothing is allocated)."""
    M, K = x.shape
    N = w_packed.shape[0]
    if x.dtype != torch.int8:
        _check_rotation(x, R, g)
    _check_weights(w_packed, N, K)
    _same_device(x, R, w_packed, w_scale, bias, a_scale, dev_status)
    _check_out(out, M, N, x)
    with torch.cuda.device(x.device):
        st = lib().ck_w4a4_linear_noalloc(
            _ptr(x), DTYPE_CODE[x.dtype], M, K, x.stride(0), x.stride(1), _ptr(R), int(g),
            _ptr(a_scale), _ptr(w_packed), N, w_packed.stride(0), _ptr(w_scale),
            DTYPE_CODE[w_scale.dtype], _ptr(bias), _ptr(out), DTYPE_CODE[out.dtype],
            out.stride(0), _ptr(dev_status), _stream(stream))
    _check(st, "ck_w4a4_linear_noalloc")
    return out


def fuse_linear_weights(parts):
    """Stack the packed weights, weight scales and biases of several linears that share one
    input along N (one-time weight preparation, done on the device by torch): parts is a list
    of (w_packed (N_i, K/2) int8, w_scale (N_i,), bias (N_i,) or None).  Returns
    (w_packed (N, K/2), w_scale (N,), bias (N,) or None, [N_i]); biases that are None become
    zeros when another part has one."""
    if not parts:
        raise ValueError("fuse_linear_weights needs at least one linear")
    ws = torch.cat([p[0] for p in parts], 0).contiguous()
    sc = torch.cat([p[1] for p in parts], 0).contiguous()
    if all(p[2] is None for p in parts):
        bias = None
    else:
        bias = torch.cat([p[2] if p[2] is not None else torch.zeros_like(p[1]) for p in parts],
                         0).contiguous()
    return ws, sc, bias, [int(p[0].shape[0]) for p in parts]


def ck_w4a4_grouped_linear(x: torch.Tensor, R: torch.Tensor | None, g: int,
                           w_packed: torch.Tensor, w_scale: torch.Tensor,
                           bias: torch.Tensor | None, group_n, *, outs=None,
                           a_scale: torch.Tensor | None = None,
                           out_dtype: torch.dtype | None = None,
                           workspace: torch.Tensor | None = None,
                           dev_status: torch.Tensor | None = None, stream=None):
    """Several linears sharing x as one call: w_packed/w_scale/bias are the groups' weights
    stacked along N (fuse_linear_weights), group_n the channels of each group.  Returns the
    list of per-group outputs (M, N_i)."""
    M, K = x.shape
    N = int(sum(group_n))
    if x.dtype != torch.int8:
        _check_rotation(x, R, g)
    _check_weights(w_packed, N, K)
    _same_device(x, R, w_packed, w_scale, bias, a_scale, workspace, dev_status)
    odt = out_dtype or (x.dtype if x.dtype != torch.int8 else w_scale.dtype)
    if outs is None:
        outs = [torch.empty(M, int(n), dtype=odt, device=x.device) for n in group_n]
    if len(outs) != len(group_n):
        raise ValueError("one output per group")
    for o, n in zip(outs, group_n):
        _check_out(o, M, int(n), x)
        if o.dtype != outs[0].dtype:
            raise ValueError("every group's output has the same dtype")
    G = len(group_n)
    gn = (ctypes.c_int64 * G)(*[int(n) for n in group_n])
    ptrs = (ctypes.c_void_p * G)(*[o.data_ptr() for o in outs])
    ldos = (ctypes.c_int64 * G)(*[o.stride(0) for o in outs])
    with torch.cuda.device(x.device):
        if workspace is None:
            nbytes = workspace_bytes(M, N, K, w_packed.stride(0))
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
        st = lib().ck_w4a4_grouped_linear(
            _ptr(x), DTYPE_CODE[x.dtype], M, K, x.stride(0), x.stride(1), _ptr(R), int(g),
            _ptr(a_scale), _ptr(w_packed), w_packed.stride(0), _ptr(w_scale),
            DTYPE_CODE[w_scale.dtype], _ptr(bias), G, gn, ptrs, ldos, DTYPE_CODE[outs[0].dtype],
            _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream))
    _check(st, "ck_w4a4_grouped_linear")
    return outs


def ck_rotate_quant_int8(x: torch.Tensor, R: torch.Tensor, g: int,
                         scale_in: torch.Tensor | None = None, codes: torch.Tensor | None = None,
                         scales: torch.Tensor | None = None,
                         dev_status: torch.Tensor | None = None, stream=None):
    """The W8A8 variant's stage 1: INT8 codes (qmax 127) and fp32 row scales of a 2-D view."""
    M, K = x.shape
    _check_rotation(x, R, g)
    _same_device(x, R, scale_in, codes, scales, dev_status)
    if codes is None:
        codes = torch.empty(M, K, dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(M, dtype=torch.float32, device=x.device)
    if codes.dtype != torch.int8 or tuple(codes.shape) != (M, K) or codes.stride(1) != 1:
        raise ValueError(f"codes must be an int8 ({M}, {K}) view with unit inner stride")
    if scales.dtype != torch.float32 or scales.numel() < M or not scales.is_contiguous():
        raise ValueError(f"scales must be a contiguous fp32 tensor of at least {M} values")
    with torch.cuda.device(x.device):
        st = lib().ck_rotate_quant_int8(_ptr(x), DTYPE_CODE[x.dtype], M, K, x.stride(0),
                                        x.stride(1), _ptr(R), g, _ptr(scale_in), _ptr(codes),
                                        codes.stride(0), _ptr(scales), _ptr(dev_status),
                                        _stream(stream))
    _check(st, "ck_rotate_quant_int8")
    return codes, scales


def ck_w8a8_linear(x: torch.Tensor, R: torch.Tensor | None, g: int, w: torch.Tensor,
                   w_scale: torch.Tensor, bias: torch.Tensor | None = None, *,
                   a_scale: torch.Tensor | None = None, out: torch.Tensor | None = None,
                   out_dtype: torch.dtype | None = None, workspace: torch.Tensor | None = None,
                   dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The W8A8 linear: x (M, K) activations (or INT8 codes with a_scale), w (N, K) int8."""
    M, K = x.shape
    N = w.shape[0]
    if x.dtype != torch.int8:
        _check_rotation(x, R, g)
    if w.dtype != torch.int8 or w.dim() != 2 or w.stride(1) != 1 or tuple(w.shape) != (N, K):
        raise ValueError(f"w must be an int8 (N, K) = ({N}, {K}) view with unit inner stride")
    _same_device(x, R, w, w_scale, bias, a_scale, workspace, dev_status)
    if out is None:
        odt = out_dtype or (x.dtype if x.dtype != torch.int8 else w_scale.dtype)
        out = torch.empty(M, N, dtype=odt, device=x.device)
    _check_out(out, M, N, x)
    with torch.cuda.device(x.device):
        if workspace is None:
            nbytes = int(lib().ck_w8a8_linear_workspace_bytes(M, N, K, w.stride(0)))
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
        st = lib().ck_w8a8_linear(
            _ptr(x), DTYPE_CODE[x.dtype], M, K, x.stride(0), x.stride(1), _ptr(R), int(g),
            _ptr(a_scale), _ptr(w), N, w.stride(0), _ptr(w_scale), DTYPE_CODE[w_scale.dtype],
            _ptr(bias), _ptr(out), DTYPE_CODE[out.dtype], out.stride(0), _ptr(workspace),
            workspace.numel(), _ptr(dev_status), _stream(stream))
    _check(st, "ck_w8a8_linear")
    return out


def ck_rotate_quant_packed(x: torch.Tensor, R: torch.Tensor, g: int, *, stochastic: bool = False,
                           seed: int = 0, offset: int = 0, scale_in: torch.Tensor | None = None,
                           packed: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                           stream=None):
    """The public packed quantizer: (packed uint8 (M, K/2), scales fp32 (M,)); stochastic
    rounding draws from Philox4x32-10 keyed by seed at counter (element index, offset)."""
    M, K = x.shape
    _check_rotation(x, R, g)
    _same_device(x, R, scale_in, packed, scales)
    if packed is None:
        packed = torch.empty(M, K // 2, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(M, dtype=torch.float32, device=x.device)
    if packed.dtype != torch.uint8 or tuple(packed.shape) != (M, K // 2) or packed.stride(1) != 1:
        raise ValueError(f"packed must be a uint8 ({M}, {K // 2}) view with unit inner stride")
    with torch.cuda.device(x.device):
        st = lib().ck_rotate_quant_packed(_ptr(x), DTYPE_CODE[x.dtype], M, K, x.stride(0),
                                          x.stride(1), _ptr(R), g, _ptr(scale_in),
                                          1 if stochastic else 0, seed & (2 ** 64 - 1),
                                          offset & (2 ** 64 - 1), _ptr(packed), packed.stride(0),
                                          _ptr(scales), _stream(stream))
    _check(st, "ck_rotate_quant_packed")
    return packed, scales


def ck_unpack_w4(packed: torch.Tensor, K: int, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """(N, K/2) packed int8 -> (N, K) int8 codes."""
    N = packed.shape[0]
    if out is None:
        out = torch.empty(N, K, dtype=torch.int8, device=packed.device)
    if packed.dim() != 2 or packed.stride(1) != 1 or packed.shape[1] < K // 2 or \
            out.dim() != 2 or out.stride(1) != 1 or tuple(out.shape) != (N, K):
        raise ValueError("ck_unpack_w4: packed must be (N, >= K/2) and out (N, K), unit inner strides")
    _same_device(packed, out)
    with torch.cuda.device(packed.device):
        st = lib().ck_unpack_w4(_ptr(packed), N, K, packed.stride(0), _ptr(out), out.stride(0),
                                _stream(stream))
    _check(st, "ck_unpack_w4")
    return out
