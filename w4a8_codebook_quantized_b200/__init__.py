"""ConvRot W4A8 codebook linear layer forward on NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/cr_w4a8.h``
(``libcr_w4a8.so``, built in-tree by ``w4a8_codebook_quantized_b200.build``).
The functions carry the C names and only marshal arguments: they take torch
CUDA tensors, pass their device pointers and the current CUDA stream, and
raise ``CrError`` on a non-OK status.  All arithmetic runs in the library's
kernels; there is no other implementation to fall back to, and a missing
library or GPU raises.

Storage of one layer (ai-toolkit convrot_w4a8_quant.py, module docstring):
    qdata     uint8/int8 [N, K/2]   packed 4-bit codes, even column = low nibble
    srel      uint8      [N, K/16]  fp8 e4m3fn group scales (byte view)
    s_channel float32    [N]        per-output-channel scale
    codebook  float32    [16]       codebook levels
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

__all__ = [
    "W4A8Linear",
    "CrError", "lib", "library_path",
    "cr_rotate_quant_act", "cr_w4a8_decode_int8", "cr_w4a8_gemm", "cr_w4a8_gemv",
    "cr_epilogue", "cr_w4a8_linear", "cr_w4a8_linear_decode_noalloc", "cr_check_device_error",
    "cr_w4a8_gemv_grouped", "cr_w4a8_linear_grouped", "CrLayer",
    "cr_w4a8_gemm_swiglu", "cr_w4a8_gemv_swiglu", "cr_w4a8_linear_swiglu", "cr_interleave_rows",
    "interleave_gate_up", "cr_w4a8_quantize_rotated", "cr_w4a8_assign_codes",
    "cr_w4a8_ste_backward", "cr_w4a8_dequant_t_bf16", "cr_selftest_wait_timeout", "cr_gemm_s8",
    "cr_w4a8_gemm_ws", "cr_w4a8_linear_ws", "cr_w4a8_ste_backward_ws", "cr_mma_i8_peak",
    "cr_status_string", "cr_version",
    "gemv_rows",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libcr_w4a8.so")

CR_OK, CR_ERR_INVALID_ARG, CR_ERR_UNSUPPORTED, CR_ERR_ALIGNMENT, CR_ERR_CUDA, CR_ERR_TIMEOUT, CR_ERR_NO_DEVICE = range(7)
CR_OUT_BF16, CR_OUT_F32 = 0, 1
CR_GEMV_MAX_M = 8
CR_MAX_LAYERS = 4


class CrLayer(ctypes.Structure):
    """cr_w4a8_layer: one layer of a grouped call (device pointers)."""
    _fields_ = [("qdata", ctypes.c_void_p), ("srel", ctypes.c_void_p), ("s_channel", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("N", ctypes.c_int64), ("out", ctypes.c_void_p),
                ("acc_out", ctypes.c_void_p)]

_lib = None
_lock = threading.Lock()


class CrError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {cr_status_string(status)} (status {status})")


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded C library with typed entry points (the raw C ABI)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise ImportError(
                    f"{_LIB_PATH} is missing: build it with `python -m w4a8_codebook_quantized_b200.build`")
            L = ctypes.CDLL(_LIB_PATH)
            P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            L.cr_status_string.argtypes = [i32]
            L.cr_status_string.restype = ctypes.c_char_p
            L.cr_version.argtypes = []
            L.cr_version.restype = ctypes.c_char_p
            L.cr_rotate_quant_act.argtypes = [P, i64, i64, i64, i32, P, P, P]
            L.cr_w4a8_decode_int8.argtypes = [P, P, P, i64, i64, P, P]
            contraction = [P, P, P, P, P, P, P, i64, i64, i64, i32, P, P, P]
            L.cr_w4a8_gemm.argtypes = contraction
            L.cr_w4a8_gemv.argtypes = contraction
            L.cr_epilogue.argtypes = [P, P, P, P, i64, i64, i32, P, P]
            L.cr_w4a8_linear.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, i32, P, P, P, P]
            L.cr_check_device_error.argtypes = [P]
            L.cr_w4a8_linear_decode_noalloc.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, i32, P, P]
            L.cr_w4a8_gemm_swiglu.argtypes = contraction[:-2] + [P]
            L.cr_w4a8_gemv_swiglu.argtypes = contraction[:-2] + [P]
            L.cr_w4a8_linear_swiglu.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, i32, P, P, P, P]
            L.cr_interleave_rows.argtypes = [P, P, i64, i64, P]
            L.cr_w4a8_quantize_rotated.argtypes = [P, P, i64, i64, P, P, P, P]
            L.cr_w4a8_assign_codes.argtypes = [P, P, P, P, P, i64, i64, P, P]
            L.cr_w4a8_ste_backward.argtypes = [P, P, P, P, P, i64, i64, i64, P, P]
            L.cr_w4a8_plan_create.argtypes = [P, P, P, P, P, i64, i64, i32, i32, ctypes.POINTER(P)]
            L.cr_w4a8_plan_forward.argtypes = [P, P, i64, P, P, P, P]
            L.cr_w4a8_plan_forward_host.argtypes = [P, P, i64, P, P, P, P, P, P]
            L.cr_w4a8_plan_gemv.argtypes = [P, P, P, i64, P, P]
            L.cr_w4a8_plan_destroy.argtypes = [P]
            L.cr_w4a8_plan_bind_host.argtypes = [P, P, i64, P, P, P, P, P, ctypes.POINTER(P)]
            L.cr_w4a8_host_call_run.argtypes = [P, P]
            L.cr_w4a8_host_call_destroy.argtypes = [P]
            L.cr_selftest_wait_timeout.argtypes = [ctypes.c_uint64, P]
            L.cr_gemm_s8.argtypes = [P, P, P, P, P, i64, i64, i64, i32, P, P, P]
            L.cr_w4a8_dequant_t_bf16.argtypes = [P, P, P, P, i64, i64, P, P]
            L.cr_w4a8_gemm_ws.argtypes = contraction[:-1] + [P, P]
            L.cr_mma_i8_peak.argtypes = [i64, ctypes.POINTER(ctypes.c_double), P]
            L.cr_w4a8_linear_ws.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, i32, P, P, P, P, P]
            L.cr_w4a8_ste_backward_ws.argtypes = [P, P, P, P, P, i64, i64, i64, P, P, P]
            LP = ctypes.POINTER(CrLayer)
            L.cr_w4a8_gemv_grouped.argtypes = [P, P, P, i64, i64, LP, i32, i32, P]
            L.cr_w4a8_linear_grouped.argtypes = [P, P, i64, i64, LP, i32, i32, i32, P, P, P]
            for name in ("cr_rotate_quant_act", "cr_w4a8_decode_int8", "cr_w4a8_gemm", "cr_w4a8_gemv",
                         "cr_epilogue", "cr_w4a8_linear", "cr_check_device_error",
                         "cr_w4a8_linear_decode_noalloc", "cr_w4a8_gemm_ws", "cr_w4a8_linear_ws",
                         "cr_w4a8_ste_backward_ws"):
                getattr(L, name).restype = i32
            _lib = L
    return _lib


def cr_status_string(status: int) -> str:
    return lib().cr_status_string(int(status)).decode()


def cr_version() -> str:
    return lib().cr_version().decode()


# ---------------------------------------------------------------- marshalling

def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        if raw is not None:  # the current stream's handle without building a Stream object
            return raw(torch.cuda.current_device())
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t, name, dtypes, ndim=None, shape=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _check(status: int, where: str) -> None:
    if status != CR_OK:
        raise CrError(status, where)


def _cuda_device_of(args, kwargs):
    """The one device of the CUDA tensors among the arguments (searched one
    level into lists and tuples), or None; ValueError when they differ."""
    torch = _torch()
    dev = None

    def visit(v, depth):
        nonlocal dev
        if isinstance(v, torch.Tensor):
            if v.is_cuda:
                if dev is None:
                    dev = v.device
                elif v.device != dev:
                    raise ValueError(f"CUDA tensors on different devices: {dev} and {v.device}")
        elif depth < 2 and isinstance(v, (list, tuple)):
            for e in v:
                visit(e, depth + 1)

    for a in args:
        visit(a, 0)
    for a in kwargs.values():
        visit(a, 0)
    return dev


def _on_device(fn):
    """Run an entry point with the device of its CUDA tensors current.

    The C library launches on the current device and the binding passes the
    current device's stream, so a call on tensors of another device must make
    that device current first; all CUDA tensor arguments must share it."""
    import functools

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        dev = _cuda_device_of(args, kwargs)
        torch = _torch()
        if dev is None or dev.index == torch.cuda.current_device():
            return fn(*args, **kwargs)
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)

    return wrapper


def _out_code(dtype) -> int:
    torch = _torch()
    if dtype == torch.bfloat16:
        return CR_OUT_BF16
    if dtype == torch.float32:
        return CR_OUT_F32
    raise TypeError(f"out dtype must be bfloat16 or float32, got {dtype}")


def gemv_rows(m: int) -> int:
    """Rows of the decode GEMV's padded activation operand: next power of two
    of M (ai-toolkit convrot_w4a8_quant.py, _gemv_mp)."""
    return 1 << max(0, (int(m) - 1).bit_length())


def _layer(qdata, srel, codebook, s_channel, bias):
    torch = _torch()
    _need(qdata, "qdata", (torch.uint8, torch.int8), 2)
    N, KH = qdata.shape
    K = 2 * KH
    _need(srel, "srel", (torch.uint8, torch.float8_e4m3fn), shape=(N, K // 16))
    _need(codebook, "codebook", (torch.float32,), shape=(16,))
    _need(s_channel, "s_channel", (torch.float32,), shape=(N,))
    if bias is not None:
        _need(bias, "bias", (torch.float32,), shape=(N,))
    return N, K


# ---------------------------------------------------------------- entry points

@_on_device
def cr_rotate_quant_act(x, mp: Optional[int] = None, act_qmax: int = 127, xq=None, xs=None,
                        stream=None) -> Tuple["torch.Tensor", "torch.Tensor"]:
    """x bf16 [M, K] -> (xq int8 [MP, K], xs fp32 [MP]); rows >= M are 0 / 1."""
    torch = _torch()
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    MP = M if mp is None else int(mp)
    if xq is None:
        xq = torch.empty(MP, K, dtype=torch.int8, device=x.device)
    if xs is None:
        xs = torch.empty(MP, dtype=torch.float32, device=x.device)
    _need(xq, "xq", (torch.int8,), shape=(MP, K))
    _need(xs, "xs", (torch.float32,), shape=(MP,))
    _check(lib().cr_rotate_quant_act(_ptr(x), M, K, MP, int(act_qmax), _ptr(xq), _ptr(xs), _stream(stream)),
           "cr_rotate_quant_act")
    return xq, xs


@_on_device
def cr_w4a8_decode_int8(qdata, srel, codebook, w8=None, stream=None):
    """Packed codes -> the int8 grid w8 [N, K]."""
    torch = _torch()
    _need(qdata, "qdata", (torch.uint8, torch.int8), 2)
    N, K = qdata.shape[0], qdata.shape[1] * 2
    _need(srel, "srel", (torch.uint8, torch.float8_e4m3fn), shape=(N, K // 16))
    _need(codebook, "codebook", (torch.float32,), shape=(16,))
    if w8 is None:
        w8 = torch.empty(N, K, dtype=torch.int8, device=qdata.device)
    _need(w8, "w8", (torch.int8,), shape=(N, K))
    _check(lib().cr_w4a8_decode_int8(_ptr(qdata), _ptr(srel), _ptr(codebook), N, K, _ptr(w8), _stream(stream)),
           "cr_w4a8_decode_int8")
    return w8


def _contraction(fn_name, xq, xs, qdata, srel, codebook, s_channel, bias, m, out_dtype, out, acc_out, stream,
                 w8_work=None):
    torch = _torch()
    N, K = _layer(qdata, srel, codebook, s_channel, bias)
    _need(xq, "xq", (torch.int8,), 2)
    _need(xs, "xs", (torch.float32,), 1)
    M = xq.shape[0] if m is None else int(m)
    if xq.shape[1] != K or xq.shape[0] < M or xs.shape[0] < M:
        raise ValueError(f"xq {tuple(xq.shape)} / xs {tuple(xs.shape)} do not match M={M}, K={K}")
    code = _out_code(out_dtype if out is None else out.dtype)
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=xq.device)
    _need(out, "out", (torch.bfloat16, torch.float32), shape=(M, N))
    if acc_out is True:
        acc_out = torch.empty(M, N, dtype=torch.int32, device=xq.device)
    if acc_out is not None and acc_out is not False:
        _need(acc_out, "acc_out", (torch.int32,), shape=(M, N))
    else:
        acc_out = None
    args = [_ptr(xq), _ptr(xs), _ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel), _ptr(bias),
            M, N, K, code, _ptr(out), _ptr(acc_out)]
    if w8_work is not None:
        _need(w8_work, "w8_work", (torch.int8,), shape=(N, K))
        fn_name = "cr_w4a8_gemm_ws"
        args.append(_ptr(w8_work))
    fn = getattr(lib(), fn_name)
    _check(fn(*args, _stream(stream)), fn_name)
    return (out, acc_out) if acc_out is not None else out


@_on_device
def cr_w4a8_gemm(xq, xs, qdata, srel, codebook, s_channel, bias=None, m: Optional[int] = None,
                 out_dtype=None, out=None, acc_out=None, stream=None, w8_work=None):
    """Prefill forward on quantised activations.  acc_out=True also returns the
    int32 accumulators (out, acc).  With w8_work (int8 [N, K]) the weight is
    decoded there (cr_w4a8_gemm_ws) and the library allocates nothing."""
    torch = _torch()
    return _contraction("cr_w4a8_gemm", xq, xs, qdata, srel, codebook, s_channel, bias, m,
                        out_dtype or torch.bfloat16, out, acc_out, stream, w8_work)


@_on_device
def cr_w4a8_gemm_ws(xq, xs, qdata, srel, codebook, s_channel, w8_work, bias=None, m: Optional[int] = None,
                    out_dtype=None, out=None, acc_out=None, stream=None):
    """cr_w4a8_gemm with the caller's weight transient w8_work int8 [N, K]."""
    torch = _torch()
    if w8_work is None:
        raise ValueError("w8_work is required")
    return _contraction("cr_w4a8_gemm_ws", xq, xs, qdata, srel, codebook, s_channel, bias, m,
                        out_dtype or torch.bfloat16, out, acc_out, stream, w8_work)


@_on_device
def cr_w4a8_gemv(xq, xs, qdata, srel, codebook, s_channel, bias=None, m: Optional[int] = None,
                 out_dtype=None, out=None, acc_out=None, stream=None):
    """Decode forward (M <= 8) on quantised activations; bitwise equal to cr_w4a8_gemm."""
    torch = _torch()
    return _contraction("cr_w4a8_gemv", xq, xs, qdata, srel, codebook, s_channel, bias, m,
                        out_dtype or torch.bfloat16, out, acc_out, stream)


@_on_device
def cr_gemm_s8(xq, xs, w8, s_channel, bias=None, m: Optional[int] = None, out_dtype=None, out=None, acc_out=None,
               stream=None):
    """The prefill contraction + epilogue on an int8 weight w8 [N, K] already
    on the grid (cr_w4a8_gemm without its decode); acc_out=True also returns
    the int32 accumulators."""
    torch = _torch()
    _need(w8, "w8", (torch.int8,), 2)
    N, K = w8.shape
    _need(s_channel, "s_channel", (torch.float32,), shape=(N,))
    if bias is not None:
        _need(bias, "bias", (torch.float32,), shape=(N,))
    _need(xq, "xq", (torch.int8,), 2)
    _need(xs, "xs", (torch.float32,), 1)
    M = xq.shape[0] if m is None else int(m)
    if xq.shape[1] != K or xq.shape[0] < M or xs.shape[0] < M:
        raise ValueError(f"xq {tuple(xq.shape)} / xs {tuple(xs.shape)} do not match M={M}, K={K}")
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype or torch.bfloat16, device=xq.device)
    _need(out, "out", (torch.bfloat16, torch.float32), shape=(M, N))
    if acc_out is True:
        acc_out = torch.empty(M, N, dtype=torch.int32, device=xq.device)
    if acc_out is not None and acc_out is not False:
        _need(acc_out, "acc_out", (torch.int32,), shape=(M, N))
    else:
        acc_out = None
    _check(lib().cr_gemm_s8(_ptr(xq), _ptr(xs), _ptr(w8), _ptr(s_channel), _ptr(bias), M, N, K,
                            _out_code(out.dtype), _ptr(out), _ptr(acc_out), _stream(stream)), "cr_gemm_s8")
    return (out, acc_out) if acc_out is not None else out


@_on_device
def cr_epilogue(acc, xs, s_channel, bias=None, out_dtype=None, out=None, stream=None):
    torch = _torch()
    _need(acc, "acc", (torch.int32,), 2)
    M, N = acc.shape
    _need(xs, "xs", (torch.float32,), 1)
    _need(s_channel, "s_channel", (torch.float32,), shape=(N,))
    if bias is not None:
        _need(bias, "bias", (torch.float32,), shape=(N,))
    out_dtype = out_dtype or torch.bfloat16
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=acc.device)
    _need(out, "out", (torch.bfloat16, torch.float32), shape=(M, N))
    if xs.shape[0] < M:
        raise ValueError("xs has fewer than M rows")
    _check(lib().cr_epilogue(_ptr(acc), _ptr(xs), _ptr(s_channel), _ptr(bias), M, N, _out_code(out.dtype),
                             _ptr(out), _stream(stream)), "cr_epilogue")
    return out


@_on_device
def cr_w4a8_linear(x, qdata, srel, codebook, s_channel, bias=None, act_qmax: int = 127, out_dtype=None,
                   out=None, xq_work=None, xs_work=None, stream=None, w8_work=None):
    """The whole layer forward: rotate + quantise x, then the decode GEMV when
    M <= 8, else the prefill GEMM.  With w8_work (int8 [N, K]) the prefill
    path decodes the weight there (cr_w4a8_linear_ws) instead of a transient
    of the library."""
    torch = _torch()
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    N, Kw = _layer(qdata, srel, codebook, s_channel, bias)
    if Kw != K:
        raise ValueError(f"x has K={K}, the layer K={Kw}")
    rows = gemv_rows(M) if 1 <= M <= CR_GEMV_MAX_M else M
    if xq_work is None:
        xq_work = torch.empty(rows, K, dtype=torch.int8, device=x.device)
    if xs_work is None:
        xs_work = torch.empty(rows, dtype=torch.float32, device=x.device)
    if xq_work.shape[0] < rows or xs_work.shape[0] < rows:
        raise ValueError(f"work buffers need {rows} rows")
    _need(xq_work, "xq_work", (torch.int8,), 2)
    _need(xs_work, "xs_work", (torch.float32,), 1)
    out_dtype = out_dtype or torch.bfloat16
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=x.device)
    _need(out, "out", (torch.bfloat16, torch.float32), shape=(M, N))
    args = [_ptr(x), _ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel), _ptr(bias), M, N, K, int(act_qmax),
            _out_code(out.dtype), _ptr(out), _ptr(xq_work), _ptr(xs_work)]
    if w8_work is not None:
        _need(w8_work, "w8_work", (torch.int8,), shape=(N, K))
        _check(lib().cr_w4a8_linear_ws(*args, _ptr(w8_work), _stream(stream)), "cr_w4a8_linear_ws")
    else:
        _check(lib().cr_w4a8_linear(*args, _stream(stream)), "cr_w4a8_linear")
    return out


@_on_device
def cr_w4a8_linear_ws(x, qdata, srel, codebook, s_channel, w8_work, bias=None, act_qmax: int = 127,
                      out_dtype=None, out=None, xq_work=None, xs_work=None, stream=None):
    """cr_w4a8_linear with the caller's weight transient w8_work int8 [N, K]
    (used when M > 8; may be None for M <= 8)."""
    torch = _torch()
    if w8_work is None:
        M = x.shape[0]
        if M > CR_GEMV_MAX_M:
            raise ValueError("w8_work is required when M > 8")
        return _linear_ws_decode(x, qdata, srel, codebook, s_channel, bias, act_qmax, out_dtype, out, xq_work,
                                 xs_work, stream)
    return cr_w4a8_linear(x, qdata, srel, codebook, s_channel, bias, act_qmax, out_dtype, out, xq_work, xs_work,
                          stream, w8_work=w8_work)


def _linear_ws_decode(x, qdata, srel, codebook, s_channel, bias, act_qmax, out_dtype, out, xq_work, xs_work,
                      stream):
    """cr_w4a8_linear_ws on the decode path (M <= 8), where no transient is used."""
    torch = _torch()
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    N, Kw = _layer(qdata, srel, codebook, s_channel, bias)
    if Kw != K:
        raise ValueError(f"x has K={K}, the layer K={Kw}")
    rows = gemv_rows(M) if M >= 1 else M
    if xq_work is None:
        xq_work = torch.empty(rows, K, dtype=torch.int8, device=x.device)
    if xs_work is None:
        xs_work = torch.empty(rows, dtype=torch.float32, device=x.device)
    _need(xq_work, "xq_work", (torch.int8,), 2)
    _need(xs_work, "xs_work", (torch.float32,), 1)
    if xq_work.shape[0] < rows or xs_work.shape[0] < rows:
        raise ValueError(f"work buffers need {rows} rows")
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype or torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16, torch.float32), shape=(M, N))
    _check(lib().cr_w4a8_linear_ws(_ptr(x), _ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel), _ptr(bias),
                                   M, N, K, int(act_qmax), _out_code(out.dtype), _ptr(out), _ptr(xq_work),
                                   _ptr(xs_work), None, _stream(stream)), "cr_w4a8_linear_ws")
    return out


class W4A8Linear:
    """A prepared layer for repeated forwards (cr_w4a8_plan_*).

    Holds qdata, srel, codebook, s_channel (and bias) as given (no copies) and
    a library plan over them: the layer is checked and the decode GEMV's
    weight maps are encoded once, here.  forward() checks only the
    activations, the output and the work buffers; forward_host() takes x and
    the output in host memory and queues both copies with the forward.  The
    caller must not resize or free the layer's tensors while the object is in
    use."""

    def __init__(self, qdata, srel, codebook, s_channel, bias=None, act_qmax: int = 127, out_dtype=None):
        torch = _torch()
        self.N, self.K = _layer(qdata, srel, codebook, s_channel, bias)
        if not 1 <= int(act_qmax) <= 127:
            raise ValueError("act_qmax must be in 1..127")
        self.act_qmax = int(act_qmax)
        self.out_dtype = out_dtype or torch.bfloat16
        self._tensors = (qdata, srel, codebook, s_channel, bias)  # keep them alive
        self.device = _cuda_device_of((qdata, srel, codebook, s_channel, bias), {})
        self._L = lib()
        handle = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(self._L.cr_w4a8_plan_create(_ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel),
                                               _ptr(bias), self.N, self.K, self.act_qmax, _out_code(self.out_dtype),
                                               ctypes.byref(handle)), "cr_w4a8_plan_create")
        self._plan = handle
        self._fwd = self._L.cr_w4a8_plan_forward
        self._fwd_host = self._L.cr_w4a8_plan_forward_host
        self._run_host = self._L.cr_w4a8_host_call_run
        # (tensors, their storage and shapes, bound call) of the last host forward
        # with caller-owned work buffers (cr_w4a8_plan_bind_host), and its lock
        self._host_args = None
        self._host_lock = threading.Lock()

    def __del__(self):
        self._drop_host_call()
        plan = getattr(self, "_plan", None)
        if plan is not None and plan.value:
            self._L.cr_w4a8_plan_destroy(plan)
            self._plan = None

    def _drop_host_call(self):
        hit = getattr(self, "_host_args", None)
        if hit is not None:
            self._host_args = None
            self._L.cr_w4a8_host_call_destroy(hit[2])

    def _work(self, x, M, xq_work, xs_work):
        torch = _torch()
        rows = gemv_rows(M) if 1 <= M <= CR_GEMV_MAX_M else M
        if xq_work is None:
            xq_work = torch.empty(rows, self.K, dtype=torch.int8, device=x.device)
        elif not xq_work.is_cuda or xq_work.dtype != torch.int8 or xq_work.dim() != 2 or xq_work.shape[0] < rows \
                or xq_work.shape[1] != self.K or not xq_work.is_contiguous():
            raise ValueError(f"xq_work must be a contiguous CUDA int8 [>= {rows}, {self.K}] tensor")
        if xs_work is None:
            xs_work = torch.empty(rows, dtype=torch.float32, device=x.device)
        elif not xs_work.is_cuda or xs_work.dtype != torch.float32 or xs_work.dim() != 1 or xs_work.shape[0] < rows:
            raise ValueError(f"xs_work must be a CUDA float32 [>= {rows}] tensor")
        return xq_work, xs_work

    def _device_ctx(self, *tensors):
        """The plan's device made current (the plan runs only there); every
        CUDA tensor given must be on it."""
        import contextlib
        torch = _torch()
        for t in tensors:
            if isinstance(t, torch.Tensor) and t.is_cuda and t.device != self.device:
                raise ValueError(f"tensor on {t.device}, the layer is on {self.device}")
        if torch.cuda.current_device() == self.device.index:
            return contextlib.nullcontext()
        return torch.cuda.device(self.device)

    def forward(self, x, out=None, xq_work=None, xs_work=None, stream=None):
        with self._device_ctx(x, out, xq_work, xs_work):
            return self._forward(x, out, xq_work, xs_work, stream)

    __call__ = forward

    def _forward(self, x, out, xq_work, xs_work, stream):
        torch = _torch()
        _need(x, "x", (torch.bfloat16,), 2)
        M, K = x.shape
        if K != self.K:
            raise ValueError(f"x has K={K}, the layer K={self.K}")
        xq_work, xs_work = self._work(x, M, xq_work, xs_work)
        if out is None:
            out = torch.empty(M, self.N, dtype=self.out_dtype, device=x.device)
        _need(out, "out", (self.out_dtype,), shape=(M, self.N))
        _check(self._fwd(self._plan, x.data_ptr(), M, out.data_ptr(), xq_work.data_ptr(), xs_work.data_ptr(),
                         _stream(stream)), "cr_w4a8_plan_forward")
        return out

    def gemv(self, xq, xs, m: Optional[int] = None, out=None, stream=None):
        """The decode GEMV on already quantised activations (xq int8 [>= M, K],
        xs fp32 [>= M], M <= 8): cr_w4a8_plan_gemv."""
        torch = _torch()
        _need(xq, "xq", (torch.int8,), 2)
        _need(xs, "xs", (torch.float32,), 1)
        M = xq.shape[0] if m is None else int(m)
        if xq.shape[1] != self.K or xq.shape[0] < M or xs.shape[0] < M:
            raise ValueError(f"xq {tuple(xq.shape)} / xs {tuple(xs.shape)} do not match M={M}, K={self.K}")
        with self._device_ctx(xq, xs, out):
            if out is None:
                out = torch.empty(M, self.N, dtype=self.out_dtype, device=xq.device)
            _need(out, "out", (self.out_dtype,), shape=(M, self.N))
            _check(self._L.cr_w4a8_plan_gemv(self._plan, xq.data_ptr(), xs.data_ptr(), M, out.data_ptr(),
                                             _stream(stream)), "cr_w4a8_plan_gemv")
        return out

    def forward_host(self, x_host, out_host, x_dev, out_dev, xq_work=None, xs_work=None, stream=None):
        """x_host [M, K] bf16 and out_host [M, N] in host memory (pinned for
        asynchronous copies), x_dev / out_dev their device buffers: queues the
        copy in, the forward and the copy out on the stream; out_host is ready
        once the stream has reached that point.  A decode batch with bf16
        outputs, N a multiple of 8 and a pinned out_host has its GEMV store y
        into out_host directly, and out_dev is then not written.  With caller-owned work
        buffers the call is bound to its tensors (cr_w4a8_plan_bind_host),
        and a repeat with the same tensors, unchanged in storage and shape,
        only queues the launches."""
        with self._device_ctx(x_dev, out_dev, xq_work, xs_work):
            return self._forward_host(x_host, out_host, x_dev, out_dev, xq_work, xs_work, stream)

    def _forward_host(self, x_host, out_host, x_dev, out_dev, xq_work, xs_work, stream):
        key = (x_host, out_host, x_dev, out_dev, xq_work, xs_work)
        # the bound call is used and replaced under the lock: the C call releases
        # the GIL, and another thread must not free the call while it runs
        with self._host_lock:
            hit = self._host_args
            if hit is not None and all(a is b for a, b in zip(hit[0], key)):
                if hit[1] == tuple(None if t is None else (t.data_ptr(), t.shape) for t in key):
                    _check(self._run_host(hit[2], _stream(stream)), "cr_w4a8_host_call_run")
                    return out_host
        torch = _torch()
        if x_host.is_cuda or out_host.is_cuda:
            raise ValueError("x_host and out_host must be host tensors")
        if x_host.dtype != torch.bfloat16 or x_host.dim() != 2 or not x_host.is_contiguous():
            raise ValueError("x_host must be a contiguous bf16 [M, K] tensor")
        M, K = x_host.shape
        if K != self.K:
            raise ValueError(f"x has K={K}, the layer K={self.K}")
        if out_host.dtype != self.out_dtype or tuple(out_host.shape) != (M, self.N) or not out_host.is_contiguous():
            raise ValueError(f"out_host must be a contiguous {self.out_dtype} [{M}, {self.N}] tensor")
        _need(x_dev, "x_dev", (torch.bfloat16,), shape=(M, K))
        _need(out_dev, "out_dev", (self.out_dtype,), shape=(M, self.N))
        xq, xs = self._work(x_dev, M, xq_work, xs_work)
        ptrs = (x_host.data_ptr(), M, out_host.data_ptr(), x_dev.data_ptr(), out_dev.data_ptr(), xq.data_ptr(),
                xs.data_ptr())
        if xq_work is None or xs_work is None:  # work buffers of this call only: nothing to bind
            _check(self._fwd_host(self._plan, *ptrs, _stream(stream)), "cr_w4a8_plan_forward_host")
            return out_host
        with self._host_lock:
            self._drop_host_call()
            call = ctypes.c_void_p()
            _check(self._L.cr_w4a8_plan_bind_host(self._plan, *ptrs, ctypes.byref(call)), "cr_w4a8_plan_bind_host")
            # the bound tensors are held with the call, so their memory outlives it
            self._host_args = (key, tuple(None if t is None else (t.data_ptr(), t.shape) for t in key), call)
            _check(self._run_host(call, _stream(stream)), "cr_w4a8_host_call_run")
        return out_host


@_on_device
def cr_w4a8_linear_decode_noalloc(x, qdata, srel, codebook, s_channel, bias=None, act_qmax: int = 127,
                                  out_dtype=None, out=None, stream=None):
    """The decode forward (M <= 8) for callers that cannot allocate device
    memory during the call (a serving loop whose device memory all belongs to
    its own allocator, or a real-time path that cannot take an allocation's
    synchronisation): the quantised activations live in a small scratch array
    the library reserves statically per device.  Pass `out` to allocate
    nothing at all.  Calls that overlap on the GPU share that scratch and
    race.  The first call on a device looks up the scratch array's address;
    make it before any stream capture on that device."""
    torch = _torch()
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    N, Kw = _layer(qdata, srel, codebook, s_channel, bias)
    if Kw != K:
        raise ValueError(f"x has K={K}, the layer K={Kw}")
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype or torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16, torch.float32), shape=(M, N))
    _check(lib().cr_w4a8_linear_decode_noalloc(_ptr(x), _ptr(qdata), _ptr(srel), _ptr(codebook),
                                               _ptr(s_channel), _ptr(bias), M, N, K, int(act_qmax),
                                               _out_code(out.dtype), _ptr(out), _stream(stream)),
           "cr_w4a8_linear_decode_noalloc")
    return out


def _grouped(layers, codebook, K, M, out_dtype, outs, acc_out, device):
    """Check a list of (qdata, srel, s_channel[, bias]) layers that share K and
    the codebook; allocate missing outputs; return the C array and the outputs."""
    torch = _torch()
    layers = list(layers)
    if not 1 <= len(layers) <= CR_MAX_LAYERS:
        raise ValueError(f"1..{CR_MAX_LAYERS} layers, got {len(layers)}")
    if outs is not None and len(outs) != len(layers):
        raise ValueError("one output per layer")
    arr = (CrLayer * len(layers))()
    res, accs = [], []
    for i, ly in enumerate(layers):
        qdata, srel, s_channel = ly[0], ly[1], ly[2]
        bias = ly[3] if len(ly) > 3 else None
        N, Kw = _layer(qdata, srel, codebook, s_channel, bias)
        if Kw != K:
            raise ValueError(f"layer {i} has K={Kw}, expected {K}")
        out = None if outs is None else outs[i]
        if out is None:
            out = torch.empty(M, N, dtype=out_dtype, device=device)
        _need(out, f"out[{i}]", (torch.bfloat16, torch.float32), shape=(M, N))
        if out.dtype != out_dtype:
            raise TypeError("all outputs of a grouped call have one dtype")
        acc = None
        if acc_out:
            acc = torch.empty(M, N, dtype=torch.int32, device=device)
        arr[i] = CrLayer(_ptr(qdata), _ptr(srel), _ptr(s_channel), _ptr(bias), N, _ptr(out), _ptr(acc))
        res.append(out)
        accs.append(acc)
    return arr, res, accs


@_on_device
def cr_w4a8_gemv_grouped(xq, xs, codebook, layers, m: Optional[int] = None, out_dtype=None, outs=None,
                         acc_out: bool = False, stream=None):
    """Decode GEMV of 1..4 layers on the same quantised activations in one
    launch.  layers: (qdata, srel, s_channel[, bias]) per layer.  Returns the
    list of outputs (and of int32 accumulators when acc_out=True); each equals
    cr_w4a8_gemv on that layer bit for bit."""
    torch = _torch()
    _need(xq, "xq", (torch.int8,), 2)
    _need(xs, "xs", (torch.float32,), 1)
    M = xq.shape[0] if m is None else int(m)
    K = xq.shape[1]
    if xq.shape[0] < M or xs.shape[0] < M:
        raise ValueError(f"xq {tuple(xq.shape)} / xs {tuple(xs.shape)} have fewer than M={M} rows")
    if out_dtype is None:
        out_dtype = outs[0].dtype if outs else torch.bfloat16
    _out_code(out_dtype)
    arr, res, accs = _grouped(layers, codebook, K, M, out_dtype, outs, acc_out, xq.device)
    _check(lib().cr_w4a8_gemv_grouped(_ptr(xq), _ptr(xs), _ptr(codebook), M, K, arr, len(res),
                                      _out_code(out_dtype), _stream(stream)), "cr_w4a8_gemv_grouped")
    return (res, accs) if acc_out else res


@_on_device
def cr_w4a8_linear_grouped(x, codebook, layers, act_qmax: int = 127, out_dtype=None, outs=None,
                           xq_work=None, xs_work=None, stream=None):
    """Forward of 1..4 layers fed the same x (q/k/v, gate/up): one rotate +
    quantise, then one grouped decode GEMV (M <= 8) or a GEMM per layer."""
    torch = _torch()
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    if out_dtype is None:
        out_dtype = outs[0].dtype if outs else torch.bfloat16
    _out_code(out_dtype)
    arr, res, _ = _grouped(layers, codebook, K, M, out_dtype, outs, False, x.device)
    rows = gemv_rows(M) if 1 <= M <= CR_GEMV_MAX_M else M
    if xq_work is None:
        xq_work = torch.empty(rows, K, dtype=torch.int8, device=x.device)
    if xs_work is None:
        xs_work = torch.empty(rows, dtype=torch.float32, device=x.device)
    _need(xq_work, "xq_work", (torch.int8,), 2)
    _need(xs_work, "xs_work", (torch.float32,), 1)
    if xq_work.shape[0] < rows or xq_work.shape[1] != K or xs_work.shape[0] < rows:
        raise ValueError(f"work buffers need {rows} rows of K={K}")
    _check(lib().cr_w4a8_linear_grouped(_ptr(x), _ptr(codebook), M, K, arr, len(res), int(act_qmax),
                                        _out_code(out_dtype), _ptr(xq_work), _ptr(xs_work), _stream(stream)),
           "cr_w4a8_linear_grouped")
    return res


def _swiglu_contraction(fn_name, xq, xs, qdata, srel, codebook, s_channel, bias, m, out_dtype, out, stream):
    torch = _torch()
    N, K = _layer(qdata, srel, codebook, s_channel, bias)
    if N % 2:
        raise ValueError(f"an interleaved gate/up layer has an even number of rows, got {N}")
    _need(xq, "xq", (torch.int8,), 2)
    _need(xs, "xs", (torch.float32,), 1)
    M = xq.shape[0] if m is None else int(m)
    if xq.shape[1] != K or xq.shape[0] < M or xs.shape[0] < M:
        raise ValueError(f"xq {tuple(xq.shape)} / xs {tuple(xs.shape)} do not match M={M}, K={K}")
    if out is None:
        out = torch.empty(M, N // 2, dtype=out_dtype, device=xq.device)
    _need(out, "out", (torch.bfloat16, torch.float32), shape=(M, N // 2))
    fn = getattr(lib(), fn_name)
    _check(fn(_ptr(xq), _ptr(xs), _ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel), _ptr(bias),
              M, N, K, _out_code(out.dtype), _ptr(out), _stream(stream)), fn_name)
    return out


@_on_device
def cr_w4a8_gemm_swiglu(xq, xs, qdata, srel, codebook, s_channel, bias=None, m: Optional[int] = None,
                        out_dtype=None, out=None, stream=None):
    """Prefill GEMM of an interleaved gate/up layer [2F, K] with SwiGLU fused
    into the epilogue: out [M, F] = silu(gate) * up."""
    torch = _torch()
    return _swiglu_contraction("cr_w4a8_gemm_swiglu", xq, xs, qdata, srel, codebook, s_channel, bias, m,
                               out_dtype or torch.bfloat16, out, stream)


@_on_device
def cr_w4a8_gemv_swiglu(xq, xs, qdata, srel, codebook, s_channel, bias=None, m: Optional[int] = None,
                        out_dtype=None, out=None, stream=None):
    """Decode GEMV (M <= 8) of an interleaved gate/up layer with SwiGLU fused;
    bitwise equal to cr_w4a8_gemm_swiglu."""
    torch = _torch()
    return _swiglu_contraction("cr_w4a8_gemv_swiglu", xq, xs, qdata, srel, codebook, s_channel, bias, m,
                               out_dtype or torch.bfloat16, out, stream)


@_on_device
def cr_w4a8_linear_swiglu(x, qdata, srel, codebook, s_channel, bias=None, act_qmax: int = 127, out_dtype=None,
                          out=None, xq_work=None, xs_work=None, stream=None):
    """The forward of an interleaved gate/up layer with SwiGLU fused:
    rotate + quantise x, then the decode GEMV (M <= 8) or the prefill GEMM."""
    torch = _torch()
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    N, Kw = _layer(qdata, srel, codebook, s_channel, bias)
    if Kw != K:
        raise ValueError(f"x has K={K}, the layer K={Kw}")
    if N % 2:
        raise ValueError(f"an interleaved gate/up layer has an even number of rows, got {N}")
    rows = gemv_rows(M) if 1 <= M <= CR_GEMV_MAX_M else M
    if xq_work is None:
        xq_work = torch.empty(rows, K, dtype=torch.int8, device=x.device)
    if xs_work is None:
        xs_work = torch.empty(rows, dtype=torch.float32, device=x.device)
    _need(xq_work, "xq_work", (torch.int8,), 2)
    _need(xs_work, "xs_work", (torch.float32,), 1)
    if xq_work.shape[0] < rows or xq_work.shape[1] != K or xs_work.shape[0] < rows:
        raise ValueError(f"work buffers need {rows} rows of K={K}")
    if out is None:
        out = torch.empty(M, N // 2, dtype=out_dtype or torch.bfloat16, device=x.device)
    _need(out, "out", (torch.bfloat16, torch.float32), shape=(M, N // 2))
    _check(lib().cr_w4a8_linear_swiglu(_ptr(x), _ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel),
                                       _ptr(bias), M, N, K, int(act_qmax), _out_code(out.dtype), _ptr(out),
                                       _ptr(xq_work), _ptr(xs_work), _stream(stream)), "cr_w4a8_linear_swiglu")
    return out


@_on_device
def cr_interleave_rows(src, dst=None, stream=None):
    """Rows [0, F) and [F, 2F) of src become pairs: dst[2f] = src[f],
    dst[2f + 1] = src[F + f] (any dtype, rows along dim 0)."""
    torch = _torch()
    if not isinstance(src, torch.Tensor) or not src.is_cuda or not src.is_contiguous() or src.dim() < 1:
        raise ValueError("src must be a contiguous CUDA tensor with at least one dimension")
    rows = src.shape[0]
    if rows % 2:
        raise ValueError(f"an even number of rows is needed, got {rows}")
    if dst is None:
        dst = torch.empty_like(src)
    if not dst.is_cuda or not dst.is_contiguous() or dst.shape != src.shape or dst.dtype != src.dtype:
        raise ValueError("dst must be a contiguous CUDA tensor of src's shape and dtype")
    row_bytes = src.numel() * src.element_size() // rows if rows else 0
    _check(lib().cr_interleave_rows(_ptr(src), _ptr(dst), rows, row_bytes, _stream(stream)), "cr_interleave_rows")
    return dst


@_on_device
def interleave_gate_up(gate, up, stream=None):
    """A gate/up pair of layers, each (qdata, srel, s_channel[, bias]) with
    the same K, as one layer with interleaved rows for the SwiGLU entry points
    (h3-rs weights.rs, QLinear::interleave_swiglu).  Returns (qdata, srel,
    s_channel, bias or None)."""
    torch = _torch()
    gate, up = list(gate), list(up)
    if len(gate) != len(up) or len(gate) not in (3, 4):
        raise ValueError("gate and up are (qdata, srel, s_channel[, bias]) of the same form")
    res = []
    for i, (g, u) in enumerate(zip(gate, up)):
        if g is None and u is None:
            res.append(None)
            continue
        if g is None or u is None or g.shape != u.shape or g.dtype != u.dtype:
            raise ValueError(f"gate and up differ in field {i}")
        res.append(cr_interleave_rows(torch.cat([g, u], dim=0).contiguous(), stream=stream))
    return tuple(res) + ((None,) if len(res) == 3 else ())


def _fixed_codebook(device):
    from .inputs import FIXED_CODEBOOK
    return _torch().tensor(FIXED_CODEBOOK, dtype=_torch().float32, device=device)


@_on_device
def cr_w4a8_quantize_rotated(w_rot, codebook=None, qdata=None, srel=None, s_channel=None, stream=None):
    """Offline quantiser: rotated fp32 weights [N, K] (K a multiple of 16) ->
    (qdata uint8 [N, K/2], srel uint8 [N, K/16] fp8 bytes, s_channel fp32 [N],
    codebook fp32 [16]).  codebook=None uses the pages' fixed codebook."""
    torch = _torch()
    _need(w_rot, "w_rot", (torch.float32,), 2)
    N, K = w_rot.shape
    if codebook is None:
        codebook = _fixed_codebook(w_rot.device)
    _need(codebook, "codebook", (torch.float32,), shape=(16,))
    if qdata is None:
        qdata = torch.empty(N, K // 2, dtype=torch.uint8, device=w_rot.device)
    if srel is None:
        srel = torch.empty(N, K // 16, dtype=torch.uint8, device=w_rot.device)
    if s_channel is None:
        s_channel = torch.empty(N, dtype=torch.float32, device=w_rot.device)
    _need(qdata, "qdata", (torch.uint8, torch.int8), shape=(N, K // 2))
    _need(srel, "srel", (torch.uint8, torch.float8_e4m3fn), shape=(N, K // 16))
    _need(s_channel, "s_channel", (torch.float32,), shape=(N,))
    _check(lib().cr_w4a8_quantize_rotated(_ptr(w_rot), _ptr(codebook), N, K, _ptr(qdata), _ptr(srel),
                                          _ptr(s_channel), _stream(stream)), "cr_w4a8_quantize_rotated")
    return qdata, srel, s_channel, codebook


@_on_device
def cr_w4a8_assign_codes(w_rot, srel, s_channel, codebook, rand=None, qdata=None, stream=None):
    """New packed codes for rotated weights on stored scales: the nearest grid
    level, or with rand [N, K] fp32 uniform draws the unbiased stochastic one."""
    torch = _torch()
    _need(w_rot, "w_rot", (torch.float32,), 2)
    N, K = w_rot.shape
    _need(srel, "srel", (torch.uint8, torch.float8_e4m3fn), shape=(N, K // 16))
    _need(s_channel, "s_channel", (torch.float32,), shape=(N,))
    _need(codebook, "codebook", (torch.float32,), shape=(16,))
    if rand is not None:
        _need(rand, "rand", (torch.float32,), shape=(N, K))
    if qdata is None:
        qdata = torch.empty(N, K // 2, dtype=torch.uint8, device=w_rot.device)
    _need(qdata, "qdata", (torch.uint8, torch.int8), shape=(N, K // 2))
    _check(lib().cr_w4a8_assign_codes(_ptr(w_rot), _ptr(srel), _ptr(s_channel), _ptr(codebook), _ptr(rand), N, K,
                                      _ptr(qdata), _stream(stream)), "cr_w4a8_assign_codes")
    return qdata


@_on_device
def cr_w4a8_ste_backward(grad, qdata, srel, codebook, s_channel, dx=None, stream=None, wt_work=None):
    """Straight-through input gradient: dx [M, K] bf16 = grad [M, N] bf16 @
    (w8 * s_channel in bf16), the layer's codes decoded again (N % 8 == 0).
    With wt_work (bf16 [K, N]) the transposed weight is built there
    (cr_w4a8_ste_backward_ws) and the library allocates nothing."""
    torch = _torch()
    N, K = _layer(qdata, srel, codebook, s_channel, None)
    _need(grad, "grad", (torch.bfloat16,), 2)
    M = grad.shape[0]
    if grad.shape[1] != N:
        raise ValueError(f"grad has {grad.shape[1]} columns, the layer N={N}")
    if dx is None:
        dx = torch.empty(M, K, dtype=torch.bfloat16, device=grad.device)
    _need(dx, "dx", (torch.bfloat16,), shape=(M, K))
    if wt_work is not None:
        _need(wt_work, "wt_work", (torch.bfloat16,), shape=(K, N))
        _check(lib().cr_w4a8_ste_backward_ws(_ptr(grad), _ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel),
                                             M, N, K, _ptr(dx), _ptr(wt_work), _stream(stream)),
               "cr_w4a8_ste_backward_ws")
        return dx
    _check(lib().cr_w4a8_ste_backward(_ptr(grad), _ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel), M, N,
                                      K, _ptr(dx), _stream(stream)), "cr_w4a8_ste_backward")
    return dx


@_on_device
def cr_w4a8_ste_backward_ws(grad, qdata, srel, codebook, s_channel, wt_work, dx=None, stream=None):
    """cr_w4a8_ste_backward with the caller's transient wt_work bf16 [K, N]."""
    if wt_work is None:
        raise ValueError("wt_work is required")
    return cr_w4a8_ste_backward(grad, qdata, srel, codebook, s_channel, dx=dx, stream=stream, wt_work=wt_work)


@_on_device
def cr_w4a8_dequant_t_bf16(qdata, srel, codebook, s_channel, wt=None, stream=None):
    """The backward's weight, transposed: wt [K, N] bf16, wt[k, n] = bf16(w8[n, k] * bf16(s_channel[n]))."""
    torch = _torch()
    N, K = _layer(qdata, srel, codebook, s_channel, None)
    if wt is None:
        wt = torch.empty(K, N, dtype=torch.bfloat16, device=qdata.device)
    _need(wt, "wt", (torch.bfloat16,), shape=(K, N))
    _check(lib().cr_w4a8_dequant_t_bf16(_ptr(qdata), _ptr(srel), _ptr(codebook), _ptr(s_channel), N, K, _ptr(wt),
                                        _stream(stream)), "cr_w4a8_dequant_t_bf16")
    return wt


def cr_mma_i8_peak(iters: int, stream=None) -> float:
    """Queue the INT8 tensor-core rate measurement kernel on the current
    device; returns the int8 operations of the launch (time it with CUDA
    events on `stream`)."""
    ops = ctypes.c_double()
    _check(lib().cr_mma_i8_peak(int(iters), ctypes.byref(ops), _stream(stream)), "cr_mma_i8_peak")
    return ops.value


def cr_selftest_wait_timeout(seconds: float = 0.005, stream=None) -> None:
    """Queue a bounded wait that nothing completes; after `seconds` it sets the
    device error word, which cr_check_device_error then reports."""
    _check(lib().cr_selftest_wait_timeout(int(seconds * 1e9), _stream(stream)), "cr_selftest_wait_timeout")


def cr_check_device_error(stream=None) -> None:
    """Synchronise the stream and raise CrError if a kernel's bounded wait ran out."""
    _check(lib().cr_check_device_error(_stream(stream)), "cr_check_device_error")
