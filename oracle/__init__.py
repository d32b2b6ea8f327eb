"""CPU oracle for the ConvRot W4A8 codebook linear forward (numpy front end).

TEST INFRASTRUCTURE ONLY.  This package may be imported only by ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py``.  The CUDA library and its Python binding never import it, and
it imports nothing from them.

Every function is a thin marshalling wrapper over the scalar C definitions
in ``cr_oracle.c`` (which carry the citations and the readings).  Arrays are
numpy; bf16 values travel as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import numpy as np

from . import build as _build

_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the oracle shared library."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            P = ctypes.c_void_p
            i64 = ctypes.c_int64
            L.or_fp8_e4m3fn_to_f32.argtypes = [ctypes.c_uint8]
            L.or_fp8_e4m3fn_to_f32.restype = ctypes.c_float
            L.or_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.or_bf16_to_f32.restype = ctypes.c_float
            L.or_f32_to_bf16_rne.argtypes = [ctypes.c_float]
            L.or_f32_to_bf16_rne.restype = ctypes.c_uint16
            L.or_unpack_codes.argtypes = [P, i64, i64, P]
            L.or_unpack_codes.restype = None
            L.or_decode_one.argtypes = [ctypes.c_float, ctypes.c_float]
            L.or_decode_one.restype = ctypes.c_int8
            L.or_decode_w8.argtypes = [P, P, P, i64, i64, P]
            L.or_decode_w8.restype = None
            L.or_hadamard_dense.argtypes = [ctypes.c_int, P]
            L.or_hadamard_dense.restype = ctypes.c_int
            L.or_rotate_rows.argtypes = [P, i64, i64, P]
            L.or_rotate_rows.restype = ctypes.c_int
            L.or_act_quant_rows.argtypes = [P, i64, i64, i64, ctypes.c_int, P, P]
            L.or_act_quant_rows.restype = ctypes.c_int
            L.or_gemm_s32_rows.argtypes = [P, P, i64, i64, i64, i64, P]
            L.or_gemm_s32_rows.restype = ctypes.c_int
            L.or_epilogue.argtypes = [P, P, P, P, i64, i64, ctypes.c_int, P]
            L.or_epilogue.restype = None
            L.or_f64_to_bf16_rne.argtypes = [ctypes.c_double]
            L.or_f64_to_bf16_rne.restype = ctypes.c_uint16
            L.or_epilogue_swiglu.argtypes = [P, P, P, P, i64, i64, ctypes.c_int, P]
            L.or_epilogue_swiglu.restype = None
            L.or_f32_to_fp8_e4m3fn.argtypes = [ctypes.c_float]
            L.or_f32_to_fp8_e4m3fn.restype = ctypes.c_uint8
            L.or_nearest_level.argtypes = [P, ctypes.c_int, ctypes.c_float]
            L.or_nearest_level.restype = ctypes.c_int
            L.or_stochastic_level.argtypes = [P, ctypes.c_int, ctypes.c_float, ctypes.c_float]
            L.or_stochastic_level.restype = ctypes.c_int
            L.or_grid_levels.argtypes = [P, ctypes.c_uint8, P]
            L.or_grid_levels.restype = None
            L.or_group_scale_als.argtypes = [P, P, P]
            L.or_group_scale_als.restype = ctypes.c_float
            L.or_quantize_rotated.argtypes = [P, i64, i64, P, P, P, P]
            L.or_quantize_rotated.restype = ctypes.c_int
            L.or_assign_codes.argtypes = [P, P, P, P, P, i64, i64, P]
            L.or_assign_codes.restype = ctypes.c_int
            L.or_dequant_bf16.argtypes = [P, P, P, P, i64, i64, P]
            L.or_dequant_bf16.restype = None
            L.or_ste_backward.argtypes = [P, P, P, P, P, i64, i64, i64, P]
            L.or_ste_backward.restype = ctypes.c_int
            _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


# ---------------------------------------------------------------- scalars

def fp8_e4m3fn_to_f32(byte: int) -> float:
    return float(lib().or_fp8_e4m3fn_to_f32(int(byte)))


def bf16_to_f32(bits: int) -> float:
    return float(lib().or_bf16_to_f32(int(bits)))


def f32_to_bf16(values) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (round to nearest even)."""
    v = _c(values, np.float32).reshape(-1)
    L = lib()
    out = np.empty(v.shape, dtype=np.uint16)
    for i, f in enumerate(v.tolist()):
        out[i] = L.or_f32_to_bf16_rne(ctypes.c_float(f))
    return out.reshape(np.shape(values))


def decode_one(cb_value: float, srel_value: float) -> int:
    return int(lib().or_decode_one(ctypes.c_float(cb_value), ctypes.c_float(srel_value)))


# ---------------------------------------------------------------- arrays

def unpack_codes(qdata) -> np.ndarray:
    """Packed codes [N, K/2] (int8 or uint8) -> codes [N, K] uint8 in 0..15."""
    q = _c(np.asarray(qdata).view(np.uint8), np.uint8)
    n, kh = q.shape
    out = np.empty((n, 2 * kh), dtype=np.uint8)
    lib().or_unpack_codes(_p(q), n, kh, _p(out))
    return out


def decode_w8(qdata, srel, codebook) -> np.ndarray:
    """Packed codes [N, K/2], fp8 group scales [N, K/16], codebook[16] -> int8 [N, K]."""
    q = _c(np.asarray(qdata).view(np.uint8), np.uint8)
    s = _c(np.asarray(srel).view(np.uint8), np.uint8)
    cb = _c(codebook, np.float32)
    n, kh = q.shape
    k = 2 * kh
    if s.shape != (n, k // 16) or cb.shape != (16,):
        raise ValueError("decode_w8: shape mismatch")
    out = np.empty((n, k), dtype=np.int8)
    lib().or_decode_w8(_p(q), _p(s), _p(cb), n, k, _p(out))
    return out


def hadamard_dense(size: int) -> np.ndarray:
    """The normalised regular Hadamard of the given power-of-4 size, fp64."""
    out = np.empty((size, size), dtype=np.float64)
    rc = lib().or_hadamard_dense(int(size), _p(out))
    if rc != 0:
        raise ValueError(f"hadamard size {size} is not a power of 4")
    return out


def rotate_rows(x_bf16) -> np.ndarray:
    """bf16 bits [M, K] -> fp32 [M, K], block-256 rotated."""
    x = _c(x_bf16, np.uint16)
    m, k = x.shape
    out = np.empty((m, k), dtype=np.float32)
    if lib().or_rotate_rows(_p(x), m, k, _p(out)) != 0:
        raise ValueError("rotate_rows: K must be a positive multiple of 256")
    return out


def act_quant(r, mp: Optional[int] = None, qmax: int = 127):
    """Rotated fp32 rows [M, K] -> (xq int8 [MP, K], xs fp32 [MP])."""
    r = _c(r, np.float32)
    m, k = r.shape
    mp = m if mp is None else int(mp)
    xq = np.empty((mp, k), dtype=np.int8)
    xs = np.empty((mp,), dtype=np.float32)
    if lib().or_act_quant_rows(_p(r), m, k, mp, int(qmax), _p(xq), _p(xs)) != 0:
        raise ValueError("act_quant: need MP >= M and 1 <= qmax <= 127")
    return xq, xs


def rotate_quant_act(x_bf16, mp: Optional[int] = None, qmax: int = 127):
    return act_quant(rotate_rows(x_bf16), mp, qmax)


def gemm_s32(xq, w8, threads: int = 1) -> np.ndarray:
    """acc[m, n] = sum_k xq[m, k] * w8[n, k], int32 (exact; int64 inside)."""
    xq = _c(xq, np.int8)
    w8 = _c(w8, np.int8)
    m, k = xq.shape
    n = w8.shape[0]
    if w8.shape[1] != k:
        raise ValueError("gemm_s32: K mismatch")
    acc = np.empty((m, n), dtype=np.int32)
    L = lib()
    threads = max(1, min(int(threads), m)) if m else 1
    bounds = [m * t // threads for t in range(threads + 1)]
    rcs = [0] * threads

    def run(t):
        rcs[t] = L.or_gemm_s32_rows(_p(xq), _p(w8), bounds[t], bounds[t + 1], n, k, _p(acc))

    if threads == 1:
        run(0)
    else:
        ts = [threading.Thread(target=run, args=(t,)) for t in range(threads)]
        for t in ts:
            t.start()
        for t in ts:
            t.join()
    if any(rcs):
        raise OverflowError("gemm_s32: accumulator left the int32 range")
    return acc


def epilogue(acc, xs, ws, bias=None, out: str = "bf16") -> np.ndarray:
    """int32 [M, N] -> bf16 bits (uint16) or fp32 [M, N]."""
    acc = _c(acc, np.int32)
    m, n = acc.shape
    xs = _c(xs, np.float32)[:m]
    ws = _c(ws, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    if out == "bf16":
        res = np.empty((m, n), dtype=np.uint16)
        flag = 1
    elif out == "f32":
        res = np.empty((m, n), dtype=np.float32)
        flag = 0
    else:
        raise ValueError(out)
    lib().or_epilogue(_p(acc), _p(xs), _p(ws), _p(b), m, n, flag, _p(res))
    return res


def f64_to_bf16(value: float) -> int:
    """One double -> bf16 bits, rounded once (nearest, ties to even)."""
    return int(lib().or_f64_to_bf16_rne(float(value)))


def interleave_rows(a) -> np.ndarray:
    """h3-rs src/weights.rs, interleave_rows: the two halves of the row
    dimension [a0 .. aF-1, b0 .. bF-1] become [a0, b0, a1, b1, ...] (rows
    carry their trailing dimensions with them)."""
    a = np.ascontiguousarray(a)
    n = a.shape[0]
    if n % 2:
        raise ValueError("an even number of rows is needed")
    halves = a.reshape((2, n // 2) + a.shape[1:])
    return np.ascontiguousarray(np.swapaxes(halves, 0, 1)).reshape(a.shape)


def epilogue_swiglu(acc, xs, ws, bias=None, out: str = "bf16") -> np.ndarray:
    """int32 [M, 2F] on interleaved gate/up rows -> silu(g) * u as bf16 bits
    (uint16) or fp32 [M, F]."""
    acc = _c(acc, np.int32)
    m, n = acc.shape
    if n % 2:
        raise ValueError("interleaved gate/up needs an even number of columns")
    f = n // 2
    xs = _c(xs, np.float32)[:m]
    ws = _c(ws, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    if out == "bf16":
        res = np.empty((m, f), dtype=np.uint16)
        flag = 1
    elif out == "f32":
        res = np.empty((m, f), dtype=np.float32)
        flag = 0
    else:
        raise ValueError(out)
    lib().or_epilogue_swiglu(_p(acc), _p(xs), _p(ws), _p(b), m, f, flag, _p(res))
    return res


def linear_swiglu(x_bf16, qdata, srel, codebook, s_channel, bias=None, qmax: int = 127,
                  out: str = "bf16", threads: int = 1) -> dict:
    """The forward of a gate/up layer stored with interleaved rows, SwiGLU
    fused into the epilogue: rotate + quantise x, decode W, contract, then
    silu(gate) * up.  Returns xq, xs, w8, acc and y [M, N/2]."""
    xq, xs = rotate_quant_act(x_bf16, None, qmax)
    w8 = decode_w8(qdata, srel, codebook)
    acc = gemm_s32(xq, w8, threads)
    y = epilogue_swiglu(acc, xs, s_channel, bias, out)
    return {"xq": xq, "xs": xs, "w8": w8, "acc": acc, "y": y}


# ---------------------------------------------------------------- offline quantiser

def f32_to_fp8(value: float) -> int:
    """One fp32 -> fp8 e4m3fn byte with torch's cast semantics (NaN on overflow)."""
    return int(lib().or_f32_to_fp8_e4m3fn(float(np.float32(value))))


def nearest_level(levels, x: float) -> int:
    """Index of the nearest of the sorted levels to fp32 x (ties to the lower)."""
    lv = _c(levels, np.float32)
    return int(lib().or_nearest_level(_p(lv), lv.size, float(np.float32(x))))


def stochastic_level(levels, x: float, u: float) -> int:
    lv = _c(levels, np.float32)
    return int(lib().or_stochastic_level(_p(lv), lv.size, float(np.float32(x)), float(np.float32(u))))


def grid_levels(codebook, srel_byte: int) -> np.ndarray:
    """The 16 int8 grid values of one fp8 group scale, as fp32."""
    cb = _c(codebook, np.float32)
    out = np.empty(16, dtype=np.float32)
    lib().or_grid_levels(_p(cb), int(srel_byte), _p(out))
    return out


def group_scale_als(gw, codebook):
    """(gs, codes) of one 16-weight group after the ALS passes."""
    g = _c(gw, np.float32)
    cb = _c(codebook, np.float32)
    q = np.empty(16, dtype=np.int32)
    gs = lib().or_group_scale_als(_p(g), _p(cb), _p(q))
    return float(np.float32(gs)), q


def quantize_rotated(w_rot, codebook):
    """w_rot fp32 [N, K] -> (qdata uint8 [N, K/2], srel uint8 [N, K/16], s_channel fp32 [N])."""
    w = _c(w_rot, np.float32)
    n, k = w.shape
    cb = _c(codebook, np.float32)
    q = np.empty((n, k // 2), dtype=np.uint8)
    s = np.empty((n, k // 16), dtype=np.uint8)
    ch = np.empty(n, dtype=np.float32)
    if lib().or_quantize_rotated(_p(w), n, k, _p(cb), _p(q), _p(s), _p(ch)) != 0:
        raise ValueError("K must be a multiple of 16")
    return q, s, ch


def assign_codes(w_rot, srel, s_channel, codebook, rand=None) -> np.ndarray:
    """New packed codes on stored scales; rand [N, K] fp32 draws for the stochastic choice."""
    w = _c(w_rot, np.float32)
    n, k = w.shape
    s, ch, cb = _c(srel, np.uint8), _c(s_channel, np.float32), _c(codebook, np.float32)
    r = None if rand is None else _c(rand, np.float32)
    q = np.empty((n, k // 2), dtype=np.uint8)
    if lib().or_assign_codes(_p(w), _p(s), _p(ch), _p(cb), _p(r), n, k, _p(q)) != 0:
        raise ValueError("K must be a multiple of 16")
    return q


# ---------------------------------------------------------------- straight-through backward

def dequant_bf16(qdata, srel, codebook, s_channel) -> np.ndarray:
    """bf16 bits [N, K] of w8 * bf16(s_channel), as the backward builds it."""
    q = _c(qdata, np.uint8)
    n, kh = q.shape
    out = np.empty((n, 2 * kh), dtype=np.uint16)
    lib().or_dequant_bf16(_p(q), _p(_c(srel, np.uint8)), _p(_c(codebook, np.float32)),
                          _p(_c(s_channel, np.float32)), n, 2 * kh, _p(out))
    return out


def ste_backward(grad_bf16, qdata, srel, codebook, s_channel) -> np.ndarray:
    """dx bf16 bits [M, K] = grad [M, N] @ dequant_bf16 [N, K] (double sums, one rounding)."""
    g = _c(grad_bf16, np.uint16)
    m, n = g.shape
    q = _c(qdata, np.uint8)
    k = 2 * q.shape[1]
    out = np.empty((m, k), dtype=np.uint16)
    if lib().or_ste_backward(_p(g), _p(q), _p(_c(srel, np.uint8)), _p(_c(codebook, np.float32)),
                             _p(_c(s_channel, np.float32)), m, n, k, _p(out)) != 0:
        raise MemoryError("oracle backward")
    return out


def linear(x_bf16, qdata, srel, codebook, s_channel, bias=None, qmax: int = 127,
           out: str = "bf16", threads: int = 1) -> dict:
    """The whole forward: rotate + quantise x, decode W, contract, epilogue.

    Returns every intermediate: xq, xs, w8, acc, y.
    """
    xq, xs = rotate_quant_act(x_bf16, None, qmax)
    w8 = decode_w8(qdata, srel, codebook)
    acc = gemm_s32(xq, w8, threads)
    y = epilogue(acc, xs, s_channel, bias, out)
    return {"xq": xq, "xs": xs, "w8": w8, "acc": acc, "y": y}


def mp_for(m: int) -> int:
    """[CR] _gemv_mp: the decode GEMV's padded row count, next power of two (1,2,4,8)."""
    return 1 << max(0, (int(m) - 1).bit_length())
