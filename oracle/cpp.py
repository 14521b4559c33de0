"""ctypes wrapper of the plain C++ FP64 oracle (``storeh_oracle.cpp``).

TEST INFRASTRUCTURE ONLY, like the rest of this package: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use it.  It shares
no code with the CUDA library.

The functions mirror the numpy oracle's names and array conventions
(``storeh_oracle.py``), so a test can run the same pin against both:
``quantize_rows``, ``dequantize_rows``, ``attend_explicit``, ``attend_absorbed``,
``residual_norm_check``, plus ``decode_lane`` (one lane's whole decode iteration, as
the CPU baseline times it).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

from .storeh_oracle import FMT_FP16, FMT_INT4, FMT_INT8, row_code_bytes, row_scale_count  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "storeh_oracle.cpp")
LIB_PATH = os.path.join(_HERE, "libstoreh_oracle.so")
# no fast-math and no FMA contraction: fp32 divisions, roundings and FP64 sums stay as written
CXX_FLAGS = ["-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(SRC):
        tmp = LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++"] + CXX_FLAGS + ["-o", tmp, SRC])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        L.oracle_quantize_rows.argtypes = [i32, i32, i64, vp, vp, vp]
        L.oracle_dequantize_rows.argtypes = [i32, i32, i64, vp, vp, vp]
        L.oracle_attend.argtypes = [i32, i64, i32, i32, i32, vp, vp, vp, vp, vp, vp, i32]
        L.oracle_residual_norm_check.argtypes = [vp, i32, i32, f32, i32, vp, vp, vp, vp]
        L.oracle_decode_lane.argtypes = [i32, i32, i32, i32, i64, vp, vp, vp, vp, vp, vp, vp, f32, i32, i32, i32,
                                         vp, vp, vp, i32]
        L.oracle_f32_to_f16.argtypes = [f32]
        L.oracle_f32_to_f16.restype = ctypes.c_uint16
        L.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f64.restype = ctypes.c_double
        L.oracle_max_threads.restype = i32
        for f in (L.oracle_quantize_rows, L.oracle_dequantize_rows, L.oracle_attend, L.oracle_residual_norm_check,
                  L.oracle_decode_lane):
            f.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _f16(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float16)).view(np.uint16)


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def quantize_rows(h: np.ndarray, fmt: int) -> Tuple[np.ndarray, np.ndarray]:
    """fp16 rows [n, d] -> (codes uint8 [n, row_code_bytes], scales [n, row_scale_count]);
    scales fp32 (INT8), fp16 (INT4) or empty fp32 (FP16), as the numpy oracle returns them."""
    h = np.asarray(h)
    assert h.dtype == np.float16 and h.ndim == 2
    n, d = h.shape
    hb = _f16(h)
    codes = np.zeros((n, row_code_bytes(fmt, d)), np.uint8)
    if fmt == FMT_FP16:
        scales = np.zeros((n, 0), np.float32)
    elif fmt == FMT_INT8:
        scales = np.zeros((n, 1), np.float32)
    else:
        scales = np.zeros((n, row_scale_count(fmt, d)), np.float16)
    lib().oracle_quantize_rows(fmt, d, n, _p(hb), _p(codes), _p(scales) if scales.size else None)
    return codes, scales


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, fmt: int, d: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    n = codes.shape[0]
    out = np.empty((n, d), np.float64)
    sc = np.ascontiguousarray(scales) if fmt != FMT_FP16 else None
    lib().oracle_dequantize_rows(fmt, d, n, _p(codes), _p(sc) if sc is not None else None, _p(out))
    return out


def _attend(form: int, h_hat, h_new, W_q, W_k, W_v, H: int, hd: int, threads: Optional[int]) -> np.ndarray:
    hh = np.ascontiguousarray(h_hat, dtype=np.float64)
    n, d = hh.shape
    assert d == H * hd
    hn = _f16(np.asarray(h_new).reshape(-1))
    Wq, Wk, Wv = (_f16(w) for w in (W_q, W_k, W_v))
    out = np.empty((H, hd), np.float64)
    lib().oracle_attend(form, n, d, H, hd, _p(hh), _p(hn), _p(Wq), _p(Wk), _p(Wv), _p(out),
                        threads if threads else max_threads())
    return out


def attend_explicit(h_hat, h_new, W_q, W_k, W_v, H: int, hd: int, threads: Optional[int] = None) -> np.ndarray:
    """K and V rebuilt explicitly for every row (the definition); FP64; out [H, hd]."""
    return _attend(0, h_hat, h_new, W_q, W_k, W_v, H, hd, threads)


def attend_absorbed(h_hat, h_new, W_q, W_k, W_v, H: int, hd: int, threads: Optional[int] = None) -> np.ndarray:
    """The algebraically equal absorbed form (used for long sampled lanes); FP64; out [H, hd]."""
    return _attend(1, h_hat, h_new, W_q, W_k, W_v, H, hd, threads)


def residual_norm_check(residual, threshold: float, it: int, loops, abort_flags, first_abort_iter):
    """Same contract as the numpy oracle's: returns (flags, first_abort_iter, norms)."""
    r = np.ascontiguousarray(residual, dtype=np.float32)
    B, d = r.shape
    lp = np.ascontiguousarray(loops, dtype=np.int32)
    flags = np.array(abort_flags, dtype=np.uint8, copy=True)
    first = np.array(first_abort_iter, dtype=np.int32, copy=True)
    norms = np.empty(B, np.float64)
    lib().oracle_residual_norm_check(_p(r), B, d, float(np.float32(threshold)), it, _p(lp), _p(flags), _p(first),
                                     _p(norms))
    return flags, first, norms


def decode_lane(fmt: int, ctx_codes: np.ndarray, ctx_scales: np.ndarray, h_new, W_q, W_k, W_v, H: int, hd: int,
                residual=None, threshold: float = 0.0, it: int = 0, loops: int = 1, form: int = 0,
                flag: int = 0, first: int = -1, threads: Optional[int] = None):
    """One lane's decode iteration: append h_new (quantised) after the lane's n_ctx cached rows
    (codes / scales as quantize_rows returns them), dequantise, attend, check.  Returns
    (out [H, hd], flag, first, codes, scales) with the appended row included."""
    d = H * hd
    n = ctx_codes.shape[0]
    codes = np.zeros((n + 1, row_code_bytes(fmt, d)), np.uint8)
    codes[:n] = ctx_codes
    if fmt == FMT_FP16:
        scales = np.zeros((n + 1, 0), np.float32)
    else:
        scales = np.zeros((n + 1,) + ctx_scales.shape[1:], ctx_scales.dtype)
        scales[:n] = ctx_scales
    hn = _f16(np.asarray(h_new).reshape(-1))
    Wq, Wk, Wv = (_f16(w) for w in (W_q, W_k, W_v))
    out = np.empty((H, hd), np.float64)
    fl = np.array([flag], np.uint8)
    fi = np.array([first], np.int32)
    res = np.ascontiguousarray(residual, dtype=np.float32).reshape(-1) if residual is not None else None
    lib().oracle_decode_lane(fmt, d, H, hd, n, _p(codes), _p(scales) if scales.size else None, _p(hn), _p(Wq),
                             _p(Wk), _p(Wv), _p(res) if res is not None else None, float(np.float32(threshold)), it,
                             loops, form, _p(out), _p(fl), _p(fi), threads if threads else max_threads())
    return out, int(fl[0]), int(fi[0]), codes, scales


def f32_to_f16_bits(x: float) -> int:
    return int(lib().oracle_f32_to_f16(float(x)))
