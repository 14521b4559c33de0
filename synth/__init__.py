"""Seeded synthetic inputs shared by the CPU oracle's tests and the GPU harness.

Holds none of the method's arithmetic: only counter-based random numbers
(SplitMix64 finaliser + Box-Muller, see ``synth.c``) and the workload shapes.
The C library is compiled in-tree by :func:`build` (gcc, OpenMP).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libtlsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``libtlsynth.so`` next to its source (no fast-math: libm stays IEEE)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.tls_f64_to_f16.argtypes = [dbl]
        L.tls_f64_to_f16.restype = ctypes.c_uint16
        L.tls_normal_f16.argtypes = [u64, u64, u64, i64, dbl, vp]
        L.tls_normal_f32.argtypes = [u64, u64, u64, i64, dbl, vp]
        L.tls_normal_f64.argtypes = [u64, u64, u64, i64, vp]
        L.tls_u64.argtypes = [u64, u64, u64, i64, vp]
        L.tls_h_rows_f16.argtypes = [u64, u64, u64, dbl, dbl, vp, i64, i64, vp]
        for f in (L.tls_normal_f16, L.tls_normal_f32, L.tls_normal_f64, L.tls_u64, L.tls_h_rows_f16):
            f.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ---------------------------------------------------------------- raw streams
def f64_to_f16(x: float) -> np.float16:
    return np.array([lib().tls_f64_to_f16(float(x))], dtype=np.uint16).view(np.float16)[0]


def normal_f64(seed: int, tid: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    lib().tls_normal_f64(seed, tid, offset, n, _ptr(out))
    return out


def normal_f16(seed: int, tid: int, offset: int, n: int, scale: float = 1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    lib().tls_normal_f16(seed, tid, offset, n, float(scale), _ptr(out))
    return out.view(np.float16)


def normal_f32(seed: int, tid: int, offset: int, n: int, scale: float = 1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().tls_normal_f32(seed, tid, offset, n, float(scale), _ptr(out))
    return out


def u64(seed: int, tid: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    lib().tls_u64(seed, tid, offset, n, _ptr(out))
    return out


# ---------------------------------------------------------------- tensor ids
TID_H = 1          # h rows, all (layer, lane, position)
TID_OUTLIER = 2    # Bernoulli draw per h row (outlier rows)
TID_WQ = 3
TID_WK = 4
TID_WV = 5
TID_RESIDUAL = 6   # residual per (iteration, lane)
TID_CTX = 7        # per-lane context length draws
TID_TRAJ = 8       # loop-iteration trajectories of h (iteration-axis delta cache inputs)

ROW_POS_BITS = 20  # positions per (layer, lane) in the row-id space
ROW_LANES = 256    # lanes per layer in the row-id space


def row_id(layer: int, lane: int, pos) -> np.ndarray:
    """Row id of h at (layer, lane, position): the counter base of that row."""
    pos = np.asarray(pos, dtype=np.uint64)
    return ((np.uint64(layer) * np.uint64(ROW_LANES) + np.uint64(lane)) << np.uint64(ROW_POS_BITS)) + pos


def h_rows_f16_into(out: np.ndarray, seed: int, row_ids: np.ndarray, d: int,
                    outlier_p: float = 0.0, outlier_mul: float = 1.0) -> None:
    """Fill ``out`` ([len(row_ids), d] float16/uint16, C-contiguous) with h rows."""
    rid = np.ascontiguousarray(row_ids, dtype=np.uint64)
    assert out.shape == (rid.shape[0], d) and out.dtype.itemsize == 2 and out.flags["C_CONTIGUOUS"]
    lib().tls_h_rows_f16(seed, TID_H, TID_OUTLIER, float(outlier_p), float(outlier_mul),
                         _ptr(rid), rid.shape[0], d, out.ctypes.data)


def h_rows_f16(seed: int, row_ids: np.ndarray, d: int, outlier_p: float = 0.0,
               outlier_mul: float = 1.0) -> np.ndarray:
    rid = np.ascontiguousarray(row_ids, dtype=np.uint64).reshape(-1)
    out = np.empty((rid.shape[0], d), dtype=np.float16)
    h_rows_f16_into(out, seed, rid, d, outlier_p, outlier_mul)
    return out


def trajectory_f16(seed: int, n_tokens: int, d: int, L: int, rho_first: float = 0.68,
                   rho_last: float = 0.04, rho_span: int = 32) -> np.ndarray:
    """Hidden-state trajectories along the loop iterations, [L+1, n_tokens, d] fp16.

    h^0 ~ N(0, 1); h^l = fp16(h^(l-1) + sigma_l z_l) with z_l ~ N(0, 1) and sigma_l set from
    |h^(l-1)| so that |h^l - h^(l-1)| / |h^l| is about rho_l, which falls geometrically from rho_first at
    iteration 1 to rho_last at iteration rho_span: the contraction the pages measure on
    the 407M / 2B models (0.68 at the first iteration to 0.04 at the 32nd).  A random walk
    with that step schedule, nothing more; every draw comes from the counter-based normals.
    """
    # token t's draws are the counters [t (L+1) d, (t+1) (L+1) d): one contiguous block for all
    # tokens, so the recurrence runs over all tokens at once
    z = normal_f64(seed, TID_TRAJ, 0, n_tokens * (L + 1) * d).reshape(n_tokens, L + 1, d)
    out = np.empty((L + 1, n_tokens, d), dtype=np.float16)
    out[0] = z[:, 0].astype(np.float16)  # round to nearest even, as normal_f16
    for l in range(1, L + 1):
        rho = rho_first * (rho_last / rho_first) ** ((l - 1) / max(rho_span - 1, 1))
        prev = out[l - 1].astype(np.float64)
        sigma = rho * np.linalg.norm(prev, axis=1, keepdims=True) / math.sqrt(d * (1.0 - rho * rho))
        out[l] = (prev + sigma * z[:, l]).astype(np.float16)
    return out


def _trajectory_f16_per_token(seed: int, n_tokens: int, d: int, L: int, rho_first: float = 0.68,
                              rho_last: float = 0.04, rho_span: int = 32) -> np.ndarray:
    """The same trajectories one token at a time (the definition the vectorised form follows)."""
    out = np.empty((L + 1, n_tokens, d), dtype=np.float16)
    for t in range(n_tokens):
        base = t * (L + 1) * d
        out[0, t] = normal_f16(seed, TID_TRAJ, base, d)
        for l in range(1, L + 1):
            rho = rho_first * (rho_last / rho_first) ** ((l - 1) / max(rho_span - 1, 1))
            zz = normal_f64(seed, TID_TRAJ, base + l * d, d)
            prev = out[l - 1, t].astype(np.float64)
            sigma = rho * np.linalg.norm(prev) / math.sqrt(d * (1.0 - rho * rho))
            out[l, t] = (prev + sigma * zz).astype(np.float16)
    return out


from .workloads import WORKLOADS, Workload, get_workload  # noqa: E402,F401
