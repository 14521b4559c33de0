"""Python binding of libtlstoreh.so, the store-h decode-attention library (sm_100a).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  There is no CPU
fallback: the first call fails loudly when the library is missing.

The same names as the C ABI in ``include/tl_storeh.h``:
``cache_bytes``, ``workspace_bytes``, ``append``, ``attn_decode``,
``residual_norm_check``, ``poll_status``.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtlstoreh.so")

TL_OK = 0
TL_ERR_INVALID_ARG = 1
TL_ERR_SHAPE = 2
TL_ERR_CAPACITY = 3
TL_ERR_UNSUPPORTED = 4
TL_ERR_CUDA = 5
TL_ERR_DEVICE_TIMEOUT = 6
TL_ERR_DEVICE_RANGE = 7

TL_H_FP16 = 0
TL_H_INT8_TOKEN = 1
TL_H_INT4_G64 = 2

# every symbol include/tl_storeh.h declares
EXPORTS = ["tl_storeh_cache_bytes", "tl_storeh_workspace_bytes", "tl_storeh_append", "tl_storeh_attn_decode",
           "tl_residual_norm_check", "tl_storeh_poll_status", "tl_status_string", "tl_last_error_message",
           "tl_storeh_abi_version", "tl_set_profile", "tl_storeh_attn_decode_static_ws",
           "tl_storeh_append_attn_decode", "tl_storeh_selftest_wait_timeout", "tl_delta_cache_bytes",
           "tl_delta_append", "tl_delta_workspace_bytes", "tl_delta_attn_decode", "tl_storeh_verify_attn",
           "tl_storeh_verify_workspace_bytes", "tl_storeh_prefill_attn", "tl_storeh_decode_ex",
           "tl_storeh_workspace_bytes_ex", "tl_storeh_attn_decode_rope", "tl_storeh_rope_workspace_bytes"]


class TLError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        super().__init__(f"{fn} -> {status}: {msg}")
        self.status = status


class Desc(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("n_pre", ctypes.c_int32), ("L_max", ctypes.c_int32), ("max_lanes", ctypes.c_int32),
                ("max_ctx", ctypes.c_int32), ("fmt", ctypes.c_int32)]


class Profile(ctypes.Structure):
    _fields_ = [("begin_events", ctypes.POINTER(ctypes.c_void_p)), ("end_events", ctypes.POINTER(ctypes.c_void_p)),
                ("capacity", ctypes.c_int32), ("recorded", ctypes.c_int32), ("launches", ctypes.c_int64)]


class DecodeOpts(ctypes.Structure):
    _fields_ = [("append", ctypes.c_int32), ("split_rows", ctypes.c_int32), ("reserved", ctypes.c_int32 * 7)]


class Cache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class DeltaDescC(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("L_max", ctypes.c_int32), ("max_lanes", ctypes.c_int32), ("max_ctx", ctypes.c_int32)]


class DeltaCacheC(ctypes.Structure):
    _fields_ = [("anchor", ctypes.c_void_p), ("deltas", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_lib_handle = None


def _load():
    """Load libtlstoreh.so once (raises when it is missing: there is no fallback)."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m store_kv_attention_b200.build_lib` "
                          "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    P = ctypes.POINTER
    L.tl_storeh_cache_bytes.argtypes = [P(Desc), P(sz), P(sz)]
    L.tl_storeh_workspace_bytes.argtypes = [P(Desc), i32, P(sz)]
    L.tl_storeh_append.argtypes = [P(Desc), Cache, i32, vp, i32, i32, vp, vp, vp, vp]
    L.tl_storeh_attn_decode.argtypes = [P(Desc), Cache, i32, vp, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp,
                                        sz, i32, vp]
    L.tl_storeh_append_attn_decode.argtypes = L.tl_storeh_attn_decode.argtypes
    L.tl_residual_norm_check.argtypes = [vp, i32, i32, f32, i32, vp, vp, vp, vp, vp]
    L.tl_storeh_poll_status.argtypes = [vp, sz, vp]
    L.tl_storeh_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_int64, vp]
    L.tl_storeh_selftest_wait_timeout.restype = ctypes.c_int
    for f in ("tl_storeh_cache_bytes", "tl_storeh_workspace_bytes", "tl_storeh_append", "tl_storeh_attn_decode",
              "tl_storeh_append_attn_decode", "tl_residual_norm_check", "tl_storeh_poll_status"):
        getattr(L, f).restype = ctypes.c_int
    L.tl_status_string.argtypes = [ctypes.c_int]
    L.tl_status_string.restype = ctypes.c_char_p
    L.tl_last_error_message.argtypes = []
    L.tl_last_error_message.restype = ctypes.c_char_p
    L.tl_storeh_abi_version.restype = ctypes.c_int32
    L.tl_storeh_attn_decode_static_ws.argtypes = [P(Desc), Cache, i32, vp, vp, vp, vp, vp, vp, vp, vp, f32, vp,
                                                  vp, vp, i32, vp, vp]
    L.tl_storeh_attn_decode_static_ws.restype = ctypes.c_int
    L.tl_set_profile.argtypes = [P(Profile)]
    L.tl_set_profile.restype = ctypes.c_int
    L.tl_delta_cache_bytes.argtypes = [P(DeltaDescC), P(sz), P(sz), P(sz)]
    L.tl_delta_cache_bytes.restype = ctypes.c_int
    L.tl_delta_append.argtypes = [P(DeltaDescC), DeltaCacheC, i32, vp, i32, i32, vp, vp, vp]
    L.tl_delta_append.restype = ctypes.c_int
    L.tl_delta_workspace_bytes.argtypes = [P(DeltaDescC), i32, P(sz)]
    L.tl_delta_workspace_bytes.restype = ctypes.c_int
    L.tl_delta_attn_decode.argtypes = [P(DeltaDescC), DeltaCacheC, i32, vp, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp,
                                       vp, vp, sz, i32, vp]
    L.tl_delta_attn_decode.restype = ctypes.c_int
    L.tl_storeh_verify_attn.argtypes = [P(Desc), Cache, i32, vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, sz, i32, vp]
    L.tl_storeh_verify_attn.restype = ctypes.c_int
    L.tl_storeh_prefill_attn.argtypes = [P(Desc), Cache, i32, vp, vp, vp, i32, vp, vp, vp, vp, vp, sz, i32, vp]
    L.tl_storeh_prefill_attn.restype = ctypes.c_int
    L.tl_storeh_verify_workspace_bytes.argtypes = [P(Desc), i32, i32, i32, P(sz)]
    L.tl_storeh_decode_ex.argtypes = [P(Desc), Cache, i32, vp, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp, sz,
                                      i32, P(DecodeOpts), vp]
    L.tl_storeh_decode_ex.restype = ctypes.c_int
    L.tl_storeh_workspace_bytes_ex.argtypes = [P(Desc), i32, P(DecodeOpts), P(sz)]
    L.tl_storeh_workspace_bytes_ex.restype = ctypes.c_int
    L.tl_storeh_attn_decode_rope.argtypes = [P(Desc), Cache, i32, vp, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp, vp, f32,
                                             vp, sz, i32, vp]
    L.tl_storeh_attn_decode_rope.restype = ctypes.c_int
    L.tl_storeh_rope_workspace_bytes.argtypes = [P(Desc), i32, P(sz)]
    L.tl_storeh_rope_workspace_bytes.restype = ctypes.c_int
    L.tl_storeh_verify_workspace_bytes.restype = ctypes.c_int
    _lib_handle = L
    return L


def __getattr__(name):
    if name == "lib":
        return _load()
    raise AttributeError(name)


def _check(st: int, fn: str) -> None:
    if st != TL_OK:
        raise TLError(st, fn, _load().tl_last_error_message().decode())


def _ptr(t) -> Optional[int]:
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


@dataclasses.dataclass
class StoreHDesc:
    d_model: int
    n_heads: int
    head_dim: int
    n_pre: int
    L_max: int
    max_lanes: int
    max_ctx: int
    fmt: int

    def c(self) -> Desc:
        return Desc(self.d_model, self.n_heads, self.head_dim, self.n_pre, self.L_max, self.max_lanes,
                    self.max_ctx, self.fmt)


def cache_bytes(desc: StoreHDesc):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_load().tl_storeh_cache_bytes(ctypes.byref(desc.c()), ctypes.byref(cb), ctypes.byref(sb)),
           "tl_storeh_cache_bytes")
    return cb.value, sb.value


def workspace_bytes(desc: StoreHDesc, n_lanes: int, split_rows: int = 0) -> int:
    """tl_storeh_workspace_bytes, or with split_rows != 0 tl_storeh_workspace_bytes_ex."""
    b = ctypes.c_size_t()
    if split_rows:
        opts = DecodeOpts(0, split_rows)
        _check(_load().tl_storeh_workspace_bytes_ex(ctypes.byref(desc.c()), n_lanes, ctypes.byref(opts),
                                                    ctypes.byref(b)), "tl_storeh_workspace_bytes_ex")
    else:
        _check(_load().tl_storeh_workspace_bytes(ctypes.byref(desc.c()), n_lanes, ctypes.byref(b)),
               "tl_storeh_workspace_bytes")
    return b.value


class StoreHCache:
    """Device buffers of one cache (torch uint8 tensors) plus a decode workspace."""

    def __init__(self, desc: StoreHDesc, device="cuda", n_lanes: Optional[int] = None, split_rows: int = 0):
        import torch
        self.desc = desc
        self.split_rows = split_rows
        cb, sb = cache_bytes(desc)
        self.codes = torch.empty(cb, dtype=torch.uint8, device=device)
        self.scales = torch.empty(max(sb, 256), dtype=torch.uint8, device=device) if sb else None
        n = n_lanes or desc.max_lanes
        self.ws_bytes = workspace_bytes(desc, n, split_rows)
        self.workspace = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=device)

    def c(self) -> Cache:
        return Cache(self.codes.data_ptr(), self.scales.data_ptr() if self.scales is not None else None)


# ---------------------------------------------------------------- iteration-axis delta cache (include/tl_delta.h)
@dataclasses.dataclass
class DeltaDesc:
    d_model: int
    n_heads: int
    head_dim: int
    L_max: int
    max_lanes: int
    max_ctx: int

    def c(self) -> DeltaDescC:
        return DeltaDescC(self.d_model, self.n_heads, self.head_dim, self.L_max, self.max_lanes, self.max_ctx)


def delta_cache_bytes(desc: DeltaDesc):
    a, d, s = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_load().tl_delta_cache_bytes(ctypes.byref(desc.c()), ctypes.byref(a), ctypes.byref(d), ctypes.byref(s)),
           "tl_delta_cache_bytes")
    return a.value, d.value, s.value


def delta_workspace_bytes(desc: DeltaDesc, n_lanes: int) -> int:
    b = ctypes.c_size_t()
    _check(_load().tl_delta_workspace_bytes(ctypes.byref(desc.c()), n_lanes, ctypes.byref(b)),
           "tl_delta_workspace_bytes")
    return b.value


class DeltaCache:
    """Device buffers of one delta cache: anchor fp16 [lanes][ctx][d], deltas int8 and
    scales fp16 [L_max-1][lanes][ctx][d or n_heads] (torch tensors); with ``n_lanes`` also a
    zeroed decode workspace for that many lanes."""

    def __init__(self, desc: DeltaDesc, device="cuda", n_lanes: Optional[int] = None):
        import torch
        self.desc = desc
        ab, db, sb = delta_cache_bytes(desc)
        self.anchor = torch.empty(ab // 2, dtype=torch.float16, device=device)
        self.deltas = torch.empty(max(db, 256), dtype=torch.int8, device=device)
        self.scales = torch.empty(max(sb // 2, 128), dtype=torch.float16, device=device)
        self.ws_bytes = delta_workspace_bytes(desc, n_lanes) if n_lanes else 0
        self.workspace = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=device) if n_lanes else None

    def c(self) -> DeltaCacheC:
        return DeltaCacheC(self.anchor.data_ptr(), self.deltas.data_ptr(), self.scales.data_ptr())


def delta_append(cache: DeltaCache, it: int, h_rows, start_pos, loops=None, stream=None) -> None:
    """h_rows: fp16 [n_lanes, n_rows, d] (device), the states of loop iteration ``it``;
    start_pos / loops int32 [n_lanes] (device)."""
    n_lanes, n_rows = int(h_rows.shape[0]), int(h_rows.shape[1])
    _check(_load().tl_delta_append(ctypes.byref(cache.desc.c()), cache.c(), it, _ptr(h_rows), n_lanes, n_rows,
                                   _ptr(start_pos), _ptr(loops), _stream(stream)), "tl_delta_append")


def delta_attn_decode(cache: DeltaCache, it: int, loops, ctx_len, h_new, W_q, W_k, W_v, out, residual=None,
                      threshold: float = 0.0, abort_flags=None, first_abort_iter=None, norms_out=None,
                      stream=None) -> None:
    """tl_delta_attn_decode: writes h_new as iteration ``it`` of each active lane's new token,
    then attends the rebuilt rows (the cache needs a workspace: DeltaCache(..., n_lanes=N))."""
    n_lanes = int(h_new.shape[0])
    _check(_load().tl_delta_attn_decode(ctypes.byref(cache.desc.c()), cache.c(), it, _ptr(loops), _ptr(ctx_len),
                                        _ptr(h_new), _ptr(W_q), _ptr(W_k), _ptr(W_v), _ptr(out), _ptr(residual),
                                        float(threshold), _ptr(abort_flags), _ptr(first_abort_iter),
                                        _ptr(norms_out), _ptr(cache.workspace), cache.ws_bytes, n_lanes,
                                        _stream(stream)), "tl_delta_attn_decode")


def append(cache: StoreHCache, layer: int, h_rows, start_pos, row_count=None, loops=None, stream=None) -> None:
    """h_rows: fp16 [n_lanes, n_rows, d] (device); start_pos/row_count/loops int32 [n_lanes] (device)."""
    n_lanes, n_rows = int(h_rows.shape[0]), int(h_rows.shape[1])
    _check(_load().tl_storeh_append(ctypes.byref(cache.desc.c()), cache.c(), layer, _ptr(h_rows), n_lanes, n_rows,
                                _ptr(start_pos), _ptr(row_count), _ptr(loops), _stream(stream)), "tl_storeh_append")


def attn_decode(cache: StoreHCache, it: int, loops, ctx_len, h_new, W_q, W_k, W_v, out,
                residual=None, threshold: float = 0.0, abort_flags=None, first_abort_iter=None,
                norms_out=None, stream=None, append: bool = False) -> None:
    """tl_storeh_attn_decode, or with append=True tl_storeh_append_attn_decode (h_new is first
    written as the new token's row of every active lane, in the same enqueue); through
    tl_storeh_decode_ex when the cache was made with a split length of its own."""
    n_lanes = int(h_new.shape[0])
    if cache.split_rows:  # the cache's workspace was sized for this split length: tl_storeh_decode_ex
        opts = DecodeOpts(1 if append else 0, cache.split_rows)
        _check(_load().tl_storeh_decode_ex(ctypes.byref(cache.desc.c()), cache.c(), it, _ptr(loops), _ptr(ctx_len),
                                           _ptr(h_new), _ptr(W_q), _ptr(W_k), _ptr(W_v), _ptr(out), _ptr(residual),
                                           float(threshold), _ptr(abort_flags), _ptr(first_abort_iter),
                                           _ptr(norms_out), cache.workspace.data_ptr(), cache.ws_bytes, n_lanes,
                                           ctypes.byref(opts), _stream(stream)), "tl_storeh_decode_ex")
        return
    name = "tl_storeh_append_attn_decode" if append else "tl_storeh_attn_decode"
    _check(getattr(_load(), name)(ctypes.byref(cache.desc.c()), cache.c(), it, _ptr(loops), _ptr(ctx_len),
                                  _ptr(h_new), _ptr(W_q), _ptr(W_k), _ptr(W_v), _ptr(out), _ptr(residual),
                                  float(threshold), _ptr(abort_flags), _ptr(first_abort_iter), _ptr(norms_out),
                                  cache.workspace.data_ptr(), cache.ws_bytes, n_lanes, _stream(stream)), name)


def attn_decode_static_ws(cache: StoreHCache, it: int, loops, ctx_len, h_new, W_q, W_k, W_v, out,
                          residual=None, threshold: float = 0.0, abort_flags=None, first_abort_iter=None,
                          norms_out=None, status_out=None, stream=None) -> None:
    """attn_decode on the library's built-in scratch (for callers that cannot allocate)."""
    n_lanes = int(h_new.shape[0])
    _check(_load().tl_storeh_attn_decode_static_ws(ctypes.byref(cache.desc.c()), cache.c(), it, _ptr(loops),
                                                   _ptr(ctx_len), _ptr(h_new), _ptr(W_q), _ptr(W_k), _ptr(W_v),
                                                   _ptr(out), _ptr(residual), float(threshold), _ptr(abort_flags),
                                                   _ptr(first_abort_iter), _ptr(norms_out), n_lanes,
                                                   _ptr(status_out), _stream(stream)),
           "tl_storeh_attn_decode_static_ws")


def verify_workspace_bytes(desc: StoreHDesc, n_lanes: int, n_branches: int, depth: int) -> int:
    b = ctypes.c_size_t()
    _check(_load().tl_storeh_verify_workspace_bytes(ctypes.byref(desc.c()), n_lanes, n_branches, depth,
                                                    ctypes.byref(b)), "tl_storeh_verify_workspace_bytes")
    return b.value


def verify_attn(cache: StoreHCache, it: int, loops, ctx_len, h_tree, W_q, W_k, W_v, out, workspace,
                stream=None) -> None:
    """tl_storeh_verify_attn: h_tree fp16 [n_lanes, K, D, d] (device) is appended at positions
    ctx_len[b] + k*D + t, then every tree token attends the context and its own branch prefix;
    out fp32 [n_lanes, K, D, H, hd]; workspace a uint8 device tensor of verify_workspace_bytes."""
    n_lanes, K, D = int(h_tree.shape[0]), int(h_tree.shape[1]), int(h_tree.shape[2])
    _check(_load().tl_storeh_verify_attn(ctypes.byref(cache.desc.c()), cache.c(), it, _ptr(loops), _ptr(ctx_len),
                                         _ptr(h_tree), K, D, _ptr(W_q), _ptr(W_k), _ptr(W_v), _ptr(out),
                                         _ptr(workspace), int(workspace.numel()), n_lanes, _stream(stream)),
           "tl_storeh_verify_attn")


def prefill_attn(cache: StoreHCache, it: int, loops, ctx_len, h_chunk, W_q, W_k, W_v, out, workspace,
                 stream=None) -> None:
    """tl_storeh_prefill_attn: h_chunk fp16 [n_lanes, T, d] appended at ctx_len[b] .. + T - 1, token
    t attending positions 0 .. ctx_len[b] + t; out fp32 [n_lanes, T, H, hd]."""
    n_lanes, T = int(h_chunk.shape[0]), int(h_chunk.shape[1])
    _check(_load().tl_storeh_prefill_attn(ctypes.byref(cache.desc.c()), cache.c(), it, _ptr(loops), _ptr(ctx_len),
                                          _ptr(h_chunk), T, _ptr(W_q), _ptr(W_k), _ptr(W_v), _ptr(out),
                                          _ptr(workspace), int(workspace.numel()), n_lanes, _stream(stream)),
           "tl_storeh_prefill_attn")


def rope_workspace_bytes(desc: StoreHDesc, n_lanes: int) -> int:
    b = ctypes.c_size_t()
    _check(_load().tl_storeh_rope_workspace_bytes(ctypes.byref(desc.c()), n_lanes, ctypes.byref(b)),
           "tl_storeh_rope_workspace_bytes")
    return b.value


def attn_decode_rope(cache: StoreHCache, it: int, loops, ctx_len, h_new, W_q, W_k, W_v, out, workspace,
                     rope_base: float = 10000.0, residual=None, threshold: float = 0.0, abort_flags=None,
                     first_abort_iter=None, norms_out=None, stream=None) -> None:
    """tl_storeh_attn_decode_rope: the decode with rotary embeddings on q and K (the new rows
    already appended); workspace a uint8 device tensor of rope_workspace_bytes."""
    n_lanes = int(h_new.shape[0])
    _check(_load().tl_storeh_attn_decode_rope(ctypes.byref(cache.desc.c()), cache.c(), it, _ptr(loops), _ptr(ctx_len),
                                              _ptr(h_new), _ptr(W_q), _ptr(W_k), _ptr(W_v), _ptr(out),
                                              _ptr(residual), float(threshold), _ptr(abort_flags),
                                              _ptr(first_abort_iter), _ptr(norms_out), float(rope_base),
                                              _ptr(workspace), int(workspace.numel()), n_lanes, _stream(stream)),
           "tl_storeh_attn_decode_rope")


def residual_norm_check(residual, threshold: float, it: int, loops, abort_flags, first_abort_iter,
                        norms_out=None, stream=None) -> None:
    n_lanes, d = int(residual.shape[0]), int(residual.shape[1])
    _check(_load().tl_residual_norm_check(_ptr(residual), n_lanes, d, float(threshold), it, _ptr(loops),
                                      _ptr(abort_flags), _ptr(first_abort_iter), _ptr(norms_out), _stream(stream)),
           "tl_residual_norm_check")


def poll_status(cache, stream=None) -> int:
    """Synchronise and return (and clear) the device status of a workspace: a StoreHCache's,
    a DeltaCache's made with n_lanes, or a workspace tensor of its own (verification, prefill)."""
    if hasattr(cache, "workspace"):
        return _load().tl_storeh_poll_status(cache.workspace.data_ptr(), cache.ws_bytes, _stream(stream))
    return _load().tl_storeh_poll_status(cache.data_ptr(), int(cache.numel()), _stream(stream))


def selftest_wait_timeout(cache: StoreHCache, limit_cycles: int, stream=None) -> None:
    """Enqueue the self-test of the timeout path: a kernel whose only wait cannot complete gives
    up after limit_cycles SM clocks and records TL_ERR_DEVICE_TIMEOUT in the workspace."""
    _check(_load().tl_storeh_selftest_wait_timeout(cache.workspace.data_ptr(), cache.ws_bytes, int(limit_cycles),
                                                   _stream(stream)), "tl_storeh_selftest_wait_timeout")


class ProfileHook:
    """Context manager: counts the library's kernel launches on this thread and
    brackets every context-streaming kernel launch with CUDA events."""

    def __init__(self, capacity: int):
        import torch
        self.events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(capacity)]
        for b, e in self.events:      # torch creates the CUDA event on its first record
            b.record()
            e.record()
        torch.cuda.synchronize()
        self._b = (ctypes.c_void_p * capacity)(*[e[0].cuda_event for e in self.events])
        self._e = (ctypes.c_void_p * capacity)(*[e[1].cuda_event for e in self.events])
        self.p = Profile(self._b, self._e, capacity, 0, 0)

    def __enter__(self):
        _check(_load().tl_set_profile(ctypes.byref(self.p)), "tl_set_profile")
        return self

    def __exit__(self, *exc):
        _load().tl_set_profile(None)
        return False

    @property
    def launches(self) -> int:
        return int(self.p.launches)

    def stream_kernel_ms(self):
        """Durations (ms) of the bracketed streaming-kernel launches (call after a synchronize)."""
        return [b.elapsed_time(e) for b, e in self.events[: self.p.recorded]]
