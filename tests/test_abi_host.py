"""The C-ABI library on the host (no GPU): it loads, exports every symbol the
header declares, sizes caches and workspaces, and rejects bad arguments
before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:TL_API\s+)?(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(tl_[a-z0-9_]+)\s*\(",
                                text, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def tl():
    from store_kv_attention_b200 import build_lib
    build_lib.build()
    import store_kv_attention_b200 as m
    return m


def test_exports_every_declared_symbol(tl):
    declared = _header_functions()
    assert len(declared) >= 9
    assert sorted(tl.EXPORTS) == declared
    raw = ctypes.CDLL(tl.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
    assert tl.lib.tl_storeh_abi_version() == 1


def _desc(tl, **kw):
    base = dict(d_model=2048, n_heads=16, head_dim=128, n_pre=2, L_max=8, max_lanes=32, max_ctx=4097,
                fmt=tl.TL_H_INT4_G64)
    base.update(kw)
    return tl.StoreHDesc(**base)


def test_cache_bytes_match_layout(tl):
    cb, sb = tl.cache_bytes(_desc(tl))
    rows = 10 * 32 * 4097
    assert cb == rows * 1024 and sb == rows * 32 * 2
    cb, sb = tl.cache_bytes(_desc(tl, fmt=tl.TL_H_INT8_TOKEN, d_model=1024, n_heads=16, head_dim=64))
    assert cb == rows * 1024 and sb == rows * 4
    cb, sb = tl.cache_bytes(_desc(tl, fmt=tl.TL_H_FP16, d_model=1024, n_heads=16, head_dim=64))
    assert cb == rows * 2048 and sb == 0


def test_workspace_bytes(tl):
    b = tl.workspace_bytes(_desc(tl), 32)
    assert b % 256 == 0 and b > 32 * 16 * 2048 * 4
    with pytest.raises(tl.TLError) as e:
        tl.workspace_bytes(_desc(tl), 33)
    assert e.value.status == tl.TL_ERR_CAPACITY


@pytest.mark.parametrize("kw,status", [
    (dict(d_model=2048, n_heads=15), 2),          # d != H * hd -> TL_ERR_SHAPE
    (dict(head_dim=96, n_heads=16, d_model=1536), 4),
    (dict(d_model=2304, n_heads=18, head_dim=128), 4),
    (dict(d_model=4096, n_heads=32, head_dim=128), 4),
    (dict(n_heads=32, head_dim=64, d_model=2048), 4),
    (dict(fmt=7), 1),
    (dict(max_ctx=0), 1),
    (dict(max_ctx=70000), 4),
    (dict(L_max=0), 1),
])
def test_desc_validation(tl, kw, status):
    with pytest.raises(tl.TLError) as e:
        tl.cache_bytes(_desc(tl, **kw))
    assert e.value.status == status


def test_calls_rejected_before_launch(tl):
    L = tl.lib
    d = _desc(tl).c()
    fake = ctypes.c_void_p(1 << 20)          # 256-aligned stand-in, never dereferenced
    cache = tl.Cache(1 << 20, 1 << 21)
    # NULL descriptor
    assert L.tl_storeh_append(None, cache, 0, fake, 1, 1, fake, None, None, None) == tl.TL_ERR_INVALID_ARG
    # lanes beyond capacity, layer outside the cache
    assert L.tl_storeh_append(ctypes.byref(d), cache, 0, fake, 33, 1, fake, None, None, None) == tl.TL_ERR_CAPACITY
    assert L.tl_storeh_append(ctypes.byref(d), cache, 10, fake, 1, 1, fake, None, None, None) == tl.TL_ERR_CAPACITY
    # misaligned cache
    bad = tl.Cache((1 << 20) + 16, 1 << 21)
    assert L.tl_storeh_append(ctypes.byref(d), bad, 0, fake, 1, 1, fake, None, None, None) == tl.TL_ERR_INVALID_ARG
    # zero rows is a no-op
    assert L.tl_storeh_append(ctypes.byref(d), cache, 0, fake, 1, 0, fake, None, None, None) == tl.TL_OK
    ws = tl.workspace_bytes(_desc(tl), 4)
    args = lambda it, n, wsb, res=None, flags=None: (ctypes.byref(d), cache, it, fake, fake, fake, fake, fake, fake,
                                                     fake, res, 50.0, flags, flags, None, fake, wsb, n, None)
    assert L.tl_storeh_attn_decode(*args(8, 4, ws)) == tl.TL_ERR_CAPACITY        # iter >= L_max
    assert L.tl_storeh_attn_decode(*args(0, 4, ws - 256)) == tl.TL_ERR_CAPACITY  # workspace too small
    assert L.tl_storeh_attn_decode(*args(0, 0, ws)) == tl.TL_ERR_INVALID_ARG
    assert L.tl_storeh_attn_decode(*args(0, 4, ws, res=fake)) == tl.TL_ERR_INVALID_ARG  # residual w/o flags
    assert L.tl_residual_norm_check(None, 1, 8, 1.0, 0, None, fake, fake, None, None) == tl.TL_ERR_INVALID_ARG
    assert L.tl_residual_norm_check(fake, 1, 8, float("nan"), 0, None, fake, fake, None, None) == tl.TL_ERR_INVALID_ARG
    assert b"threshold" in L.tl_last_error_message()
    assert L.tl_status_string(tl.TL_ERR_DEVICE_TIMEOUT).startswith(b"TL_ERR_DEVICE_TIMEOUT")


# --------------------------------------------------------------------------- delta cache (tl_delta.h)
def test_delta_cache_bytes_match_layout(tl):
    a, d, s = tl.delta_cache_bytes(tl.DeltaDesc(2048, 16, 128, 8, 32, 4097))
    rows = 32 * 4097
    assert (a, d, s) == (rows * 2048 * 2, 7 * rows * 2048, 7 * rows * 16 * 2)
    assert tl.delta_cache_bytes(tl.DeltaDesc(256, 4, 64, 1, 2, 10)) == (2 * 10 * 256 * 2, 0, 0)


@pytest.mark.parametrize("kw,status", [
    (dict(n_heads=15), 2),
    (dict(head_dim=96, n_heads=16, d_model=1536), 4),
    (dict(d_model=4096, n_heads=32), 4),
    (dict(L_max=0), 1),
    (dict(max_ctx=0), 1),
])
def test_delta_desc_validation(tl, kw, status):
    base = dict(d_model=2048, n_heads=16, head_dim=128, L_max=8, max_lanes=32, max_ctx=4097)
    base.update(kw)
    with pytest.raises(tl.TLError) as e:
        tl.delta_cache_bytes(tl.DeltaDesc(**base))
    assert e.value.status == status


def test_delta_append_rejected_before_launch(tl):
    L = tl.lib
    d = tl.DeltaDesc(2048, 16, 128, 4, 2, 64).c()
    fake = ctypes.c_void_p(1 << 20)
    cache = tl.DeltaCacheC(1 << 20, 1 << 21, 1 << 22)
    assert L.tl_delta_append(None, cache, 0, fake, 1, 1, fake, None, None) == tl.TL_ERR_INVALID_ARG
    assert L.tl_delta_append(ctypes.byref(d), cache, 4, fake, 1, 1, fake, None, None) == tl.TL_ERR_CAPACITY
    assert L.tl_delta_append(ctypes.byref(d), cache, -1, fake, 1, 1, fake, None, None) == tl.TL_ERR_CAPACITY
    assert L.tl_delta_append(ctypes.byref(d), cache, 0, fake, 3, 1, fake, None, None) == tl.TL_ERR_CAPACITY
    bad = tl.DeltaCacheC((1 << 20) + 16, 1 << 21, 1 << 22)
    assert L.tl_delta_append(ctypes.byref(d), bad, 0, fake, 1, 1, fake, None, None) == tl.TL_ERR_INVALID_ARG
    no_deltas = tl.DeltaCacheC(1 << 20, None, None)
    assert L.tl_delta_append(ctypes.byref(d), no_deltas, 1, fake, 1, 1, fake, None, None) == tl.TL_ERR_INVALID_ARG
    assert L.tl_delta_append(ctypes.byref(d), cache, 1, ctypes.c_void_p((1 << 20) + 8), 1, 1, fake, None,
                             None) == tl.TL_ERR_INVALID_ARG
    assert L.tl_delta_append(ctypes.byref(d), cache, 0, fake, 1, 0, fake, None, None) == tl.TL_OK


def test_delta_workspace_and_decode_rejected_before_launch(tl):
    desc = tl.DeltaDesc(2048, 16, 128, 4, 4, 1000)
    ws = tl.delta_workspace_bytes(desc, 2)
    sdesc = tl.StoreHDesc(2048, 16, 128, n_pre=0, L_max=1, max_lanes=2, max_ctx=1000, fmt=tl.TL_H_FP16)
    # the decode workspace (with hi and lo query images: 2 lanes x 16 more rows x d fp16) and two
    # small per-lane arrays; the rows are rebuilt inside the streaming kernel, with no scratch copy
    base = tl.workspace_bytes(sdesc, 2, split_rows=256) + 2 * 16 * 2048 * 2  # 256-row splits
    assert base < ws < base + 4096 and ws % 256 == 0
    with pytest.raises(tl.TLError) as e:
        tl.delta_workspace_bytes(desc, 5)
    assert e.value.status == tl.TL_ERR_CAPACITY
    with pytest.raises(tl.TLError) as e:
        tl.delta_workspace_bytes(tl.DeltaDesc(2048, 32, 64, 4, 4, 1000), 2)  # 32 heads
    assert e.value.status == tl.TL_ERR_UNSUPPORTED
    L = tl.lib
    d = desc.c()
    fake = ctypes.c_void_p(1 << 20)
    cache = tl.DeltaCacheC(1 << 20, 1 << 21, 1 << 22)
    args = lambda it, n, wsb, ws_ptr=fake, res=None, flags=None: (
        ctypes.byref(d), cache, it, fake, fake, fake, fake, fake, fake, fake, res, ctypes.c_float(50.0), flags, None,
        None, ws_ptr, wsb, n, None)
    assert L.tl_delta_attn_decode(*args(4, 2, ws)) == tl.TL_ERR_CAPACITY          # iter outside [0, L_max)
    assert L.tl_delta_attn_decode(*args(0, 5, ws)) == tl.TL_ERR_CAPACITY          # lanes beyond the cache
    assert L.tl_delta_attn_decode(*args(0, 2, ws - 256)) == tl.TL_ERR_CAPACITY    # workspace too small
    assert L.tl_delta_attn_decode(*args(0, 2, ws, ws_ptr=ctypes.c_void_p((1 << 20) + 16))) == tl.TL_ERR_INVALID_ARG
    assert L.tl_delta_attn_decode(*args(0, 2, ws, res=fake)) == tl.TL_ERR_INVALID_ARG  # residual without flags
    assert L.tl_delta_attn_decode(None, cache, 0, fake, fake, fake, fake, fake, fake, fake, None,
                                  ctypes.c_float(0.0), None, None, None, fake, ws, 2, None) == tl.TL_ERR_INVALID_ARG


# --------------------------------------------------------------------------- tree verification, prefill
def test_verify_and_prefill_rejected_before_launch(tl):
    L = tl.lib
    desc = _desc(tl)
    d = desc.c()
    fake = ctypes.c_void_p(1 << 20)
    cache = tl.Cache(1 << 20, 1 << 21)
    ws = tl.verify_workspace_bytes(desc, 2, 3, 4)
    assert ws >= tl.workspace_bytes(desc, 24) and ws % 256 == 0
    args = lambda it, n, K, D, wsb: (ctypes.byref(d), cache, it, fake, fake, fake, K, D, fake, fake, fake, fake, fake,
                                     wsb, n, None)
    assert L.tl_storeh_verify_attn(*args(0, 2, 3, 4, ws - 256)) == tl.TL_ERR_CAPACITY   # workspace too small
    assert L.tl_storeh_verify_attn(*args(8, 2, 3, 4, ws)) == tl.TL_ERR_CAPACITY         # iter >= L_max
    assert L.tl_storeh_verify_attn(*args(0, 33, 3, 4, ws)) == tl.TL_ERR_CAPACITY        # lanes beyond capacity
    assert L.tl_storeh_verify_attn(*args(0, 2, 0, 4, ws)) == tl.TL_ERR_INVALID_ARG
    assert L.tl_storeh_verify_attn(*args(0, 2, 33, 32, ws)) == tl.TL_ERR_UNSUPPORTED    # > 1024 tree tokens
    nul = (ctypes.byref(d), cache, 0, fake, fake, None, 3, 4, fake, fake, fake, fake, fake, ws, 2, None)
    assert L.tl_storeh_verify_attn(*nul) == tl.TL_ERR_INVALID_ARG                       # h_tree NULL
    assert L.tl_storeh_prefill_attn(ctypes.byref(d), cache, 0, fake, fake, fake, 0, fake, fake, fake, fake, fake, ws,
                                    2, None) == tl.TL_ERR_INVALID_ARG                    # no tokens
    with pytest.raises(tl.TLError):
        tl.verify_workspace_bytes(desc, 2, 40, 40)


def test_decode_options_rejected_before_launch(tl):
    L = tl.lib
    desc = _desc(tl)
    d = desc.c()
    fake = ctypes.c_void_p(1 << 20)
    cache = tl.Cache(1 << 20, 1 << 21)
    b = ctypes.c_size_t()
    for split, want in ((0, tl.TL_OK), (128, tl.TL_OK), (512, tl.TL_OK), (100, tl.TL_ERR_INVALID_ARG),
                        (2048, tl.TL_ERR_INVALID_ARG), (-1, tl.TL_ERR_INVALID_ARG)):
        opts = tl.DecodeOpts(0, split)
        assert L.tl_storeh_workspace_bytes_ex(ctypes.byref(d), 4, ctypes.byref(opts), ctypes.byref(b)) == want, split
    # shorter splits need more partial results
    assert tl.workspace_bytes(desc, 4, 128) > tl.workspace_bytes(desc, 4, 1024) == tl.workspace_bytes(desc, 4)
    opts = tl.DecodeOpts(0, 128)
    opts.reserved[3] = 1
    assert L.tl_storeh_workspace_bytes_ex(ctypes.byref(d), 4, ctypes.byref(opts), ctypes.byref(b)) == tl.TL_ERR_INVALID_ARG
    ws = tl.workspace_bytes(desc, 4, 128)
    args = lambda o, wsb: (ctypes.byref(d), cache, 0, fake, fake, fake, fake, fake, fake, fake, None, 0.0, None, None,
                           None, fake, wsb, 4, o, None)
    assert L.tl_storeh_decode_ex(*args(None, ws)) == tl.TL_ERR_INVALID_ARG
    assert L.tl_storeh_decode_ex(*args(ctypes.byref(tl.DecodeOpts(2, 128)), ws)) == tl.TL_ERR_INVALID_ARG
    # the default-split workspace is too small for 128-row splits
    assert L.tl_storeh_decode_ex(*args(ctypes.byref(tl.DecodeOpts(0, 128)), tl.workspace_bytes(desc, 4))) == \
        tl.TL_ERR_CAPACITY
    # 65536 positions in splits of 128 rows for 64 lanes: the merge state does not fit
    big = tl.StoreHDesc(2048, 16, 128, n_pre=1, L_max=2, max_lanes=64, max_ctx=65536, fmt=2)
    with pytest.raises(tl.TLError) as e:
        tl.workspace_bytes(big, 64, 128)
    assert e.value.status == tl.TL_ERR_UNSUPPORTED


def test_rope_decode_rejected_before_launch(tl):
    L = tl.lib
    desc = _desc(tl)
    d = desc.c()
    fake = ctypes.c_void_p(1 << 20)
    cache = tl.Cache(1 << 20, 1 << 21)
    ws = tl.rope_workspace_bytes(desc, 4)
    assert ws > tl.workspace_bytes(desc, 4)
    args = lambda it, base, wsb: (ctypes.byref(d), cache, it, fake, fake, fake, fake, fake, fake, fake, None, 0.0, None,
                                  None, None, base, fake, wsb, 4, None)
    assert L.tl_storeh_attn_decode_rope(*args(0, 10000.0, ws - 256)) == tl.TL_ERR_CAPACITY
    assert L.tl_storeh_attn_decode_rope(*args(8, 10000.0, ws)) == tl.TL_ERR_CAPACITY
    assert L.tl_storeh_attn_decode_rope(*args(0, 1.0, ws)) == tl.TL_ERR_INVALID_ARG
    assert L.tl_storeh_attn_decode_rope(*args(0, float("nan"), ws)) == tl.TL_ERR_INVALID_ARG
