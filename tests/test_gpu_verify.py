"""Multi-query attention over the store-h cache on the GPU, through the C ABI: tree
verification (tl_storeh_verify_attn) and chunked prefill (tl_storeh_prefill_attn)
[Architecture-Exclusive Features, "Tree speculative decoding"; "What this list is not":
chunked prefill].

Checks: every tree token's output against the tree oracle (max-abs 2e-3, relative L2 1e-3);
the appended tree rows bit-exact with the oracle's quantiser; a prefill chunk bit-identical to
the same tokens decoded one by one (the pages' "bit-identical to sequential generation");
inactive and out-of-range lanes left unwritten and reported.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import oracle.cpp
from oracle import tree_oracle
from synth.workloads import get_workload, small_variant

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from store_kv_attention_b200 import build_lib
    build_lib.build()


def _f16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).cuda()


def _workload(fmt, ctx, loops, L_max=2):
    base = {0: "fp16_407m", 1: "int8_b16", 2: "int4_2b"}[fmt]
    w = small_variant(get_workload(base), ctx=ctx, loops=loops, name=f"{base}_tree")
    return dataclasses.replace(w, L_max=L_max)


def _tree_states(w, it, K, D):
    """fp16 [B, K, D, d]: token (k, t) of lane b is the generator's row at position ctx + k D + t."""
    layer = w.n_pre + it
    return np.stack([w.h_rows(layer, b, w.ctx[b], K * D).reshape(K, D, w.d) for b in range(w.B)])


def _cache_rows(dw, layer, b, pos0, n):
    """Codes and scales of n rows of (layer, lane b) from the device cache."""
    w = dw.w
    mc = dw.desc.max_ctx
    cb = oracle.row_code_bytes(w.fmt, w.d)
    ns = oracle.row_scale_count(w.fmt, w.d)
    codes = dw.cache.codes[: w.n_layers * w.B * mc * cb].view(w.n_layers, w.B, mc, cb)[layer, b, pos0:pos0 + n]
    if ns == 0:
        return codes.cpu().numpy(), np.zeros((n, 0), np.float32)
    sdt = np.float32 if w.fmt == 1 else np.float16
    isz = np.dtype(sdt).itemsize
    sc = dw.cache.scales[: w.n_layers * w.B * mc * ns * isz].view(w.n_layers, w.B, mc, ns * isz)[layer, b, pos0:pos0 + n]
    return codes.cpu().numpy(), sc.cpu().numpy().view(sdt).reshape(n, ns)


def _close(got, want, tag):
    got = np.asarray(got, np.float64)
    assert np.all(np.isfinite(got)), tag
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err <= MAX_ABS and rel <= REL_L2, f"{tag}: max-abs {err:.3g} rel-L2 {rel:.3g}"


@pytest.mark.parametrize("fmt,ctx,K,D", [
    (0, [0, 37, 1100], 3, 4),      # FP16 (d = 1024, hi/lo operands); a lane with no cached position
    (1, [5, 1023, 300], 2, 5),     # INT8 per token with outlier rows; a context ending at a split edge
    (2, [130, 2049, 7], 4, 3),     # INT4 g64 (d = 2048); a context over two splits
    (2, [64, 700, 1500, 9], 4, 5),  # 80 query tokens: two groups of the decode kernels
])
def test_tree_verify_matches_oracle(fmt, ctx, K, D):
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    it = 1
    loops = [2] * len(ctx)
    loops[1] = 1                   # lane 1 is past its loop count at this iteration: not touched
    w = _workload(fmt, ctx, loops)
    dw = DeviceWorkload(w, max_ctx=max(ctx) + K * D + 3)
    h_tree = _tree_states(w, it, K, D)
    ws = torch.zeros(tl.verify_workspace_bytes(dw.desc, w.B, K, D), dtype=torch.uint8, device="cuda")
    out = torch.full((w.B, K, D, w.H, w.hd), float("nan"), dtype=torch.float32, device="cuda")
    tl.verify_attn(dw.cache, it, dw.loops, dw.ctx, _f16(h_tree), dw.W["q"], dw.W["k"], dw.W["v"], out, ws)
    torch.cuda.synchronize()
    assert tl.poll_status(ws) == tl.TL_OK
    got = out.cpu().numpy()
    W = [w.weight(k) for k in "qkv"]
    layer = w.n_pre + it
    for b in range(w.B):
        if it >= w.loops[b]:
            assert np.all(np.isnan(got[b])), f"inactive lane {b} was written"
            continue
        # the tree rows in the cache, bit-exact with the oracle's quantiser
        want_c, want_s = oracle.cpp.quantize_rows(h_tree[b].reshape(K * D, w.d), w.fmt)
        c, s = _cache_rows(dw, layer, b, w.ctx[b], K * D)
        assert np.array_equal(c, want_c) and np.array_equal(s.view(np.uint8), want_s.view(np.uint8))
        # every token against the tree oracle, over the rows as the cache holds them
        cc, cs = oracle.cpp.quantize_rows(w.h_rows(layer, b, 0, w.ctx[b]), w.fmt)
        h_ctx = oracle.cpp.dequantize_rows(cc, cs, w.fmt, w.d)
        h_rows = oracle.cpp.dequantize_rows(want_c, want_s, w.fmt, w.d).reshape(K, D, w.d)
        for k in range(K):
            for t in range(D):
                rows = tree_oracle.tree_rows(h_ctx, h_rows, k, t)
                want = oracle.cpp.attend_absorbed(rows, h_tree[b, k, t], *W, w.H, w.hd)
                _close(got[b, k, t], want, f"fmt {fmt} lane {b} branch {k} depth {t}")
    # the explicit-form tree oracle itself on one lane (its pinned definition)
    b = 0
    cc, cs = oracle.cpp.quantize_rows(w.h_rows(layer, b, 0, w.ctx[b]), w.fmt)
    tc, ts = oracle.cpp.quantize_rows(h_tree[b].reshape(K * D, w.d), w.fmt)
    want = tree_oracle.tree_verify(oracle.dequantize_rows(cc, cs, w.fmt, w.d),
                                   oracle.dequantize_rows(tc, ts, w.fmt, w.d).reshape(K, D, w.d), h_tree[b], *W,
                                   w.H, w.hd)
    for k in range(K):
        for t in range(D):
            _close(got[b, k, t], want[k, t], f"tree oracle lane 0 ({k}, {t})")


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_prefill_bitwise_equals_sequential_decodes(fmt):
    """A chunk of T tokens through tl_storeh_prefill_attn gives, token for token, the bits of T
    single-token decodes (append then decode with ctx_len + t cached positions)."""
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    ctx = [0, 200, 1021, 1500]
    T = 4                           # 4 lanes x 4 tokens: the same padded lane count as a 4-lane decode
    w = _workload(fmt, ctx, [2, 2, 2, 2])
    it = 1
    mc = max(ctx) + T + 1
    pre, seq = DeviceWorkload(w, max_ctx=mc), DeviceWorkload(w, max_ctx=mc, fill=False)
    seq.cache.codes.copy_(pre.cache.codes)
    if pre.cache.scales is not None:
        seq.cache.scales.copy_(pre.cache.scales)
    chunk = _tree_states(w, it, 1, T)[:, 0]  # [B, T, d]
    ws = torch.zeros(tl.verify_workspace_bytes(pre.desc, w.B, 1, T), dtype=torch.uint8, device="cuda")
    out = torch.full((w.B, T, w.H, w.hd), float("nan"), dtype=torch.float32, device="cuda")
    tl.prefill_attn(pre.cache, it, pre.loops, pre.ctx, _f16(chunk), pre.W["q"], pre.W["k"], pre.W["v"], out, ws)
    dec = torch.full_like(out, float("nan"))
    for t in range(T):
        ct = (seq.ctx + t).to(torch.int32)
        rows = _f16(chunk[:, t:t + 1])
        tl.append(seq.cache, w.n_pre + it, rows, ct, loops=seq.loops)
        o = torch.full((w.B, w.H, w.hd), float("nan"), dtype=torch.float32, device="cuda")
        tl.attn_decode(seq.cache, it, seq.loops, ct, rows[:, 0].contiguous(), seq.W["q"], seq.W["k"], seq.W["v"], o)
        dec[:, t] = o
    torch.cuda.synchronize()
    assert tl.poll_status(ws) == tl.TL_OK and tl.poll_status(seq.cache) == tl.TL_OK
    assert torch.equal(pre.cache.codes, seq.cache.codes)
    if pre.cache.scales is not None:
        assert torch.equal(pre.cache.scales, seq.cache.scales)
    a, b = out.cpu().numpy(), dec.cpu().numpy()
    assert np.all(np.isfinite(a))
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    # and one lane's tokens against the oracle
    W = [w.weight(k) for k in "qkv"]
    layer = w.n_pre + it
    for b_ in (0, 2):
        rows = np.concatenate([w.h_rows(layer, b_, 0, w.ctx[b_]), chunk[b_]])
        c, s = oracle.cpp.quantize_rows(rows, w.fmt)
        hh = oracle.cpp.dequantize_rows(c, s, w.fmt, w.d)
        for t in range(T):
            want = oracle.cpp.attend_absorbed(hh[: w.ctx[b_] + t + 1], chunk[b_, t], *W, w.H, w.hd)
            _close(a[b_, t], want, f"prefill fmt {fmt} lane {b_} token {t}")


def test_tree_that_does_not_fit_is_skipped_and_reported():
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    K, D = 2, 3
    w = _workload(2, [10, 50], [2, 2])
    dw = DeviceWorkload(w, max_ctx=55)     # lane 1: 50 + 6 > 55
    h_tree = _tree_states(w, 0, K, D)
    ws = torch.zeros(tl.verify_workspace_bytes(dw.desc, w.B, K, D), dtype=torch.uint8, device="cuda")
    out = torch.full((w.B, K, D, w.H, w.hd), float("nan"), dtype=torch.float32, device="cuda")
    tl.verify_attn(dw.cache, 0, dw.loops, dw.ctx, _f16(h_tree), dw.W["q"], dw.W["k"], dw.W["v"], out, ws)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.all(np.isfinite(got[0])) and np.all(np.isnan(got[1]))
    assert tl.poll_status(ws) == tl.TL_ERR_DEVICE_RANGE
    assert tl.poll_status(ws) == tl.TL_OK


def test_prefill_long_chunk_spans_groups():
    """A chunk of 70 tokens on 2 lanes (140 query tokens: three groups of the decode kernels),
    sampled tokens against the oracle, the chunk rows bit-exact in the cache."""
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    T = 70
    w = _workload(2, [900, 3], [2, 2])
    it = 0
    dw = DeviceWorkload(w, max_ctx=max(w.ctx) + T + 1)
    chunk = _tree_states(w, it, 1, T)[:, 0]
    ws = torch.zeros(tl.verify_workspace_bytes(dw.desc, w.B, 1, T), dtype=torch.uint8, device="cuda")
    out = torch.full((w.B, T, w.H, w.hd), float("nan"), dtype=torch.float32, device="cuda")
    tl.prefill_attn(dw.cache, it, dw.loops, dw.ctx, _f16(chunk), dw.W["q"], dw.W["k"], dw.W["v"], out, ws)
    torch.cuda.synchronize()
    assert tl.poll_status(ws) == tl.TL_OK
    got = out.cpu().numpy()
    assert np.all(np.isfinite(got))
    W = [w.weight(k) for k in "qkv"]
    layer = w.n_pre + it
    for b in range(w.B):
        rows = np.concatenate([w.h_rows(layer, b, 0, w.ctx[b]), chunk[b]])
        c, s = oracle.cpp.quantize_rows(rows, w.fmt)
        cc, cs = _cache_rows(dw, layer, b, 0, w.ctx[b] + T)
        assert np.array_equal(cc, c) and np.array_equal(cs.view(np.uint8), s.view(np.uint8))
        hh = oracle.cpp.dequantize_rows(c, s, w.fmt, w.d)
        for t in (0, 1, 63, 64, 69):
            want = oracle.cpp.attend_absorbed(hh[: w.ctx[b] + t + 1], chunk[b, t], *W, w.H, w.hd)
            _close(got[b, t], want, f"lane {b} token {t}")



@pytest.mark.parametrize("d,H,hd,fmt", [(768, 12, 64, 0), (1280, 10, 128, 2)], ids=["d768_fp16", "d1280_int4"])
def test_tree_verify_unusual_shapes(d, H, hd, fmt):
    """Tree verification where the projection kernels run on clusters of 4 (d_model / 64 = 12, 20)."""
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    from synth.workloads import Workload
    K, D, it = 2, 3, 0
    w = Workload(name=f"tree_d{d}", d=d, H=H, hd=hd, n_pre=1, L_max=1, fmt=fmt, seed=57, ctx=[0, 129, 1030],
                 loops=[1, 1, 1], residual_scale=1.0, threshold=50.0)
    dw = DeviceWorkload(w, max_ctx=max(w.ctx) + K * D + 1)
    h_tree = _tree_states(w, it, K, D)
    ws = torch.zeros(tl.verify_workspace_bytes(dw.desc, w.B, K, D), dtype=torch.uint8, device="cuda")
    out = torch.full((w.B, K, D, w.H, w.hd), float("nan"), dtype=torch.float32, device="cuda")
    tl.verify_attn(dw.cache, it, dw.loops, dw.ctx, _f16(h_tree), dw.W["q"], dw.W["k"], dw.W["v"], out, ws)
    torch.cuda.synchronize()
    assert tl.poll_status(ws) == tl.TL_OK
    got = out.cpu().numpy()
    W = [w.weight(k) for k in "qkv"]
    layer = w.n_pre + it
    for b in range(w.B):
        cc, cs = oracle.cpp.quantize_rows(w.h_rows(layer, b, 0, w.ctx[b]), w.fmt)
        h_ctx = oracle.cpp.dequantize_rows(cc, cs, w.fmt, w.d)
        tc, ts = oracle.cpp.quantize_rows(h_tree[b].reshape(K * D, w.d), w.fmt)
        h_rows = oracle.cpp.dequantize_rows(tc, ts, w.fmt, w.d).reshape(K, D, w.d)
        for k in range(K):
            for t in range(D):
                rows = tree_oracle.tree_rows(h_ctx, h_rows, k, t)
                want = oracle.cpp.attend_absorbed(rows, h_tree[b, k, t], *W, w.H, w.hd)
                _close(got[b, k, t], want, f"d {d} lane {b} branch {k} depth {t}")


def test_large_tree_over_groups_and_tiles():
    """8 branches x 20 tokens on 2 lanes: 320 query tokens in 5 groups of the decode kernels, each
    token's own-branch rows crossing a 128-row tile edge for the second lane."""
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    K, D, it = 8, 20, 0
    w = _workload(2, [5, 100], [1, 1], L_max=1)
    dw = DeviceWorkload(w, max_ctx=max(w.ctx) + K * D + 1)
    h_tree = _tree_states(w, it, K, D)
    ws = torch.zeros(tl.verify_workspace_bytes(dw.desc, w.B, K, D), dtype=torch.uint8, device="cuda")
    out = torch.full((w.B, K, D, w.H, w.hd), float("nan"), dtype=torch.float32, device="cuda")
    tl.verify_attn(dw.cache, it, dw.loops, dw.ctx, _f16(h_tree), dw.W["q"], dw.W["k"], dw.W["v"], out, ws)
    torch.cuda.synchronize()
    assert tl.poll_status(ws) == tl.TL_OK
    got = out.cpu().numpy()
    assert np.all(np.isfinite(got))
    W = [w.weight(k) for k in "qkv"]
    layer = w.n_pre + it
    for b in range(w.B):
        cc, cs = oracle.cpp.quantize_rows(w.h_rows(layer, b, 0, w.ctx[b]), w.fmt)
        h_ctx = oracle.cpp.dequantize_rows(cc, cs, w.fmt, w.d)
        tc, ts = oracle.cpp.quantize_rows(h_tree[b].reshape(K * D, w.d), w.fmt)
        h_rows = oracle.cpp.dequantize_rows(tc, ts, w.fmt, w.d).reshape(K, D, w.d)
        for k in (0, 3, 7):
            for t in (0, 1, 19):
                rows = tree_oracle.tree_rows(h_ctx, h_rows, k, t)
                want = oracle.cpp.attend_absorbed(rows, h_tree[b, k, t], *W, w.H, w.hd)
                _close(got[b, k, t], want, f"lane {b} branch {k} depth {t}")
