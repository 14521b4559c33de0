"""Parity of the CUDA path (through the C ABI) with the plain C++ CPU oracle (oracle/cpp.py).

Bars: codes and scales bit-exact; abort flags and first-abort iterations
identical; attention outputs within max-abs 2e-3 and relative L2 1e-3 of the
oracle per (lane, iteration); a mixed-batch lane bitwise equal to its solo
run; nothing outside a lane's layers and positions is read.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.cpp
import synth
from synth.workloads import get_workload, select_lanes, small_variant

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from store_kv_attention_b200 import build_lib
    build_lib.build()


def _dw(w, **kw):
    from synth.device import DeviceWorkload
    return DeviceWorkload(w, **kw)


def _oracle_lane(w, it, b, form="explicit"):
    layer = w.n_pre + it
    rows = np.concatenate([w.h_rows(layer, b, 0, w.ctx[b]), w.h_new(it)[b:b + 1]])
    codes, scales = oracle.cpp.quantize_rows(rows, w.fmt)
    hh = oracle.cpp.dequantize_rows(codes, scales, w.fmt, w.d)
    W = [w.weight(k) for k in "qkv"]
    f = oracle.cpp.attend_explicit if form == "explicit" else oracle.attend_absorbed
    return f(hh, w.h_new(it)[b], *W, w.H, w.hd)


def _assert_close(got, want, tag):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), tag
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err.max() <= MAX_ABS and rel <= REL_L2, f"{tag}: max-abs {err.max():.3g} rel-L2 {rel:.3g}"
    return err.max(), rel


# --------------------------------------------------------------------------- append: codes
@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_append_codes_bit_exact(fmt):
    import store_kv_attention_b200 as tl
    d = 2048 if fmt == 2 else 1024
    H, hd = (16, 128) if fmt == 2 else (16, 64)
    rng = np.random.default_rng(11 + fmt)
    n = 300
    h = (rng.standard_normal((n, d)) * np.exp(rng.uniform(-4, 4, (n, 1)))).astype(np.float16)
    h[0] = 0                                                 # zero row -> scale 0, codes 0
    h[1, :64] = np.array([7, 0.5, 1.5, 2.5, 3.5, -3.5, 6.5, -7] * 8, np.float16)  # ties
    h[2] = np.float16(1e-7)                                  # fp16 subnormals
    h[3, ::2] *= np.float16(100)                            # wide range inside a row
    desc = tl.StoreHDesc(d, H, hd, n_pre=1, L_max=2, max_lanes=2, max_ctx=n + 5, fmt=fmt)
    cache = tl.StoreHCache(desc)
    cache.codes.fill_(0xAB)
    if cache.scales is not None:
        cache.scales.fill_(0xCD)
    hd_t = torch.from_numpy(h.view(np.int16)).view(torch.float16).cuda()
    rows = torch.stack([hd_t, hd_t.flip(0)])                 # lane 1 gets the rows reversed
    start = torch.tensor([3, 0], dtype=torch.int32, device="cuda")
    tl.append(cache, 2, rows, start)
    torch.cuda.synchronize()
    cb = oracle.row_code_bytes(fmt, d)
    codes = cache.codes.view(3, 2, n + 5, cb).cpu().numpy()
    for lane, src, p0 in ((0, h, 3), (1, h[::-1].copy(), 0)):
        want_c, want_s = oracle.cpp.quantize_rows(src, fmt)
        assert np.array_equal(codes[2, lane, p0:p0 + n], want_c), f"codes lane {lane}"
        if fmt != 0:
            ns = oracle.row_scale_count(fmt, d)
            sdt = np.float32 if fmt == 1 else np.float16
            sc = cache.scales.view(-1)[:3 * 2 * (n + 5) * ns * np.dtype(sdt).itemsize].cpu().numpy()
            sc = sc.view(sdt).reshape(3, 2, n + 5, ns)
            assert np.array_equal(sc[2, lane, p0:p0 + n].view(np.uint8), want_s.astype(sdt).view(np.uint8))
    # untouched positions stay untouched
    assert np.all(codes[2, 0, :3] == 0xAB) and np.all(codes[2, 1, n:] == 0xAB) and np.all(codes[:2] == 0xAB)


def test_append_skips_lanes_past_their_loops_and_out_of_range_rows():
    import store_kv_attention_b200 as tl
    d, H, hd = 256, 4, 64
    desc = tl.StoreHDesc(d, H, hd, n_pre=1, L_max=3, max_lanes=3, max_ctx=8, fmt=0)
    cache = tl.StoreHCache(desc)
    cache.codes.fill_(0)
    rows = torch.ones((3, 4, d), dtype=torch.float16, device="cuda")
    loops = torch.tensor([1, 2, 3], dtype=torch.int32, device="cuda")
    start = torch.tensor([0, 6, 0], dtype=torch.int32, device="cuda")     # lane 1 runs past max_ctx
    count = torch.tensor([4, 4, 2], dtype=torch.int32, device="cuda")
    tl.append(cache, 2, rows, start, row_count=count, loops=loops)         # layer 2 = iteration 1
    torch.cuda.synchronize()
    c = cache.codes.view(4, 3, 8, 2 * d).cpu().numpy().view(np.float16)
    assert np.all(c[2, 0] == 0)                        # loops=1: layer 2 is beyond the lane's depth
    assert np.all(c[2, 1, 6:8] == 1) and np.all(c[2, 1, :6] == 0)
    assert np.all(c[2, 2, :2] == 1) and np.all(c[2, 2, 2:] == 0)


# --------------------------------------------------------------------------- safety check
@pytest.mark.parametrize("flag_mix", [False, True])
def test_norm_flags_identical(flag_mix):
    import store_kv_attention_b200 as tl
    w = get_workload("int4_mixed")
    res = [w.residual(it, flag_mix) for it in range(6)]
    loops = np.array(w.loops, np.int32)
    loops[5] = 0
    f = np.zeros(w.B, np.uint8)
    fi = np.full(w.B, -1, np.int32)
    df = torch.zeros(w.B, dtype=torch.uint8, device="cuda")
    dfi = torch.full((w.B,), -1, dtype=torch.int32, device="cuda")
    dl = torch.from_numpy(loops).cuda()
    for it in range(6):
        r = res[it].copy()
        if it == 2:
            r *= 0.01          # a quiet iteration: flags stay sticky
        f, fi, nrm = oracle.cpp.residual_norm_check(r, w.threshold, it, loops, f, fi)
        dn = torch.full((w.B,), float("nan"), device="cuda")
        tl.residual_norm_check(torch.from_numpy(r).cuda(), w.threshold, it, dl, df, dfi, norms_out=dn)
        torch.cuda.synchronize()
        assert np.array_equal(df.cpu().numpy(), f) and np.array_equal(dfi.cpu().numpy(), fi)
        act = ~np.isnan(nrm)
        assert np.allclose(dn.cpu().numpy()[act], nrm[act], rtol=1e-6)
    if flag_mix:
        assert 0 < f.sum() < w.B


# --------------------------------------------------------------------------- decode: small sizes
SMALL = [
    ("tiny_fp16", None, None),
    ("fp16_407m", [0, 1, 127, 128, 129, 1030, 2200], [8, 3, 8, 1, 5, 8, 2]),
    ("int8_b16", [0, 5, 255, 1023, 1024, 2047, 2049], [8, 8, 2, 7, 8, 4, 8]),
    ("int4_2b", [0, 3, 130, 1000, 1025, 2048, 3000], [8, 1, 8, 6, 8, 8, 3]),
    ("int4_mixed", [1, 129, 700, 1024, 2500, 64], [4, 16, 32, 4, 16, 32]),
]


def _small(name, ctx, loops):
    w = get_workload(name)
    if ctx is None:
        return w
    return small_variant(w, ctx=ctx, loops=loops, name=name + "_small")


@pytest.mark.parametrize("name,ctx,loops", SMALL, ids=[s[0] for s in SMALL])
def test_decode_matches_oracle_small(name, ctx, loops):
    w = _small(name, ctx, loops)
    dw = _dw(w, flag_mix=True)
    dw.step()
    torch.cuda.synchronize()
    out = dw.out.cpu().numpy()
    f = np.zeros(w.B, np.uint8)
    fi = np.full(w.B, -1, np.int32)
    its = range(w.L_max) if w.L_max <= 8 else [0, 3, 4, 15, 16, 31]
    for it in range(w.L_max):
        for b in range(w.B):
            active = it < w.loops[b]
            if not active:
                assert np.all(np.isnan(out[it, b])), f"inactive lane {b} iteration {it} was written"
            elif it in its:
                _assert_close(out[it, b], _oracle_lane(w, it, b), f"{name} lane {b} it {it}")
        f, fi, _ = oracle.cpp.residual_norm_check(w.residual(it, True), w.threshold, it, np.array(w.loops), f, fi)
    assert np.array_equal(dw.flags.cpu().numpy(), f) and np.array_equal(dw.first.cpu().numpy(), fi)
    import store_kv_attention_b200 as tl
    assert tl.poll_status(dw.cache) == tl.TL_OK


def test_mixed_batch_lane_bitwise_equals_solo():
    """Architecture-Exclusive Features, "L-aware batching": a lane of a mixed batch
    gives bit-for-bit the result of the same lane run alone."""
    w = _small("int4_mixed", [1, 129, 700, 1024, 2500, 64], [4, 16, 32, 4, 16, 32])
    mixed = _dw(w)
    mixed.step()
    torch.cuda.synchronize()
    a_all = mixed.out.cpu().numpy()
    for b in (1, 4, 5):
        solo = _dw(select_lanes(w, [b]))
        solo.step()
        torch.cuda.synchronize()
        s = solo.out[:, 0].cpu().numpy()
        assert np.array_equal(a_all[:, b].view(np.uint32), s.view(np.uint32)), f"lane {b}"
        assert solo.flags.item() == mixed.flags[b].item() and solo.first.item() == mixed.first[b].item()


def test_poisoned_layers_and_positions_are_not_read():
    import store_kv_attention_b200 as tl
    w = _small("int8_b16", [3, 300, 1100], [2, 8, 5])
    clean = _dw(w)
    clean.step()
    dirty = _dw(w, fill=False)
    # poison everything first (0x7f / 0x80 int8 codes and NaN scales), then write the real rows
    dirty.cache.codes.fill_(0x7F)
    dirty.cache.scales.view(torch.float32)[:].fill_(float("nan"))
    dirty.fill_context()
    dirty.step()
    torch.cuda.synchronize()
    a, b = clean.out.cpu().numpy(), dirty.out.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert tl.poll_status(dirty.cache) == tl.TL_OK


def test_out_of_range_lane_is_skipped_and_reported():
    import store_kv_attention_b200 as tl
    w = _small("tiny_fp16", [5, 9], [2, 2])
    w.L_max = 2
    dw = _dw(w)
    dw.ctx[1] = w.max_ctx + 7           # beyond the cache
    dw.append_new(0)                    # lane 1's row is not written: its position is out of range
    dw.decode(0)
    torch.cuda.synchronize()
    out = dw.out[0].cpu().numpy()
    assert np.all(np.isfinite(out[0])) and np.all(np.isnan(out[1]))
    assert tl.poll_status(dw.cache) == tl.TL_ERR_DEVICE_RANGE
    assert tl.poll_status(dw.cache) == tl.TL_OK        # cleared by the poll


# --------------------------------------------------------------------------- decode: full sizes, sampled
# The benchmarked entry point (tl_storeh_append_attn_decode) at the benchmarked sizes, against
# the separate append + decode calls on a copy of the same cache (whole cache byte for byte,
# outputs bit for bit), the oracle's quantiser (every appended row), the oracle's attention
# (sampled lanes: the forced-abort lanes, the last lane) and the oracle's safety check.
FULL = [
    ("fp16_407m", [(it, 0) for it in range(8)]),
    ("int8_b16", [(0, 0), (3, 7), (7, 15)]),
    ("int4_2b", [(0, 0), (7, 1), (4, 17), (7, 31)]),
    ("int4_mixed", [(0, 0), (3, 1), (3, 15), (10, 20), (31, 47), (15, 33)]),
]


def _new_rows_from_cache(dw, it):
    """Codes and scales of every lane's row at (layer n_pre + it, position ctx[b]), from the device."""
    w = dw.w
    cb = oracle.row_code_bytes(w.fmt, w.d)
    ns = oracle.row_scale_count(w.fmt, w.d)
    codes = dw.cache.codes[: w.n_layers * w.B * w.max_ctx * cb].view(w.n_layers, w.B, w.max_ctx, cb)
    lanes = torch.arange(w.B, device=dw.ctx.device)
    c = codes[w.n_pre + it, lanes, dw.ctx.long()].cpu().numpy()
    if ns == 0:
        return c, None
    sdt = np.float32 if w.fmt == 1 else np.float16
    nbytes = w.n_layers * w.B * w.max_ctx * ns * np.dtype(sdt).itemsize
    sc = dw.cache.scales[:nbytes].view(w.n_layers, w.B, w.max_ctx, ns * np.dtype(sdt).itemsize)
    return c, sc[w.n_pre + it, lanes, dw.ctx.long()].cpu().numpy().view(sdt)


@pytest.mark.parametrize("name,samples", FULL, ids=[f[0] for f in FULL])
def test_decode_full_size_sampled(name, samples):
    import store_kv_attention_b200 as tl
    w = get_workload(name)
    fus = _dw(w)
    sep = _dw(w, fill=False)
    sep.cache.codes.copy_(fus.cache.codes)
    if fus.cache.scales is not None:
        sep.cache.scales.copy_(fus.cache.scales)
    act = np.array([[it < w.loops[b] for b in range(w.B)] for it in range(w.L_max)])
    # both residual variants: literal (every lane over the threshold) and flag-mix
    for flag_mix in (False, True):
        res = torch.stack([torch.from_numpy(w.residual(it, flag_mix)) for it in range(w.L_max)]).cuda()
        for dw in (fus, sep):
            dw.residual = res
            dw.reset_flags()
            dw.out.fill_(float("nan"))
        fus.step(fused_append=True)
        sep.step()
        torch.cuda.synchronize()
        assert torch.equal(fus.cache.codes, sep.cache.codes)
        if fus.cache.scales is not None:
            assert torch.equal(fus.cache.scales, sep.cache.scales)
        out = fus.out.cpu().numpy()
        assert np.array_equal(out.view(np.uint32), sep.out.cpu().numpy().view(np.uint32))
        assert torch.equal(fus.flags, sep.flags) and torch.equal(fus.first, sep.first)
        f = np.zeros(w.B, np.uint8)
        fi = np.full(w.B, -1, np.int32)
        for it in range(w.L_max):
            f, fi, _ = oracle.cpp.residual_norm_check(w.residual(it, flag_mix), w.threshold, it, np.array(w.loops), f, fi)
        assert np.array_equal(fus.flags.cpu().numpy(), f) and np.array_equal(fus.first.cpu().numpy(), fi)
        if flag_mix and w.B > 1:
            assert 0 < f.sum() < w.B
        # every active (lane, iteration) was written, every inactive one was not
        assert np.all(np.isfinite(out[act])) and np.all(np.isnan(out[~act]))
    # the new token's row of every active (lane, iteration), bit-exact with the oracle's quantiser
    for it in range(w.L_max):
        bs = [b for b in range(w.B) if act[it, b]]
        want_c, want_s = oracle.cpp.quantize_rows(w.h_new(it)[bs], w.fmt)
        got_c, got_s = _new_rows_from_cache(fus, it)
        assert np.array_equal(got_c[bs], want_c), f"{name} codes of iteration {it}"
        if got_s is not None:
            assert np.array_equal(got_s[bs].view(np.uint8), want_s.astype(got_s.dtype).view(np.uint8))
    for it, b in samples:
        assert it < w.loops[b]
        _assert_close(out[it, b], _oracle_lane(w, it, b, form="absorbed"), f"{name} lane {b} it {it}")
    assert tl.poll_status(fus.cache) == tl.TL_OK and tl.poll_status(sep.cache) == tl.TL_OK


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_fused_append_more_lanes_than_ctas(fmt):
    """d = 256 runs the projection kernels on 8 CTAs, so with 40 lanes the fused append's lane
    loop and the safety check's lane loop make several trips per CTA (lanes 0-19 over the
    threshold, 20-39 under it)."""
    import dataclasses
    base = get_workload("tiny_fp16")
    n = 40
    ctx = [(53 * b * b + 17 * b) % 700 for b in range(n)]
    ctx[3], ctx[5] = 0, 1
    loops = [1 + (b % 3) for b in range(n)]
    w = dataclasses.replace(base, fmt=fmt, ctx=ctx, loops=loops, L_max=3, name=f"d256_fmt{fmt}_40lanes",
                            outlier_p=0.01 if fmt == 1 else 0.0, outlier_mul=8.0, forced_lanes=20)
    sep, fus = _dw(w, flag_mix=True, fill=False), _dw(w, flag_mix=True, fill=False)
    for dw in (sep, fus):
        dw.cache.codes.fill_(0x5A)
        if dw.cache.scales is not None:
            dw.cache.scales.fill_(0x5A)
        dw.fill_context()
    sep.step()
    fus.step(fused_append=True)
    torch.cuda.synchronize()
    assert torch.equal(sep.cache.codes, fus.cache.codes)
    if sep.cache.scales is not None:
        assert torch.equal(sep.cache.scales, fus.cache.scales)
    a = fus.out.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), sep.out.cpu().numpy().view(np.uint32))
    assert torch.equal(sep.flags, fus.flags) and torch.equal(sep.first, fus.first)
    # the safety check of every lane (more lanes than CTAs: each CTA checks several)
    f = np.zeros(w.B, np.uint8)
    fi = np.full(w.B, -1, np.int32)
    for it in range(w.L_max):
        f, fi, _ = oracle.cpp.residual_norm_check(w.residual(it, True), w.threshold, it, np.array(w.loops), f, fi)
    assert 0 < f.sum() < w.B
    assert np.array_equal(fus.flags.cpu().numpy(), f) and np.array_equal(fus.first.cpu().numpy(), fi)
    for it in range(w.L_max):
        bs = [b for b in range(w.B) if it < w.loops[b]]
        want_c, want_s = oracle.cpp.quantize_rows(w.h_new(it)[bs], w.fmt)
        got_c, got_s = _new_rows_from_cache(fus, it)
        assert np.array_equal(got_c[bs], want_c)
        if got_s is not None:
            assert np.array_equal(got_s[bs].view(np.uint8), want_s.astype(got_s.dtype).view(np.uint8))
        for b in (bs[0], bs[len(bs) // 2], bs[-1]):
            _assert_close(a[it, b], _oracle_lane(w, it, b), f"{w.name} lane {b} it {it}")


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["fp16_407m", "int8_b16", "int4_2b"])
def test_decode_bitwise_reproducible(name):
    """Repeating a decode gives bit-identical outputs.  Every reduction has a fixed order,
    so any difference comes from a pipeline hand-off that read data before it was ready
    (for instance a ring slot whose parity was taken from an earlier use)."""
    w = _small(name, [127, 1000, 2047], [2, 2, 2])
    dw = _dw(w)
    dw.step()
    torch.cuda.synchronize()
    ref = dw.out[0].cpu().numpy().copy()
    for _ in range(6):
        dw.decode(0)
        torch.cuda.synchronize()
        assert np.array_equal(dw.out[0].cpu().numpy(), ref, equal_nan=True)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["fp16_407m", "int8_b16", "int4_2b"])
def test_decode_has_no_stalled_waits(name):
    """No decode of a full-size lane takes anywhere near the kernels' bounded-wait limit
    (about 2 s).  A wait that can never succeed (an exit-path wait on a ring slot whose barrier
    has moved two phases on, say) ends only at that limit and leaves the results intact, so
    neither the status word nor the outputs would show it; the time does."""
    import time
    w = get_workload(name)
    w = select_lanes(w, [0])
    dw = _dw(w)
    worst = 0.0
    for rep in range(3):
        for it in range(w.L_max):
            dw.append_new(it)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            dw.decode(it)
            torch.cuda.synchronize()
            worst = max(worst, time.perf_counter() - t0)
    assert worst < 0.25, f"{name}: slowest decode took {worst:.3f} s"


def test_decode_at_maximum_sizes():
    """The largest decode call the kernels take: 64 lanes, one of them with 65535 cached
    positions (64 splits of 1024 rows, the most a lane can have), the others ragged down to no
    cached position at all; sampled lanes against the oracle."""
    import dataclasses
    import store_kv_attention_b200 as tl
    ctx = [65535] + [(37 * b * b + 11 * b) % 3000 for b in range(1, 64)]
    ctx[1], ctx[2], ctx[63] = 0, 1, 4097
    loops = [2 if b % 2 == 0 else 1 for b in range(64)]
    w = dataclasses.replace(get_workload("int4_2b"), ctx=ctx, loops=loops, n_pre=1, L_max=2, name="int4_2b_max")
    dw = _dw(w)
    dw.step()
    torch.cuda.synchronize()
    assert tl.poll_status(dw.cache) == tl.TL_OK
    out = dw.out.cpu().numpy()
    for it, b in [(0, 0), (1, 0), (0, 1), (0, 2), (1, 40), (0, 63)]:
        assert it < w.loops[b]
        _assert_close(out[it, b], _oracle_lane(w, it, b, form="absorbed"), f"max sizes lane {b} it {it}")
    act = np.array([[it < w.loops[b] for b in range(w.B)] for it in range(w.L_max)])
    assert np.all(np.isfinite(out[act])) and np.all(np.isnan(out[~act]))


@pytest.mark.parametrize("name,ctx,loops", [
    ("fp16_407m", [0, 5, 130, 1030], [3, 1, 3, 2]),
    ("int8_b16", [1, 255, 1024, 2049], [2, 3, 1, 3]),
    ("int4_2b", [0, 3, 1000, 2048], [3, 1, 2, 3]),
], ids=["fp16", "int8", "int4"])
def test_fused_append_equals_separate_calls(name, ctx, loops):
    """tl_storeh_append_attn_decode writes exactly the rows tl_storeh_append writes (cache bytes
    identical) and gives bit-identical outputs, flags and first-abort iterations."""
    w = _small(name, ctx, loops)
    sep, fus = _dw(w, flag_mix=True, fill=False), _dw(w, flag_mix=True, fill=False)
    for dw in (sep, fus):  # the same bytes everywhere, so that the whole caches can be compared
        dw.cache.codes.fill_(0x5A)
        if dw.cache.scales is not None:
            dw.cache.scales.fill_(0x5A)
        dw.fill_context()
    sep.step()
    fus.step(fused_append=True)
    torch.cuda.synchronize()
    assert torch.equal(sep.cache.codes, fus.cache.codes)
    if sep.cache.scales is not None:
        assert torch.equal(sep.cache.scales, fus.cache.scales)
    a, b = sep.out.cpu().numpy(), fus.out.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert torch.equal(sep.flags, fus.flags) and torch.equal(sep.first, fus.first)
    # and against the oracle, for one active lane per iteration
    for it in range(w.L_max):
        bs = [bb for bb in range(w.B) if it < w.loops[bb]]
        if bs:
            _assert_close(b[it, bs[-1]], _oracle_lane(w, it, bs[-1]), f"{name} fused lane {bs[-1]} it {it}")


def test_device_timeout_is_reported_and_cleared():
    """The failure-detection path, without a GPU fault: a kernel's wait that cannot complete
    gives up after its bound, the status word reports TL_ERR_DEVICE_TIMEOUT once (then it is
    cleared), and the library keeps working afterwards."""
    import store_kv_attention_b200 as tl
    w = get_workload("tiny_fp16")
    dw = _dw(w)
    tl.selftest_wait_timeout(dw.cache, 2_000_000)  # about 1 ms of SM clocks
    assert tl.poll_status(dw.cache) == tl.TL_ERR_DEVICE_TIMEOUT
    assert tl.poll_status(dw.cache) == tl.TL_OK
    dw.step()
    torch.cuda.synchronize()
    assert tl.poll_status(dw.cache) == tl.TL_OK
    out = dw.out.cpu().numpy()
    _assert_close(out[0, 0], _oracle_lane(w, 0, 0), "after the timeout self-test")


# --------------------------------------------------------------------------- per-call split length
@pytest.mark.parametrize("name,ctx,loops,split", [
    ("fp16_407m", [2048], [8], 128),
    ("int8_b16", [0, 255, 1100, 2049], [8, 3, 8, 5], 256),
    ("int4_mixed", [1, 129, 700, 1024, 2500, 64], [4, 16, 32, 4, 16, 32], 512),
], ids=["fp16_split128", "int8_split256", "int4_split512"])
def test_split_rows_option_matches_oracle_and_solo(name, ctx, loops, split):
    """tl_storeh_decode_ex with a shorter split: outputs against the oracle, flags identical, and
    each lane bit-identical to its solo run with the same split length (batch independence)."""
    import store_kv_attention_b200 as tl
    w = _small(name, ctx, loops)
    dw = _dw(w, flag_mix=True, split_rows=split)
    dw.step(fused_append=True)
    torch.cuda.synchronize()
    assert tl.poll_status(dw.cache) == tl.TL_OK
    out = dw.out.cpu().numpy()
    f = np.zeros(w.B, np.uint8)
    fi = np.full(w.B, -1, np.int32)
    its = range(w.L_max) if w.L_max <= 8 else [0, 3, 4, 15, 16, 31]
    for it in range(w.L_max):
        for b in range(w.B):
            if it >= w.loops[b]:
                assert np.all(np.isnan(out[it, b]))
            elif it in its:
                _assert_close(out[it, b], _oracle_lane(w, it, b, form="absorbed"), f"{name} split {split} lane {b} it {it}")
        f, fi, _ = oracle.cpp.residual_norm_check(w.residual(it, True), w.threshold, it, np.array(w.loops), f, fi)
    assert np.array_equal(dw.flags.cpu().numpy(), f) and np.array_equal(dw.first.cpu().numpy(), fi)
    for b in sorted({0, w.B - 1}):
        solo = _dw(select_lanes(w, [b]), flag_mix=True, split_rows=split, max_ctx=w.max_ctx)
        solo.step(fused_append=True)
        torch.cuda.synchronize()
        assert np.array_equal(out[:, b].view(np.uint32), solo.out[:, 0].cpu().numpy().view(np.uint32)), f"lane {b}"


def test_call_with_no_active_lane_writes_nothing():
    """Every lane past its loop count at this iteration: the call launches, writes no output,
    appends no row, leaves the flags alone and reports nothing."""
    import store_kv_attention_b200 as tl
    w = _small("int4_2b", [5, 300, 1500], [2, 1, 3])
    w.L_max = 4
    dw = _dw(w)
    before = dw.cache.codes.clone()
    it = 3                                  # every lane has loops <= 3
    dw.out[it].fill_(float("nan"))
    dw.decode(it, append=True)
    torch.cuda.synchronize()
    assert np.all(np.isnan(dw.out[it].cpu().numpy()))
    assert torch.equal(before, dw.cache.codes)
    assert np.all(dw.flags.cpu().numpy() == 0) and np.all(dw.first.cpu().numpy() == -1)
    assert tl.poll_status(dw.cache) == tl.TL_OK


def test_call_with_fewer_lanes_than_the_cache_holds():
    """A cache sized for 8 lanes, called with its first 3: the rows are addressed with the cache's
    lane stride, and each lane gives the bits of the 8-lane call (the lanes are independent)."""
    import store_kv_attention_b200 as tl
    w = _small("int8_b16", [3, 700, 1500, 20, 1030, 5, 260, 999], [2] * 8)
    w.L_max = 2
    full = _dw(w)
    full.step()
    torch.cuda.synchronize()
    part = _dw(w)
    n = 3
    out = torch.full((w.L_max, n, w.H, w.hd), float("nan"), dtype=torch.float32, device="cuda")
    for it in range(w.L_max):
        part.append_new(it)
        tl.attn_decode(part.cache, it, part.loops[:n], part.ctx[:n], part.h_new[it][:n].contiguous(), part.W["q"],
                       part.W["k"], part.W["v"], out[it], residual=part.residual[it][:n].contiguous(),
                       threshold=w.threshold, abort_flags=part.flags[:n], first_abort_iter=part.first[:n])
    torch.cuda.synchronize()
    assert tl.poll_status(part.cache) == tl.TL_OK
    a, b = full.out[:, :n].cpu().numpy(), out.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert torch.equal(full.flags[:n], part.flags[:n]) and torch.equal(full.first[:n], part.first[:n])


def test_cache_without_pre_layers():
    """n_pre = 0: the loop block's layers start at layer 0 of the cache."""
    w = _small("tiny_fp16", [0, 77, 300], [2, 1, 2])
    w.n_pre = 0
    dw = _dw(w)
    dw.step()
    torch.cuda.synchronize()
    out = dw.out.cpu().numpy()
    for it in range(w.L_max):
        for b in range(w.B):
            if it < w.loops[b]:
                _assert_close(out[it, b], _oracle_lane(w, it, b), f"n_pre 0 lane {b} it {it}")
            else:
                assert np.all(np.isnan(out[it, b]))
