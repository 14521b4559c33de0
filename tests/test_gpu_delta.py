"""Parity of the iteration-axis delta cache on the GPU (through the C ABI) with the CPU oracle
(oracle/delta_oracle.py): the writer's anchor, INT8 codes and fp16 scales bit-exact, nothing
written for lanes past their loop count or positions outside the cache; the decode's outputs
within max-abs 2e-3 and relative L2 1e-3 of attention over the exact rebuild, safety-check
flags identical, lanes past their loop count left unwritten."""
import numpy as np
import pytest
import torch

import synth
from oracle import delta_oracle as D

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from store_kv_attention_b200 import build_lib
    build_lib.build()


def _fill_sentinels(cache):
    cache.anchor.view(torch.int16).fill_(0x5A5A)
    cache.deltas.fill_(0x5A)
    cache.scales.view(torch.int16).fill_(0x5A5A)


def _views(cache, desc):
    rows = desc.max_lanes * desc.max_ctx
    a = cache.anchor[: rows * desc.d_model].view(desc.max_lanes, desc.max_ctx, desc.d_model).cpu().numpy()
    L = desc.L_max - 1
    dl = cache.deltas[: L * rows * desc.d_model].view(L, desc.max_lanes, desc.max_ctx, desc.d_model).cpu().numpy()
    sc = cache.scales[: L * rows * desc.n_heads].view(L, desc.max_lanes, desc.max_ctx, desc.n_heads).cpu().numpy()
    return a, dl, sc


@pytest.mark.parametrize("d,H,L_max,n_lanes,n_rows", [(256, 4, 5, 3, 70), (2048, 16, 4, 2, 33), (1024, 16, 6, 2, 129)])
def test_writer_bit_exact(d, H, L_max, n_lanes, n_rows):
    import store_kv_attention_b200 as tl
    hd = d // H
    max_ctx = 260
    desc = tl.DeltaDesc(d, H, hd, L_max, n_lanes, max_ctx)
    cache = tl.DeltaCache(desc)
    _fill_sentinels(cache)
    start = np.array([0, 57, 3][:n_lanes], dtype=np.int32)
    traj = synth.trajectory_f16(17 + d, n_lanes * n_rows, d, L_max - 1)  # [L_max, lanes*rows, d]
    start_d = torch.from_numpy(start).cuda()
    for it in range(L_max):
        rows = torch.from_numpy(traj[it].reshape(n_lanes, n_rows, d)).cuda()
        tl.delta_append(cache, it, rows, start_d)
    torch.cuda.synchronize()
    a, dl, sc = _views(cache, desc)
    want_a, want_c, want_s = D.encode_trajectory(traj, H, "rebuilt")
    for b in range(n_lanes):
        sl = slice(b * n_rows, (b + 1) * n_rows)
        pos = slice(start[b], start[b] + n_rows)
        assert np.array_equal(a[b, pos], want_a[sl]), b
        assert np.array_equal(dl[:, b, pos], want_c[:, sl]), b
        assert np.array_equal(sc[:, b, pos].view(np.uint16), want_s[:, sl].view(np.uint16)), b
        # positions outside the written range keep the sentinels
        assert np.all(a[b, : start[b]].view(np.uint16) == 0x5A5A)
        assert np.all(dl[:, b, start[b] + n_rows:].view(np.uint8) == 0x5A)


def test_writer_skips_lanes_past_their_loops_and_out_of_range_rows():
    import store_kv_attention_b200 as tl
    d, H, L_max, n_lanes, n_rows, max_ctx = 256, 4, 4, 3, 6, 8
    desc = tl.DeltaDesc(d, H, d // H, L_max, n_lanes, max_ctx)
    cache = tl.DeltaCache(desc)
    _fill_sentinels(cache)
    traj = synth.trajectory_f16(5, n_lanes * n_rows, d, L_max - 1)
    loops = torch.tensor([4, 2, 1], dtype=torch.int32, device="cuda")
    start = torch.tensor([0, 4, -2], dtype=torch.int32, device="cuda")  # lane 1 runs past max_ctx, lane 2 starts before 0
    for it in range(L_max):
        rows = torch.from_numpy(traj[it].reshape(n_lanes, n_rows, d)).cuda()
        tl.delta_append(cache, it, rows, start, loops=loops)
    torch.cuda.synchronize()
    a, dl, sc = _views(cache, desc)
    want_a, want_c, want_s = D.encode_trajectory(traj, H, "rebuilt")
    # lane 0: every iteration, positions 0..5
    assert np.array_equal(a[0, :6], want_a[0:6]) and np.array_equal(dl[:, 0, :6], want_c[:, 0:6])
    # lane 1: iterations 0 and 1 only, positions 4..7 (rows 0..3); iterations 2, 3 untouched
    assert np.array_equal(a[1, 4:8], want_a[6:10]) and np.array_equal(dl[0, 1, 4:8], want_c[0, 6:10])
    assert np.all(dl[1:, 1].view(np.uint8) == 0x5A) and np.all(sc[1:, 1].view(np.uint16) == 0x5A5A)
    assert np.all(a[1, :4].view(np.uint16) == 0x5A5A)
    # lane 2: iteration 0 only, rows 2..5 at positions 0..3; no delta written
    assert np.array_equal(a[2, 0:4], want_a[14:18]) and np.all(a[2, 4:].view(np.uint16) == 0x5A5A)
    assert np.all(dl[:, 2].view(np.uint8) == 0x5A)


# --------------------------------------------------------------------------- decode over the delta cache
MAX_ABS = 2e-3
REL_L2 = 1e-3


def _weights(seed, d):
    return [synth.normal_f16(seed, 40 + i, 0, d * d, scale=1.0 / np.sqrt(d)).reshape(d, d) for i in range(3)]


# The streaming stage rebuilds every attended row by the FP32 prefix sum and feeds it to the
# tensor cores as fp16 hi + lo parts, so the outputs carry the FP32 rebuild.  (The earlier
# composition rounded the rebuilt rows to fp16 first and missed the bar at d = 1024.)
@pytest.mark.parametrize("d,H,L_max,ctx,max_ctx", [
    (256, 4, 3, [150, 37], 200),
    (1024, 16, 3, [500, 64], 600),
    (1024, 16, 8, [1030, 5], 1100),      # deep levels, a context over two splits
    (2048, 16, 4, [1100, 300], 1200),    # the 2B-like shape
    (768, 12, 3, [300, 40], 400),        # projection clusters of 4 (d_model / 64 = 12)
    (1280, 10, 3, [200, 700], 800),
])
def test_decode_matches_oracle(d, H, L_max, ctx, max_ctx):
    import oracle
    import store_kv_attention_b200 as tl
    hd = d // H
    n_lanes = len(ctx)
    desc = tl.DeltaDesc(d, H, hd, L_max, n_lanes, max_ctx)
    cache = tl.DeltaCache(desc, n_lanes=n_lanes)
    _fill_sentinels(cache)
    loops = np.array([L_max, 2][:n_lanes], dtype=np.int32)
    trajs = [synth.trajectory_f16(31 + 7 * b + d, ctx[b] + 1, d, L_max - 1) for b in range(n_lanes)]
    # context rows 0..ctx_b-1 of every iteration, one lane per call (the other lane's rows land
    # outside the cache and are skipped)
    for it in range(L_max):
        for b in range(n_lanes):
            rows = np.zeros((n_lanes, ctx[b], d), dtype=np.float16)
            rows[b] = trajs[b][it, : ctx[b]]
            start = np.full(n_lanes, max_ctx, dtype=np.int32)
            start[b] = 0
            tl.delta_append(cache, it, torch.from_numpy(rows).cuda(), torch.from_numpy(start).cuda())
    Wq, Wk, Wv = _weights(5, d)
    Wq_d, Wk_d, Wv_d = (torch.from_numpy(w).cuda() for w in (Wq, Wk, Wv))
    loops_d = torch.from_numpy(loops).cuda()
    ctx_d = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    residual = (synth.normal_f32(9, 60, 0, n_lanes * d, scale=4.0).reshape(n_lanes, d))
    flags = torch.zeros(n_lanes, dtype=torch.uint8, device="cuda")
    first = torch.full((n_lanes,), -1, dtype=torch.int32, device="cuda")
    want_flags = np.zeros(n_lanes, dtype=np.uint8)
    want_first = np.full(n_lanes, -1, dtype=np.int32)
    enc = [D.encode_trajectory(trajs[b], H, "rebuilt") for b in range(n_lanes)]
    for it in range(L_max):
        h_new = np.stack([trajs[b][it, ctx[b]] for b in range(n_lanes)])
        out = torch.full((n_lanes, d), float("nan"), dtype=torch.float32, device="cuda")
        tl.delta_attn_decode(cache, it, loops_d, ctx_d, torch.from_numpy(h_new).cuda(), Wq_d, Wk_d, Wv_d, out,
                             residual=torch.from_numpy(residual).cuda(), threshold=50.0, abort_flags=flags,
                             first_abort_iter=first)
        torch.cuda.synchronize()
        assert tl.poll_status(cache) == tl.TL_OK  # no lane out of range, no wait gave up
        got = out.cpu().numpy()
        for b in range(n_lanes):
            if it >= loops[b]:
                assert np.all(np.isnan(got[b])), (it, b)
                continue
            a, c, s = enc[b]
            rows = D.reconstruct(a, c, s, it, H)  # positions 0..ctx_b, the new token last
            want = oracle.attend_explicit(rows, h_new[b], Wq, Wk, Wv, H, hd).reshape(d)
            err = np.abs(got[b] - want)
            assert err.max() <= MAX_ABS, (it, b, err.max())
            assert np.linalg.norm(got[b] - want) <= REL_L2 * np.linalg.norm(want), (it, b)
        want_flags, want_first, _ = oracle.residual_norm_check(residual, 50.0, it, loops, want_flags, want_first)
    assert np.array_equal(flags.cpu().numpy(), want_flags)
    assert np.array_equal(first.cpu().numpy(), want_first)
