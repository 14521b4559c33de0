"""Parity of the iteration-axis delta-cache writer (tl_delta_append, through the C ABI) with
the CPU oracle (oracle/delta_oracle.py): anchor, INT8 codes and fp16 scales bit-exact, and
nothing written for lanes past their loop count or positions outside the cache."""
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
