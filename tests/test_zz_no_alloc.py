"""The decode entry point for callers that cannot allocate device memory.

`tl_storeh_attn_decode_static_ws` runs the decode on scratch compiled into the
library instead of a caller-allocated workspace.  Some callers cannot call
cudaMalloc (plug-ins inside another application's memory budget, code that
must not allocate once its streams are set up); this checks that, called
through the C ABI twice in a row, it gives what `tl_storeh_attn_decode` gives,
and that requests too large for the built-in scratch are refused.

Kept in its own file, collected last, so a run that stops at the first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from synth.workloads import get_workload, small_variant

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


@pytest.fixture(scope="module")
def tl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from store_kv_attention_b200 import build_lib
    build_lib.build()
    import store_kv_attention_b200 as m
    return m


def _close(a, b):
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b))
    err = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert err <= MAX_ABS and rel <= REL_L2, (err, rel)


@pytest.mark.parametrize("name,ctx,loops", [
    ("int4_2b", [7, 1030, 2100, 300], [2, 2, 1, 2]),
    ("int8_b16", [2049, 5, 1500], [2, 2, 2]),
])
def test_static_scratch_matches_workspace_entry_point(tl, name, ctx, loops):
    from synth.device import DeviceWorkload
    w = small_variant(get_workload(name), ctx=ctx, loops=loops)
    w.L_max = 2
    dw = DeviceWorkload(w)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for it in range(2):                      # two calls in a row, different iterations
        dw.append_new(it)
        dw.decode(it)                        # the existing entry point (caller workspace)
        want = dw.out[it].clone()
        flags_want, first_want = dw.flags.clone(), dw.first.clone()
        got = torch.full_like(want, float("nan"))
        flags = torch.zeros_like(dw.flags)
        first = torch.full_like(dw.first, -1)
        if it == 1:                          # carry the sticky flags of iteration 0
            flags.copy_(flags_prev)
            first.copy_(first_prev)
        tl.attn_decode_static_ws(dw.cache, it, dw.loops, dw.ctx, dw.h_new[it], dw.W["q"], dw.W["k"], dw.W["v"], got,
                                 residual=dw.residual[it], threshold=w.threshold, abort_flags=flags,
                                 first_abort_iter=first, status_out=status)
        torch.cuda.synchronize()
        if it == 1:                          # after a warm-up call the call takes no device memory
            spare = torch.empty_like(got)
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
            alloc_before = torch.cuda.memory_allocated()
            tl.attn_decode_static_ws(dw.cache, it, dw.loops, dw.ctx, dw.h_new[it], dw.W["q"], dw.W["k"],
                                     dw.W["v"], spare, status_out=status)
            torch.cuda.synchronize()
            assert torch.cuda.mem_get_info()[0] == free_before
            assert torch.cuda.memory_allocated() == alloc_before
        act = [b for b in range(w.B) if it < w.loops[b]]
        idle = [b for b in range(w.B) if it >= w.loops[b]]
        _close(got[act].cpu().numpy(), want[act].cpu().numpy())
        # the same kernels with fixed reduction orders: bit-identical, so stale scratch contents
        # or a wrong offset inside the array would show even where they stay inside the tolerance
        assert torch.equal(got[act], want[act])
        assert torch.all(torch.isnan(got[idle]))          # inactive lanes are not written
        assert torch.equal(flags, flags_want) and torch.equal(first, first_want)
        assert int(status.item()) == 0
        flags_prev, first_prev = flags.clone(), first.clone()
    assert tl.poll_status(dw.cache) == tl.TL_OK


def test_static_scratch_refuses_oversized_requests(tl):
    desc = tl.StoreHDesc(2048, 16, 128, n_pre=2, L_max=32, max_lanes=48, max_ctx=8193, fmt=tl.TL_H_INT4_G64)
    need = tl.workspace_bytes(desc, 48)
    assert need > 32 << 20
    fake = 1 << 20                           # never dereferenced: the size check comes first
    with pytest.raises(tl.TLError) as e:
        st = tl.lib.tl_storeh_attn_decode_static_ws(
            ctypes.byref(desc.c()), tl.Cache(fake, fake), 0, fake, fake, fake, fake, fake, fake, fake, None, 0.0,
            None, None, None, 48, None, None)
        tl._check(st, "tl_storeh_attn_decode_static_ws")
    assert e.value.status == tl.TL_ERR_CAPACITY
    assert b"exceeds the built-in" in tl.lib.tl_last_error_message()
