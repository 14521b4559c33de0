"""The RoPE-compatible decode on the GPU (tl_storeh_attn_decode_rope) through the C ABI,
against the RoPE-variant oracle: outputs within max-abs 2e-3 and relative L2 1e-3, the
safety check's flags identical, inactive lanes untouched."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import oracle.cpp
from oracle import rope_oracle
from synth.workloads import get_workload, small_variant

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from store_kv_attention_b200 import build_lib
    build_lib.build()


@pytest.mark.parametrize("name,ctx,loops,base", [
    ("tiny_fp16", [0, 130, 300], [2, 2, 1], 10000.0),
    ("fp16_407m", [7, 1100, 2048], [2, 1, 2], 10000.0),
    ("int8_b16", [1, 255, 1500], [2, 2, 2], 500000.0),
    ("int4_2b", [127, 1030, 2100], [2, 2, 1], 10000.0),
], ids=["fp16_d256", "fp16_d1024", "int8_d1024", "int4_d2048"])
def test_rope_decode_matches_oracle(name, ctx, loops, base):
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    w = dataclasses.replace(small_variant(get_workload(name), ctx=ctx, loops=loops), L_max=2)
    dw = DeviceWorkload(w, flag_mix=True)
    ws = torch.zeros(tl.rope_workspace_bytes(dw.desc, w.B), dtype=torch.uint8, device="cuda")
    W = [w.weight(k) for k in "qkv"]
    f = np.zeros(w.B, np.uint8)
    fi = np.full(w.B, -1, np.int32)
    for it in range(2):
        dw.append_new(it)
        tl.attn_decode_rope(dw.cache, it, dw.loops, dw.ctx, dw.h_new[it], dw.W["q"], dw.W["k"], dw.W["v"],
                            dw.out[it], ws, rope_base=base, residual=dw.residual[it], threshold=w.threshold,
                            abort_flags=dw.flags, first_abort_iter=dw.first)
        torch.cuda.synchronize()
        assert tl.poll_status(ws) == tl.TL_OK
        got = dw.out[it].cpu().numpy()
        layer = w.n_pre + it
        for b in range(w.B):
            if it >= w.loops[b]:
                assert np.all(np.isnan(got[b])), f"inactive lane {b} was written"
                continue
            rows = np.concatenate([w.h_rows(layer, b, 0, w.ctx[b]), w.h_new(it)[b:b + 1]])
            c, s = oracle.cpp.quantize_rows(rows, w.fmt)
            hh = oracle.cpp.dequantize_rows(c, s, w.fmt, w.d)
            want = rope_oracle.attend_rope(hh, w.h_new(it)[b], *W, w.H, w.hd, base=base)
            g = got[b].astype(np.float64)
            err = np.abs(g - want).max()
            rel = np.linalg.norm(g - want) / np.linalg.norm(want)
            assert err <= MAX_ABS and rel <= REL_L2, f"{name} lane {b} it {it}: max-abs {err:.3g} rel-L2 {rel:.3g}"
        f, fi, _ = oracle.cpp.residual_norm_check(w.residual(it, True), w.threshold, it, np.array(w.loops), f, fi)
    assert np.array_equal(dw.flags.cpu().numpy(), f) and np.array_equal(dw.first.cpu().numpy(), fi)


def test_rope_decode_long_context():
    """A 60,000-position lane: angles up to 6e4 rad, which the FP64 table must reduce exactly."""
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    w = dataclasses.replace(small_variant(get_workload("tiny_fp16"), ctx=[60000, 17], loops=[1, 1]), L_max=1)
    dw = DeviceWorkload(w)
    ws = torch.zeros(tl.rope_workspace_bytes(dw.desc, w.B), dtype=torch.uint8, device="cuda")
    dw.append_new(0)
    tl.attn_decode_rope(dw.cache, 0, dw.loops, dw.ctx, dw.h_new[0], dw.W["q"], dw.W["k"], dw.W["v"], dw.out[0], ws)
    torch.cuda.synchronize()
    assert tl.poll_status(ws) == tl.TL_OK
    got = dw.out[0].cpu().numpy()
    W = [w.weight(k) for k in "qkv"]
    for b in range(w.B):
        rows = np.concatenate([w.h_rows(w.n_pre, b, 0, w.ctx[b]), w.h_new(0)[b:b + 1]])
        c, s_ = oracle.cpp.quantize_rows(rows, w.fmt)
        hh = oracle.cpp.dequantize_rows(c, s_, w.fmt, w.d)
        want = rope_oracle.attend_rope(hh, w.h_new(0)[b], *W, w.H, w.hd)
        g = got[b].astype(np.float64)
        err = np.abs(g - want).max()
        rel = np.linalg.norm(g - want) / np.linalg.norm(want)
        assert err <= MAX_ABS and rel <= REL_L2, f"lane {b}: max-abs {err:.3g} rel-L2 {rel:.3g}"


@pytest.mark.parametrize("d,H,hd,fmt", [(768, 12, 64, 0), (1536, 12, 128, 2)], ids=["d768_fp16", "d1536_int4"])
def test_rope_decode_d_model_not_a_multiple_of_512(d, H, hd, fmt):
    """Every head's scores when 512 does not divide d_model (the K columns in blocks of 256)."""
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    from synth.workloads import Workload
    w = Workload(name=f"rope_d{d}", d=d, H=H, hd=hd, n_pre=1, L_max=1, fmt=fmt, seed=77, ctx=[300, 1025],
                 loops=[1, 1], residual_scale=1.0, threshold=50.0)
    dw = DeviceWorkload(w)
    ws = torch.zeros(tl.rope_workspace_bytes(dw.desc, w.B), dtype=torch.uint8, device="cuda")
    dw.append_new(0)
    tl.attn_decode_rope(dw.cache, 0, dw.loops, dw.ctx, dw.h_new[0], dw.W["q"], dw.W["k"], dw.W["v"], dw.out[0], ws)
    torch.cuda.synchronize()
    assert tl.poll_status(ws) == tl.TL_OK
    got = dw.out[0].cpu().numpy()
    W = [w.weight(k) for k in "qkv"]
    for b in range(w.B):
        rows = np.concatenate([w.h_rows(w.n_pre, b, 0, w.ctx[b]), w.h_new(0)[b:b + 1]])
        c, s_ = oracle.cpp.quantize_rows(rows, w.fmt)
        hh = oracle.cpp.dequantize_rows(c, s_, w.fmt, w.d)
        want = rope_oracle.attend_rope(hh, w.h_new(0)[b], *W, w.H, w.hd)
        g = got[b].astype(np.float64)
        err = np.abs(g - want).max()
        rel = np.linalg.norm(g - want) / np.linalg.norm(want)
        assert err <= MAX_ABS and rel <= REL_L2, f"lane {b}: max-abs {err:.3g} rel-L2 {rel:.3g}"
