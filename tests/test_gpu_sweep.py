"""A seeded sweep over shapes the named workloads do not reach (d_model 512 / 768 / 1280 / 1536 /
1792, head_dim 128 at d_model 1024, odd lane counts), every cache format and split length, with
contexts on and around the tile and split edges, against the C++ oracle (absorbed form, which
the CPU tests pin to the explicit rebuild).  Bars as the decode parity tests: max-abs 2e-3 and
relative L2 1e-3 per (lane, iteration), flags identical, inactive lanes untouched."""
import dataclasses
import random

import numpy as np
import pytest
import torch

import oracle
import oracle.cpp
from synth.workloads import Workload

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3
SHAPES = [(256, 4, 64), (512, 8, 64), (768, 12, 64), (1024, 8, 128), (1024, 16, 64), (1280, 10, 128),
          (1536, 12, 128), (1792, 14, 128), (2048, 16, 128)]
EDGES = [0, 1, 2, 127, 128, 129, 255, 256, 511, 512, 513, 1023, 1024, 1025, 1500, 2047, 2048, 2049]


def _cases(n=18, seed=7):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        d, H, hd = SHAPES[i % len(SHAPES)]
        fmt = rng.randrange(3)
        if fmt == 1 and d > 1024:
            fmt = 2  # INT8 above d_model 1024: the relative bar only (test_int8_above_1024_* below)
        B = rng.randint(1, 6)
        ctx = [rng.choice(EDGES) for _ in range(B)]
        L = 3
        loops = [rng.randint(1, L) for _ in range(B)]
        split = rng.choice([0, 128, 256, 512])
        out.append((d, H, hd, fmt, ctx, loops, L, split, i))
    return out


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from store_kv_attention_b200 import build_lib
    build_lib.build()


@pytest.mark.parametrize("d,H,hd,fmt,ctx,loops,L,split,i", _cases(),
                         ids=[f"d{c[0]}_h{c[2]}_f{c[3]}_b{len(c[4])}_s{c[7]}" for c in _cases()])
def test_sweep_matches_oracle(d, H, hd, fmt, ctx, loops, L, split, i):
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    w = Workload(name=f"sweep{i}", d=d, H=H, hd=hd, n_pre=1, L_max=L, fmt=fmt, seed=100 + i, ctx=ctx, loops=loops,
                 residual_scale=4.0, threshold=50.0, outlier_p=0.02 if fmt == 1 else 0.0, outlier_mul=8.0,
                 forced_lanes=1)
    dw = DeviceWorkload(w, flag_mix=True, split_rows=split)
    dw.step(fused_append=bool(i % 2))
    torch.cuda.synchronize()
    assert tl.poll_status(dw.cache) == tl.TL_OK
    out = dw.out.cpu().numpy()
    W = [w.weight(k) for k in "qkv"]
    f = np.zeros(w.B, np.uint8)
    fi = np.full(w.B, -1, np.int32)
    for it in range(w.L_max):
        layer = w.n_pre + it
        for b in range(w.B):
            if it >= w.loops[b]:
                assert np.all(np.isnan(out[it, b])), f"inactive lane {b} iteration {it} was written"
                continue
            rows = np.concatenate([w.h_rows(layer, b, 0, w.ctx[b]), w.h_new(it)[b:b + 1]])
            c, s = oracle.cpp.quantize_rows(rows, w.fmt)
            hh = oracle.cpp.dequantize_rows(c, s, w.fmt, w.d)
            want = oracle.cpp.attend_absorbed(hh, w.h_new(it)[b], *W, w.H, w.hd)
            got = out[it, b].astype(np.float64)
            assert np.all(np.isfinite(got))
            err = np.abs(got - want).max()
            rel = np.linalg.norm(got - want) / np.linalg.norm(want)
            assert err <= MAX_ABS and rel <= REL_L2, f"lane {b} it {it}: max-abs {err:.3g} rel-L2 {rel:.3g}"
        f, fi, _ = oracle.cpp.residual_norm_check(w.residual(it, True), w.threshold, it, np.array(w.loops), f, fi)
    assert np.array_equal(dw.flags.cpu().numpy(), f) and np.array_equal(dw.first.cpu().numpy(), fi)


def _int8_large(d, H, hd):
    from synth.device import DeviceWorkload
    w = Workload(name=f"int8_d{d}", d=d, H=H, hd=hd, n_pre=1, L_max=1, fmt=1, seed=31, ctx=[700, 1500],
                 loops=[1, 1], residual_scale=4.0, threshold=50.0, outlier_p=0.02, outlier_mul=8.0)
    dw = DeviceWorkload(w)
    dw.step()
    torch.cuda.synchronize()
    W = [w.weight(k) for k in "qkv"]
    res = []
    for b in range(w.B):
        rows = np.concatenate([w.h_rows(w.n_pre, b, 0, w.ctx[b]), w.h_new(0)[b:b + 1]])
        c, s = oracle.cpp.quantize_rows(rows, w.fmt)
        hh = oracle.cpp.dequantize_rows(c, s, w.fmt, w.d)
        want = oracle.cpp.attend_absorbed(hh, w.h_new(0)[b], *W, w.H, w.hd)
        got = dw.out[0, b].cpu().numpy().astype(np.float64)
        res.append((np.abs(got - want).max(), np.linalg.norm(got - want) / np.linalg.norm(want)))
    return res


@pytest.mark.parametrize("d,H,hd", [(1792, 14, 128), (2048, 16, 128)])
def test_int8_above_1024_relative_bar(d, H, hd):
    """INT8 rows with x8 outlier rows above d_model 1024: relative L2 within 1e-3."""
    for err, rel in _int8_large(d, H, hd):
        assert rel <= REL_L2, f"rel-L2 {rel:.3g}"


@pytest.mark.xfail(strict=True, reason="above d_model 1024 the absorbed query and P are single fp16 operands; "
                                       "outputs of magnitude ~25 exceed max-abs 2e-3")
@pytest.mark.parametrize("d,H,hd", [(1792, 14, 128), (2048, 16, 128)])
def test_int8_above_1024_absolute_bar(d, H, hd):
    for err, rel in _int8_large(d, H, hd):
        assert err <= MAX_ABS, f"max-abs {err:.3g}"
