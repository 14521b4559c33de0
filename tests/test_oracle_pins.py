"""Pins of the CPU oracle against things other than itself (no GPU).

* hand-worked quantiser cases and nibble order (tests/golden/*.txt);
* the quantiser equals the nearest grid point (brute force over all codes);
* closed-form quantisation error on Gaussian h against the pages' K/V errors;
* attention against torch's library attention over explicitly stored K/V;
* textbook special cases (one row; identical rows);
* the variable-L layer-range invariant and NaN poisoning;
* L-aware batching: a mixed lane equals its solo run;
* the safety check on exact norms and the pages' measured example.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import oracle.cpp
import synth
from synth.workloads import small_variant

# Both oracles, the numpy one and the plain C++ one, must pass every pin that applies to them.
IMPLS = [pytest.param(oracle, id="numpy"), pytest.param(oracle.cpp, id="cpp")]

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([c.strip() for c in line.split("|")])
    return rows


# --------------------------------------------------------------------------- quantiser
@pytest.mark.parametrize("ora", IMPLS)
def test_int8_hand_cases(ora):
    for scale, xs, codes in _read_golden("quant_int8_hand.txt"):
        x = np.array([float(v) for v in xs.split()], dtype=np.float16)
        row = np.zeros((1, 64), np.float16)
        row[0, :x.size] = x
        c, s = ora.quantize_rows(row, oracle.FMT_INT8)
        assert s.dtype == np.float32 and s[0, 0] == np.float32(float(scale))
        want = np.array([int(v) for v in codes.split()], dtype=np.int8)
        assert np.array_equal(c.view(np.int8)[0, :x.size], want), (xs, c.view(np.int8)[0, :x.size])
        assert np.all(c.view(np.int8)[0, x.size:] == 0)


@pytest.mark.parametrize("ora", IMPLS)
def test_int4_hand_cases_and_nibble_order(ora):
    for scale, xs, codes, hexbytes in _read_golden("quant_int4_hand.txt"):
        x = np.array([float(v) for v in xs.split()], dtype=np.float16)
        row = np.zeros((1, 64), np.float16)
        row[0, :x.size] = x
        c, s = ora.quantize_rows(row, oracle.FMT_INT4)
        assert s.dtype == np.float16 and s[0, 0] == np.float16(float(scale))
        want = np.array([int(v) for v in codes.split()], dtype=np.int8)
        assert np.array_equal(oracle.unpack_int4(c)[0, :x.size], want)
        want_bytes = bytes.fromhex("".join(hexbytes.split()))
        assert c[0, :len(want_bytes)].tobytes() == want_bytes


@pytest.mark.parametrize("fmt,qmax", [(oracle.FMT_INT8, 127), (oracle.FMT_INT4, 7)])
@pytest.mark.parametrize("ora", IMPLS)
def test_quantiser_is_nearest_grid_point(ora, fmt, qmax):
    """Brute force: every code is the grid point c*scale nearest to x (ties to even c),
    except where the exact quotient lies within an fp32 rounding of a tie."""
    rng = np.random.default_rng(5)
    h = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-3, 3, (64, 1)))).astype(np.float16)
    h[3, :] = 0
    codes, scales = ora.quantize_rows(h, fmt)
    c = codes.view(np.int8) if fmt == oracle.FMT_INT8 else oracle.unpack_int4(codes)
    group = 256 if fmt == oracle.FMT_INT8 else 64
    sc = np.repeat(scales.astype(np.float64).reshape(64, -1), group, axis=1)
    grid = np.arange(-qmax, qmax + 1, dtype=np.float64)
    x = h.astype(np.float64)
    bad = 0
    for i in range(64):
        for k in range(256):
            if sc[i, k] == 0:
                assert c[i, k] == 0
                continue
            dist = np.abs(x[i, k] - grid * sc[i, k])
            best = np.flatnonzero(dist == dist.min())
            want = grid[best[0]] if best.size == 1 else grid[best[np.argmin(np.abs(grid[best]) % 2)]]
            if c[i, k] != want:
                t = x[i, k] / sc[i, k]
                assert abs(abs(t - np.trunc(t)) - 0.5) < 1e-6 * abs(t), (i, k, t, c[i, k], want)
                bad += 1
    assert bad <= 2
    # the group scale is amax / qmax (fp32 IEEE; INT4 then rounded to fp16)
    g = np.abs(x).reshape(64, -1, group).max(axis=2)
    if fmt == oracle.FMT_INT8:
        assert np.array_equal(scales[:, 0], (g[:, 0].astype(np.float32) / np.float32(127)))
    else:
        assert np.array_equal(scales, (g.astype(np.float32) / np.float32(7)).astype(np.float16))


@pytest.mark.parametrize("fmt", [oracle.FMT_FP16, oracle.FMT_INT8, oracle.FMT_INT4])
@pytest.mark.parametrize("ora", IMPLS)
def test_roundtrip_bound(ora, fmt):
    rng = np.random.default_rng(1)
    h = rng.standard_normal((32, 1024)).astype(np.float16)
    codes, scales = ora.quantize_rows(h, fmt)
    hh = ora.dequantize_rows(codes, scales, fmt, 1024)
    x = h.astype(np.float64)
    if fmt == oracle.FMT_FP16:
        assert np.array_equal(hh, x)  # FP16-h is lossless: K/V rebuilt bit-exactly
        return
    group = 1024 if fmt == oracle.FMT_INT8 else 64
    s = np.repeat(scales.astype(np.float64).reshape(32, -1), group, axis=1)
    # |x/s - code| <= 1/2 up to the rounding of the fp32 quotient x/s (one ulp of it)
    assert np.all(np.abs(hh - x) <= s * (0.5 + np.abs(x / s) * 2.0 ** -23))


@pytest.mark.parametrize("fmt,d,lo,hi", [(oracle.FMT_INT8, 1024, 0.004, 0.010),
                                         (oracle.FMT_INT4, 2048, 0.08, 0.12)])
@pytest.mark.parametrize("ora", IMPLS)
def test_closed_form_kv_error(ora, fmt, d, lo, hi):
    """K relative L2 error on Gaussian h equals the uniform-rounding closed form
    sqrt(sum scale^2/12 / sum h^2), and lands where the pages put it: about 0.6%
    for INT8-h and about 10% for INT4-h (Architecture-Exclusive Features,
    "Store-h KV cache", mode table)."""
    w = synth.get_workload("int8_b16" if fmt == oracle.FMT_INT8 else "int4_2b")
    h = w.h_rows(w.n_pre, 0, 0, 512)
    if fmt == oracle.FMT_INT8:
        h = synth.h_rows_f16(w.seed, synth.row_id(w.n_pre, 0, np.arange(512)), d)  # no outliers
    codes, scales = ora.quantize_rows(h, fmt)
    hh = ora.dequantize_rows(codes, scales, fmt, d)
    Wk = w.weight("k").astype(np.float64)
    x = h.astype(np.float64)
    K, Kh = x @ Wk.T, hh @ Wk.T
    rel = np.linalg.norm(Kh - K) / np.linalg.norm(K)
    group = d if fmt == oracle.FMT_INT8 else 64
    s = np.repeat(scales.astype(np.float64).reshape(512, -1), group, axis=1)
    predicted = math.sqrt(np.sum(s * s / 12.0) / np.sum(x * x))
    assert abs(rel / predicted - 1) < 0.05, (rel, predicted)
    assert lo < rel < hi


# --------------------------------------------------------------------------- attention
def _tiny(H=2, hd=8, n=7, seed=0):
    rng = np.random.default_rng(seed)
    d = H * hd
    W = [(rng.standard_normal((d, d)) / math.sqrt(d)).astype(np.float16) for _ in range(3)]
    h = rng.standard_normal((n, d)).astype(np.float16)
    return d, W, h


def _library_stored_kv(h_rows64, h_new, W, H, hd):
    """Brute force with explicitly stored K/V: torch.nn.functional.linear (weights
    [out, in]) computes K, V once per row, and torch's scaled_dot_product_attention
    (default scale 1/sqrt(head_dim)) attends the single query over all rows."""
    Wq, Wk, Wv = (torch.from_numpy(w.astype(np.float64)) for w in W)
    rows = torch.from_numpy(h_rows64)
    K = torch.nn.functional.linear(rows, Wk)          # stored at append time
    V = torch.nn.functional.linear(rows, Wv)
    q = torch.nn.functional.linear(torch.from_numpy(h_new.astype(np.float64)), Wq)
    n = rows.shape[0]
    qh = q.view(1, H, 1, hd)
    Kh = K.view(n, H, hd).permute(1, 0, 2).unsqueeze(0)
    Vh = V.view(n, H, hd).permute(1, 0, 2).unsqueeze(0)
    o = torch.nn.functional.scaled_dot_product_attention(qh, Kh, Vh)
    return o.view(H, hd).numpy()


@pytest.mark.parametrize("form", ["explicit", "absorbed"])
@pytest.mark.parametrize("fmt", [oracle.FMT_FP16, oracle.FMT_INT8, oracle.FMT_INT4])
@pytest.mark.parametrize("ora", IMPLS)
def test_attention_matches_library_over_stored_kv(ora, form, fmt):
    H, hd = 2, 32
    d, W, h = _tiny(H=H, hd=hd, n=9, seed=fmt)
    codes, scales = ora.quantize_rows(h, fmt)
    hh = ora.dequantize_rows(codes, scales, fmt, d)
    f = ora.attend_explicit if form == "explicit" else ora.attend_absorbed
    got = f(hh, h[-1], *W, H, hd)
    want = _library_stored_kv(hh, h[-1], W, H, hd)
    assert np.max(np.abs(got - want)) <= 1e-12 * max(1.0, np.max(np.abs(want)))


def test_fp16_h_identical_to_stored_kv():
    """FP16-h rebuilds K/V bit-exactly: the rows read back from the cache are the
    appended rows, so stored-K/V attention and store-h attention coincide
    (Architecture-Exclusive Features, "Store-h KV cache": FP16-h K/V bit-exact)."""
    H, hd = 4, 16
    d, W, h = _tiny(H=H, hd=hd, n=12, seed=3)
    cache = oracle.OracleCache(oracle.FMT_FP16, d, n_pre=1, L_max=1)
    cache.append(1, 0, 0, h[:-1])
    out, *_ = oracle.decode_iteration(cache, 0, [1], [11], h[-1:], *W, H, hd, None, 50.0,
                                      np.zeros(1, np.uint8), np.full(1, -1, np.int32))
    x = h.astype(np.float64)
    Wk, Wv = (w.astype(np.float64) for w in W[1:])
    K_stored, V_stored = x @ Wk.T, x @ Wv.T
    codes, scales = cache.read_rows(1, 0, 12)
    hh = oracle.dequantize_rows(codes, scales, oracle.FMT_FP16, d)
    assert np.array_equal(hh @ Wk.T, K_stored) and np.array_equal(hh @ Wv.T, V_stored)
    assert np.max(np.abs(out[0] - _library_stored_kv(x, h[-1], W, H, hd))) < 1e-12


@pytest.mark.parametrize("ora", IMPLS)
def test_absorbed_equals_explicit_at_workload_shape(ora):
    w = synth.get_workload("int4_2b")
    h = w.h_rows(w.n_pre, 0, 0, 257)
    codes, scales = ora.quantize_rows(h, w.fmt)
    hh = ora.dequantize_rows(codes, scales, w.fmt, w.d)
    W = [w.weight(k) for k in "qkv"]
    a = ora.attend_explicit(hh, h[-1], *W, w.H, w.hd)
    b = ora.attend_absorbed(hh, h[-1], *W, w.H, w.hd)
    assert np.max(np.abs(a - b)) < 1e-12


@pytest.mark.parametrize("ora", IMPLS)
def test_single_row_gives_v_of_new_token(ora):
    """With no cached positions the softmax has one entry, so o_j = (W_v h_new)_j."""
    H, hd = 2, 16
    d, W, h = _tiny(H=H, hd=hd, n=1, seed=4)
    hh = h.astype(np.float64)
    for f in (ora.attend_explicit, ora.attend_absorbed):
        o = f(hh, h[0], *W, H, hd)
        v = W[2].astype(np.float64) @ hh[0]
        assert np.max(np.abs(o.reshape(-1) - v)) < 1e-13


@pytest.mark.parametrize("ora", IMPLS)
def test_identical_rows_give_their_v(ora):
    H, hd = 2, 16
    d, W, h = _tiny(H=H, hd=hd, n=1, seed=6)
    rows = np.repeat(h.astype(np.float64), 10, axis=0)
    o = ora.attend_explicit(rows, h[0] * np.float16(3), *W, H, hd)
    assert np.max(np.abs(o.reshape(-1) - W[2].astype(np.float64) @ rows[0])) < 1e-13


@pytest.mark.parametrize("ora", IMPLS)
def test_softmax_scale_is_inverse_sqrt_head_dim(ora):
    """Two rows whose head-0 scores differ by exactly sqrt(hd)*ln(3): weights 3/4 and 1/4."""
    H, hd = 1, 16
    d = 16
    Wq = np.eye(d, dtype=np.float16)
    Wk = np.eye(d, dtype=np.float16)
    Wv = np.eye(d, dtype=np.float16)
    q = np.zeros(d, np.float16)
    q[0] = 1
    r1 = np.zeros(d)
    r1[1] = 1.0
    r2 = np.zeros(d)
    r2[0] = math.sqrt(hd) * math.log(3.0)
    r2[1] = 0.0
    rows = np.stack([r1, r2])
    o = ora.attend_explicit(rows, q, Wq, Wk, Wv, H, hd)
    want = 0.25 * r1 + 0.75 * r2
    assert np.max(np.abs(o.reshape(-1) - want)) < 1e-12


# --------------------------------------------------------------------------- variable-L, lanes
def _run_oracle_batch(w, its, lanes, form="explicit", poison=False, record=None):
    """Fill context rows of the attended layers, then run iterations ``its``."""
    cache = oracle.OracleCache(w.fmt, w.d, w.n_pre, w.L_max)
    for b in lanes:
        for layer in range(w.n_layers):
            if poison or (w.n_pre <= layer < w.n_pre + w.loops[b]):
                cache.append(layer, b, 0, w.h_rows(layer, b, 0, w.ctx[b]))
            if poison:
                # positions past the new token, and layers the lane must not read: NaN rows
                bad = np.full((3, w.d), np.nan, np.float16)
                cache.append(layer, b, w.ctx[b] + 1, bad)
                if not (w.n_pre <= layer < w.n_pre + w.loops[b]):
                    cache.append(layer, b, 0, np.full((w.ctx[b] + 1, w.d), np.nan, np.float16))
    W = [w.weight(k) for k in "qkv"]
    outs = []
    flags = np.zeros(len(lanes), np.uint8)
    first = np.full(len(lanes), -1, np.int32)
    for it in its:
        hn = w.h_new(it)[lanes]
        sub_loops = [w.loops[b] for b in lanes]
        sub_ctx = [w.ctx[b] for b in lanes]
        # the oracle's lane index is the position in `lanes`; remap cache keys
        remapped = oracle.OracleCache(w.fmt, w.d, w.n_pre, w.L_max)
        remapped.rows = {(layer, lanes.index(b)): v for (layer, b), v in cache.rows.items() if b in lanes}
        if record is not None:
            orig2 = remapped.read_rows

            def rec2(layer, lane, n, _o=orig2):
                record.append((layer, lanes[lane], n))
                return _o(layer, lane, n)
            remapped.read_rows = rec2
        res = w.residual(it)[lanes]
        o, flags, first, _ = oracle.decode_iteration(remapped, it, sub_loops, sub_ctx, hn, *W, w.H, w.hd,
                                                     res, w.threshold, flags, first, form=form)
        for (layer, i), v in remapped.rows.items():
            cache.rows[(layer, lanes[i])] = v
        outs.append(o)
    return np.stack(outs), flags, first


def _small_mixed():
    w = synth.get_workload("tiny_fp16")
    w = small_variant(w, ctx=[5, 9, 3], loops=[1, 3, 2])
    w.L_max = 3
    return w


def test_layer_range_invariant_and_poison():
    w = _small_mixed()
    rec = []
    clean, *_ = _run_oracle_batch(w, range(3), [0, 1, 2], record=rec)
    for layer, lane, n in rec:
        assert w.n_pre <= layer < w.n_pre + w.loops[lane]
        assert n == w.ctx[lane] + 1
    seen = {(layer, lane) for layer, lane, _ in rec}
    assert seen == {(w.n_pre + i, b) for b in range(3) for i in range(w.loops[b])}
    dirty, *_ = _run_oracle_batch(w, range(3), [0, 1, 2], poison=True)
    active = ~np.isnan(clean)
    assert np.array_equal(active, ~np.isnan(dirty))
    assert np.array_equal(clean[active], dirty[active])
    # inactive (lane, iteration) pairs produce nothing
    for it in range(3):
        for b in range(3):
            assert np.all(np.isnan(clean[it, b])) == (it >= w.loops[b])


def test_mixed_batch_lane_equals_solo_run():
    """Architecture-Exclusive Features, "L-aware batching": a mixed-batch lane is
    bit-exact with a solo run at its own loop count."""
    w = _small_mixed()
    mixed, fm, firstm = _run_oracle_batch(w, range(3), [0, 1, 2])
    for b in range(3):
        solo, fs, firsts = _run_oracle_batch(w, range(3), [b])
        assert np.array_equal(mixed[:, b], solo[:, 0], equal_nan=True)
        assert fm[b] == fs[0] and firstm[b] == firsts[0]


# --------------------------------------------------------------------------- safety check
@pytest.mark.parametrize("ora", IMPLS)
def test_norm_exact_triples_and_strictness(ora):
    r = np.zeros((3, 8), np.float32)
    r[0, :2] = [3, 4]          # norm 5
    r[1, :3] = [2, 3, 6]       # norm 7
    r[2, :2] = [30, 40]        # norm 50
    flags, first, norms = ora.residual_norm_check(r, 5.0, 0, np.array([4, 4, 4]),
                                                     np.zeros(3, np.uint8), np.full(3, -1, np.int32))
    assert np.array_equal(norms, [5.0, 7.0, 50.0])
    assert list(flags) == [0, 1, 1] and list(first) == [-1, 0, 0]
    flags, first, _ = ora.residual_norm_check(r, 50.0, 1, np.array([4, 4, 4]),
                                                 np.zeros(3, np.uint8), np.full(3, -1, np.int32))
    assert list(flags) == [0, 0, 0]  # exactly at the threshold is not "exceeds"


@pytest.mark.parametrize("ora", IMPLS)
def test_norm_sticky_and_inactive_lanes(ora):
    big = np.full((2, 4), 100.0, np.float32)
    small = np.zeros((2, 4), np.float32)
    loops = np.array([3, 1])
    f, first, _ = ora.residual_norm_check(big, 10.0, 0, loops, np.zeros(2, np.uint8),
                                             np.full(2, -1, np.int32))
    assert list(f) == [1, 1] and list(first) == [0, 0]
    f, first, norms = ora.residual_norm_check(small, 10.0, 1, loops, f, first)
    assert list(f) == [1, 1] and list(first) == [0, 0]
    assert norms[0] == 0 and np.isnan(norms[1])
    f, first, _ = ora.residual_norm_check(big, 10.0, 2, loops, np.zeros(2, np.uint8),
                                             np.full(2, -1, np.int32))
    assert list(f) == [1, 0] and list(first) == [2, -1]  # lane 1 has only one iteration


@pytest.mark.parametrize("ora", IMPLS)
def test_pages_safety_example(ora):
    for thr, norm, it, flag, first in _read_golden("safety_check_example.txt"):
        r = np.zeros((1, 2048), np.float32)
        r[0, 0] = float(norm)
        f, fi, n = ora.residual_norm_check(r, float(thr), int(it), np.array([8]),
                                              np.zeros(1, np.uint8), np.full(1, -1, np.int32))
        assert f[0] == int(flag) and fi[0] == int(first)
        assert abs(n[0] - float(norm)) < 1e-5


# --------------------------------------------------------------------------- generator
def test_generator_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * np.exp(rng.uniform(-25, 12, 20000)),
                        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26]])
    got = np.array([synth.f64_to_f16(v) for v in x])
    with np.errstate(over="ignore"):
        want = x.astype(np.float16)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_generator_moments_and_determinism():
    z = synth.normal_f64(9, 1, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    assert np.array_equal(z[1000:1010], synth.normal_f64(9, 1, 1000, 10))
    w = synth.get_workload("int8_b16")
    rows = w.h_rows(w.n_pre, 0, 0, 4000)
    big = np.max(np.abs(rows.astype(np.float32)), axis=1) > 10
    assert 0.003 < big.mean() < 0.02   # ~1% outlier rows scaled x8
    w5 = synth.get_workload("int4_mixed")
    assert min(w5.ctx) >= 1024 and max(w5.ctx) <= 8192 and len(set(w5.ctx)) > 40


# --------------------------------------------------------------------------- the C++ oracle
def test_cpp_fp16_rounding_matches_ieee():
    """The C++ oracle's binary32 -> binary16 rounding (INT4 scales) is IEEE round-to-nearest-even,
    checked against numpy's conversion over a wide range, subnormals, ties and overflow."""
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(50000) * np.exp(rng.uniform(-25, 12, 50000)),
                        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                         2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, -1e-9]]).astype(np.float32)
    got = np.array([oracle.cpp.f32_to_f16_bits(v) for v in x], np.uint16)
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt,d", [(oracle.FMT_FP16, 256), (oracle.FMT_INT8, 1024), (oracle.FMT_INT4, 2048)])
def test_cpp_quantiser_and_dequant_equal_numpy(fmt, d):
    rng = np.random.default_rng(fmt + 3)
    h = (rng.standard_normal((80, d)) * np.exp(rng.uniform(-6, 6, (80, 1)))).astype(np.float16)
    h[0] = 0
    h[1, :8] = np.array([0.5, 1.5, 2.5, -2.5, 3.5, 6.5, -7, 7], np.float16)
    h[2] = np.float16(3e-7)
    c1, s1 = oracle.quantize_rows(h, fmt)
    c2, s2 = oracle.cpp.quantize_rows(h, fmt)
    assert np.array_equal(c1, c2) and s1.dtype == s2.dtype and np.array_equal(s1.view(np.uint8), s2.view(np.uint8))
    assert np.array_equal(oracle.dequantize_rows(c1, s1, fmt, d), oracle.cpp.dequantize_rows(c2, s2, fmt, d))


@pytest.mark.parametrize("form", ["explicit", "absorbed"])
@pytest.mark.parametrize("H,hd,n", [(1, 8, 1), (2, 16, 9), (4, 64, 33)])
def test_cpp_attention_equals_numpy(form, H, hd, n):
    d, W, h = _tiny(H=H, hd=hd, n=n, seed=H + n)
    hh = h.astype(np.float64)
    f1 = oracle.attend_explicit if form == "explicit" else oracle.attend_absorbed
    f2 = oracle.cpp.attend_explicit if form == "explicit" else oracle.cpp.attend_absorbed
    a, b = f1(hh, h[-1], *W, H, hd), f2(hh, h[-1], *W, H, hd)
    assert np.max(np.abs(a - b)) <= 1e-12 * max(1.0, np.max(np.abs(a)))
    # the OpenMP split over heads does not change a single bit
    assert np.array_equal(b, f2(hh, h[-1], *W, H, hd, threads=1))


@pytest.mark.parametrize("fmt", [oracle.FMT_FP16, oracle.FMT_INT8, oracle.FMT_INT4])
def test_cpp_decode_lane_equals_numpy_decode_iteration(fmt):
    """One lane's whole iteration (append, dequant, explicit attention, safety check) in C++
    against the numpy oracle's decode_iteration on the same lane."""
    w = synth.get_workload({0: "tiny_fp16", 1: "int8_b16", 2: "int4_2b"}[fmt])
    w = small_variant(w, ctx=[45], loops=[2])
    it, layer = 1, w.n_pre + 1
    ctx_rows = w.h_rows(layer, 0, 0, 45)
    W = [w.weight(k) for k in "qkv"]
    res = w.residual(it)
    cache = oracle.OracleCache(w.fmt, w.d, w.n_pre, w.L_max)
    cache.append(layer, 0, 0, ctx_rows)
    want, wf, wfi, _ = oracle.decode_iteration(cache, it, [2], [45], w.h_new(it)[:1], *W, w.H, w.hd, res,
                                               w.threshold, np.zeros(1, np.uint8), np.full(1, -1, np.int32))
    cc, cs = oracle.cpp.quantize_rows(ctx_rows, fmt)
    got, gf, gfi, codes, scales = oracle.cpp.decode_lane(fmt, cc, cs, w.h_new(it)[0], *W, w.H, w.hd, residual=res[0],
                                                         threshold=w.threshold, it=it, loops=2)
    assert np.max(np.abs(got - want[0])) <= 1e-12 * max(1.0, np.max(np.abs(want)))
    assert (gf, gfi) == (int(wf[0]), int(wfi[0]))
    rc, rs = cache.read_rows(layer, 0, 46)
    assert np.array_equal(codes, rc)
    if fmt != oracle.FMT_FP16:
        assert np.array_equal(scales.view(np.uint8), rs.view(np.uint8))
