"""CPU oracle for the store-h decode-attention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports or calls this
module; only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg do.  It shares no code with the CUDA library.

What it computes, and where the pages define it:

* Store-h cache.  Instead of K and V, the cache keeps the pre-QKV hidden
  state h of every (layer, token); at attention time K = W_k h and V = W_v h
  are rebuilt with the loop block's shared weights.
  [Novel Contributions, "Novel Mechanism: Store-h KV Cache";
  Architecture-Exclusive Features, "Store-h KV cache"]
* Storage modes FP16-h / INT8-h / INT4-h [Architecture-Exclusive Features,
  "Store-h KV cache", mode table].  The pages give only the byte counts, so the
  quantisers follow the workload statement: INT8 symmetric per token,
  scale = amax/127 in fp32; INT4 symmetric per group of 64 along d,
  scale = fp16(amax/7); round half to even; two codes per byte, low nibble
  first.  Dequantisation is exact in FP64.
* Variable-L cache: n_pre + L_max layers; loop iteration i fills and reads
  layer n_pre + i, which stays valid for every L >= i+1; a lane with loop
  count L never touches layers >= n_pre + L.
  [Architecture-Exclusive Features, "Variable-L KV cache", "L-aware batching"]
* Per-iteration safety check: the L2 norm of the FP32 residual after every
  loop iteration; generation aborts when it exceeds the threshold.
  [Novel Contributions, "Novel: Per-Iteration Safety Check";
  Architecture-Exclusive Features, "Per-iteration safety check"]

Readings where the pages are silent (each listed in the design notes):
the new token is appended to the cache first and read back quantised like
every other row, while its query comes from the unquantised h; softmax scale
1/sqrt(head_dim); no positional rotation and no biases; "exceeds" is strict;
flags are sticky and a lane that aborted is still computed.

Every function below is pinned by a ``-m "not gpu"`` test against something
other than itself (library attention over explicitly stored K/V, closed
forms, hand-worked quantiser cases, invariants); see ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import numpy as np

FMT_FP16 = 0
FMT_INT8 = 1
FMT_INT4 = 2
INT4_GROUP = 64


# --------------------------------------------------------------------------- layout sizes
def row_code_bytes(fmt: int, d: int) -> int:
    """Bytes of codes per cached row."""
    return {FMT_FP16: 2 * d, FMT_INT8: d, FMT_INT4: d // 2}[fmt]


def row_scale_count(fmt: int, d: int) -> int:
    """Scales per cached row (fp32 for INT8, fp16 for INT4)."""
    return {FMT_FP16: 0, FMT_INT8: 1, FMT_INT4: d // INT4_GROUP}[fmt]


# --------------------------------------------------------------------------- quantiser
def quantize_rows(h: np.ndarray, fmt: int) -> Tuple[np.ndarray, np.ndarray]:
    """Quantise fp16 rows h [n, d] for the cache.

    Returns (codes uint8 [n, row_code_bytes], scales [n, row_scale_count])
    with scales float32 (INT8) or float16 (INT4) and an empty array for FP16.

    INT8, per token: amax = max|x| (fp32, exact from fp16); scale = amax / 127
    (fp32 IEEE division); code = clamp(rne(x / scale), -127, 127) with x/scale an
    fp32 IEEE division.  INT4, per group of 64: scale = fp16_rne(amax / 7.0f);
    code = clamp(rne(x / float(scale)), -7, 7); byte j of a group holds element
    2j in its low nibble and 2j+1 in its high nibble (two's complement).
    A zero scale gives all-zero codes.
    """
    h = np.asarray(h)
    assert h.dtype == np.float16 and h.ndim == 2
    n, d = h.shape
    if fmt == FMT_FP16:
        return h.copy().view(np.uint8).reshape(n, 2 * d), np.zeros((n, 0), np.float32)
    x = h.astype(np.float32)  # exact
    if fmt == FMT_INT8:
        amax = np.max(np.abs(x), axis=1)
        scale = (amax / np.float32(127.0)).astype(np.float32)
        codes = np.zeros((n, d), dtype=np.int8)
        nz = scale > 0
        q = x[nz] / scale[nz, None]           # fp32 / fp32 -> fp32, IEEE
        codes[nz] = np.clip(np.rint(q), -127, 127).astype(np.int8)   # rint: ties to even
        return codes.view(np.uint8), scale.reshape(n, 1)
    if fmt == FMT_INT4:
        assert d % INT4_GROUP == 0
        g = x.reshape(n, d // INT4_GROUP, INT4_GROUP)
        amax = np.max(np.abs(g), axis=2)
        scale16 = (amax / np.float32(7.0)).astype(np.float32).astype(np.float16)  # RNE to fp16
        div = scale16.astype(np.float32)
        codes = np.zeros(g.shape, dtype=np.int8)
        nz = div > 0
        q = g[nz] / div[nz][:, None]
        codes[nz] = np.clip(np.rint(q), -7, 7).astype(np.int8)
        nib = (codes.reshape(n, d).astype(np.int16) & 0xF).astype(np.uint8)
        packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
        return packed, scale16
    raise ValueError(fmt)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """uint8 [n, d/2] -> int8 codes [n, d] (low nibble = even element)."""
    lo = (packed & 0xF).astype(np.int8)
    hi = (packed >> 4).astype(np.int8)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, fmt: int, d: int) -> np.ndarray:
    """Exact FP64 dequantisation: h_hat = code * scale (fp16 rows are returned as is)."""
    n = codes.shape[0]
    if fmt == FMT_FP16:
        return np.ascontiguousarray(codes).view(np.float16).reshape(n, d).astype(np.float64)
    if fmt == FMT_INT8:
        return codes.view(np.int8).astype(np.float64) * scales.astype(np.float64).reshape(n, 1)
    if fmt == FMT_INT4:
        c = unpack_int4(codes).astype(np.float64).reshape(n, d // INT4_GROUP, INT4_GROUP)
        return (c * scales.astype(np.float64)[:, :, None]).reshape(n, d)
    raise ValueError(fmt)


# --------------------------------------------------------------------------- attention
def _softmax(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - np.max(s))
    return e / np.sum(e)


def attend_explicit(h_hat: np.ndarray, h_new: np.ndarray, W_q: np.ndarray, W_k: np.ndarray,
                    W_v: np.ndarray, H: int, hd: int) -> np.ndarray:
    """Decode attention of one lane at one loop iteration, rebuilding K and V explicitly.

    h_hat [n, d]: the dequantised cached rows 0..n-1 of the iteration's layer
    (row n-1 is the new token, already appended).  q = W_q h_new from the
    unquantised fp16 h_new; K_c = W_k h_c and V_c = W_v h_c for every row
    (weights row-major [out, in]); per head j (rows j*hd..(j+1)*hd-1 of q, K,
    V): s_c = q_j . K_cj / sqrt(hd), p = softmax(s), o_j = sum_c p_c V_cj.
    All FP64.  Returns o [H, hd].
    """
    d = W_q.shape[0]
    assert d == H * hd
    Wq, Wk, Wv = (np.asarray(w, dtype=np.float64) for w in (W_q, W_k, W_v))
    q = Wq @ np.asarray(h_new, dtype=np.float64)
    K = h_hat @ Wk.T
    V = h_hat @ Wv.T
    out = np.empty((H, hd), dtype=np.float64)
    for j in range(H):
        cols = slice(j * hd, (j + 1) * hd)
        p = _softmax((K[:, cols] @ q[cols]) / math.sqrt(hd))
        out[j] = p @ V[:, cols]
    return out


def attend_absorbed(h_hat: np.ndarray, h_new: np.ndarray, W_q: np.ndarray, W_k: np.ndarray,
                    W_v: np.ndarray, H: int, hd: int) -> np.ndarray:
    """The same result through the algebraically equal absorbed form.

    Per head j: qt_j = W_k[j]^T q_j (a d-vector), s_c = qt_j . h_c / sqrt(hd),
    p = softmax(s), u_j = sum_c p_c h_c, o_j = W_v[j] u_j, where W_k[j] and
    W_v[j] are the hd rows of head j.  Equal to :func:`attend_explicit` up to
    FP64 rounding (pinned by a test); used where the explicit rebuild is too
    slow on a CPU (large sampled lanes).
    """
    d = W_q.shape[0]
    assert d == H * hd
    Wq, Wk, Wv = (np.asarray(w, dtype=np.float64) for w in (W_q, W_k, W_v))
    q = Wq @ np.asarray(h_new, dtype=np.float64)
    out = np.empty((H, hd), dtype=np.float64)
    for j in range(H):
        rows = slice(j * hd, (j + 1) * hd)
        qt = Wk[rows].T @ q[rows]
        p = _softmax((h_hat @ qt) / math.sqrt(hd))
        u = p @ h_hat
        out[j] = Wv[rows] @ u
    return out


# --------------------------------------------------------------------------- safety check
def residual_norm_check(residual: np.ndarray, threshold: float, it: int, loops: np.ndarray,
                        abort_flags: np.ndarray, first_abort_iter: np.ndarray
                        ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Per-lane check after loop iteration ``it``.

    For each lane b with it < loops[b]: n2 = sum_k r_k^2 with every term exact
    in FP64; the lane aborts iff n2 > threshold^2 (strict; threshold taken as
    the fp32 value).  Flags are sticky; first_abort_iter[b] records the first
    iteration that set the flag.  Lanes with it >= loops[b] are left as they
    are.  Returns (flags, first_abort_iter, norms) with norms = sqrt(n2) for
    active lanes and NaN for inactive ones.
    """
    r = np.asarray(residual, dtype=np.float32).astype(np.float64)
    thr = float(np.float32(threshold))
    flags = np.array(abort_flags, dtype=np.uint8, copy=True)
    first = np.array(first_abort_iter, dtype=np.int32, copy=True)
    norms = np.full(r.shape[0], np.nan)
    for b in range(r.shape[0]):
        if it >= int(loops[b]):
            continue
        n2 = float(np.sum(r[b] * r[b]))
        norms[b] = math.sqrt(n2)
        if n2 > thr * thr:
            if flags[b] == 0:
                first[b] = it
            flags[b] = 1
    return flags, first, norms


# --------------------------------------------------------------------------- cache + step
class OracleCache:
    """The variable-L store-h cache: n_pre + L_max layers, lanes, positions.

    Rows are kept quantised, exactly as :func:`quantize_rows` produced them.
    Reads go through :meth:`read_rows`, which tests may wrap to record which
    (layer, lane, position) ranges a decode touches.
    """

    def __init__(self, fmt: int, d: int, n_pre: int, L_max: int):
        self.fmt, self.d, self.n_pre, self.L_max = fmt, d, n_pre, L_max
        self.rows: Dict[Tuple[int, int], Tuple[np.ndarray, np.ndarray]] = {}

    @property
    def n_layers(self) -> int:
        return self.n_pre + self.L_max

    def append(self, layer: int, lane: int, pos0: int, h: np.ndarray) -> None:
        """Quantise h [n, d] and store it at positions pos0..pos0+n-1."""
        assert 0 <= layer < self.n_layers
        codes, scales = quantize_rows(h, self.fmt)
        key = (layer, lane)
        cb, sc = row_code_bytes(self.fmt, self.d), row_scale_count(self.fmt, self.d)
        end = pos0 + codes.shape[0]
        old_c, old_s = self.rows.get(key, (np.zeros((0, cb), np.uint8),
                                           np.zeros((0, sc), scales.dtype if sc else np.float32)))
        if old_c.shape[0] < end:
            grow = end - old_c.shape[0]
            old_c = np.concatenate([old_c, np.zeros((grow, cb), np.uint8)])
            old_s = np.concatenate([old_s, np.zeros((grow, sc), old_s.dtype)])
        old_c[pos0:end] = codes
        old_s[pos0:end] = scales
        self.rows[key] = (old_c, old_s)

    def read_rows(self, layer: int, lane: int, n: int) -> Tuple[np.ndarray, np.ndarray]:
        codes, scales = self.rows[(layer, lane)]
        return codes[:n], scales[:n]


def decode_iteration(cache: OracleCache, it: int, loops, ctx_len, h_new: np.ndarray,
                     W_q: np.ndarray, W_k: np.ndarray, W_v: np.ndarray, H: int, hd: int,
                     residual: Optional[np.ndarray], threshold: float,
                     abort_flags: np.ndarray, first_abort_iter: np.ndarray,
                     form: str = "explicit"):
    """One loop iteration ``it`` of store-h decode for a batch of lanes.

    For every lane b with it < loops[b]: append the new token's h at layer
    n_pre+it, position ctx_len[b]; attend over positions 0..ctx_len[b] of that
    layer; then run the residual check.  Inactive lanes produce no output
    (NaN rows here) and keep their flags.  Returns (out [B, H, hd] FP64,
    flags, first_abort_iter, norms).
    """
    B = len(loops)
    layer = cache.n_pre + it
    out = np.full((B, H, hd), np.nan)
    attend = attend_explicit if form == "explicit" else attend_absorbed
    for b in range(B):
        if it >= int(loops[b]):
            continue
        c = int(ctx_len[b])
        cache.append(layer, b, c, h_new[b:b + 1])
        codes, scales = cache.read_rows(layer, b, c + 1)
        h_hat = dequantize_rows(codes, scales, cache.fmt, cache.d)
        out[b] = attend(h_hat, h_new[b], W_q, W_k, W_v, H, hd)
    flags, first, norms = abort_flags, first_abort_iter, np.full(B, np.nan)
    if residual is not None:
        flags, first, norms = residual_norm_check(residual, threshold, it, np.asarray(loops),
                                                  abort_flags, first_abort_iter)
    return out, flags, first, norms
