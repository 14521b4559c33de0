"""CPU oracle for the iteration-axis delta cache of h (test infrastructure only).

TEST INFRASTRUCTURE ONLY, like ``storeh_oracle``: only ``tests/`` may use it, and it
shares no code with the CUDA library.

What it computes, and where the pages define it
[Architecture-Exclusive Features, "Iteration-axis delta-KV"; Measured benchmarks,
"iteration-axis delta-KV: full forward-path PPL A/B"]:

* Along the loop iterations a token's hidden state follows a contracting trajectory, so
  instead of quantising every h^l directly the cache keeps, per token, one fp16 anchor h^0
  and, per loop iteration l >= 1, an INT8 delta with one fp16 scale per head (a
  [tokens, n_heads] scale grid per iteration).
* The rows are rebuilt at attention time by a prefix sum, per token and element:
  h^l = h^0 + sum_{i=1..l} scale[i, head] * dh^i, accumulated in FP32.
* The writer forms dh^l = h^l - h^(l-1) and picks the per-head scale.

Readings where the pages are silent (each listed in the design notes):

1. The INT8 per-head quantiser follows the INT4-h group rule with 127 levels: per head of
   hd elements, amax = max |dh| (fp32), scale = fp16_rne(amax / 127.0f),
   code = clamp(rne(dh / float(scale)), -127, 127) with an fp32 IEEE division; a zero scale
   gives zero codes.  The fp16 scale is the stored value and the divisor.
2. dh^l is taken against a reference state h_ref^(l-1).  Default (``reference="rebuilt"``):
   the state the cache itself rebuilds for iteration l-1, as the FP32 prefix sum, so the
   rebuild error of iteration l is that of dh^l alone.  This is the reading the pages' own
   account supports: a direct quantiser pays full precision every iteration while the delta
   scheme pays only the shrinking |dh^l|, and its advantage over direct INT8 grows with L
   (their reconstruction-error study, 1.68x at L=8 to 2.85x at L=32).  The alternative
   (``reference="exact"``) uses the exact previous state h^(l-1); its error carries every
   earlier iteration's rounding, and its advantage does not grow with L.  Both are pinned.
   The difference h^l - h_ref is formed in fp32 (exact for the fp16 exact reference).
3. Iteration l of the loop reads the anchor and the deltas 1..l only; deltas of later
   iterations are never read (the same variable-L addressing as the store-h cache).
4. The rebuild that attention sees is the definition, h^0 + sum scale * code in exact FP64;
   the FP32 prefix sum (``prefix_sum_fp32``) is the pages' stated precision and is what the
   rebuilt reference of reading 2 uses, so a writer on the GPU can make the same integer
   decisions.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

DELTA_QMAX = 127


def _heads(x: np.ndarray, n_heads: int) -> np.ndarray:
    n, d = x.shape
    assert d % n_heads == 0
    return x.reshape(n, n_heads, d // n_heads)


def quantize_delta_heads(delta: np.ndarray, n_heads: int) -> Tuple[np.ndarray, np.ndarray]:
    """Quantise fp32 deltas [n, d] per head (reading 1).

    Returns (codes int8 [n, d], scales fp16 [n, n_heads])."""
    x = np.asarray(delta)
    assert x.dtype == np.float32 and x.ndim == 2
    n, d = x.shape
    g = _heads(x, n_heads)
    amax = np.max(np.abs(g), axis=2)                                              # fp32, exact
    scale16 = (amax / np.float32(DELTA_QMAX)).astype(np.float32).astype(np.float16)  # fp32 division, RNE to fp16
    div = scale16.astype(np.float32)
    codes = np.zeros(g.shape, dtype=np.int8)
    nz = div > 0
    q = g[nz] / div[nz][:, None]                                                  # fp32 / fp32, IEEE
    codes[nz] = np.clip(np.rint(q), -DELTA_QMAX, DELTA_QMAX).astype(np.int8)      # rint: ties to even
    return codes.reshape(n, d), scale16


def dequantize_delta(codes: np.ndarray, scales: np.ndarray, n_heads: int) -> np.ndarray:
    """Exact FP64 value of one iteration's deltas: code * scale of its head, [n, d]."""
    n, d = codes.shape
    c = _heads(codes.astype(np.float64), n_heads)
    return (c * scales.astype(np.float64)[:, :, None]).reshape(n, d)


def prefix_sum_fp32(anchor: np.ndarray, codes: np.ndarray, scales: np.ndarray, l: int,
                    n_heads: int) -> np.ndarray:
    """The pages' FP32 rebuild of iteration l: acc = float(h^0), then acc += scale_i * code_i
    for i = 1..l in order, each addition rounded to fp32 (each product is exact in fp32:
    an 11-bit scale times an 8-bit code).  codes [L, n, d], scales [L, n, H]; level i is
    index i-1."""
    acc = anchor.astype(np.float32)
    for i in range(1, l + 1):
        n, d = acc.shape
        term = (_heads(codes[i - 1].astype(np.float32), n_heads) *
                scales[i - 1].astype(np.float32)[:, :, None]).reshape(n, d)
        acc = (acc + term).astype(np.float32)
    return acc


def reconstruct(anchor: np.ndarray, codes: np.ndarray, scales: np.ndarray, l: int,
                n_heads: int) -> np.ndarray:
    """h^l as the cache defines it, exactly in FP64: h^0 + sum_{i=1..l} scale_i * code_i.
    Reads the anchor and levels 1..l only (reading 3)."""
    h = anchor.astype(np.float64)
    for i in range(1, l + 1):
        h = h + dequantize_delta(codes[i - 1], scales[i - 1], n_heads)
    return h


def encode_trajectory(traj: np.ndarray, n_heads: int, reference: str = "rebuilt"
                      ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Write side for tokens whose states along the loop are traj [L+1, n, d] (fp16):
    traj[0] is the anchor, traj[l] the state of iteration l.

    Returns (anchor fp16 [n, d], codes int8 [L, n, d], scales fp16 [L, n, H]) with level l
    at index l-1; dh^l = traj[l] - reference state of l-1 (reading 2)."""
    traj = np.asarray(traj)
    assert traj.dtype == np.float16 and traj.ndim == 3
    assert reference in ("exact", "rebuilt")
    L = traj.shape[0] - 1
    n, d = traj.shape[1:]
    anchor = traj[0].copy()
    codes = np.zeros((L, n, d), dtype=np.int8)
    scales = np.zeros((L, n, n_heads), dtype=np.float16)
    for l in range(1, L + 1):
        if reference == "exact":
            ref = traj[l - 1].astype(np.float32)
        else:
            ref = prefix_sum_fp32(anchor, codes, scales, l - 1, n_heads)
        delta = (traj[l].astype(np.float32) - ref).astype(np.float32)
        codes[l - 1], scales[l - 1] = quantize_delta_heads(delta, n_heads)
    return anchor, codes, scales


def delta_cache_bytes(d: int, n_heads: int, L: int, n_tokens: int) -> int:
    """Bytes of one loop block's delta cache for n_tokens tokens: the fp16 anchor (2d per
    token) plus, per iteration, d INT8 codes and n_heads fp16 scales per token."""
    return n_tokens * (2 * d + L * (d + 2 * n_heads))
