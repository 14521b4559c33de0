"""The five store-h decode workloads, with their seeded synthetic inputs.

Shapes follow the decode configurations of the TinyLoop "Store-h KV cache"
pages (407M-like and 2B-like looped models, FP16-h / INT8-h / INT4-h, mixed
per-lane loop counts).  All values are synthetic: h ~ N(0,1) fp16, weights
~ N(0, 1/d) fp16, residual fp32 ~ N(0,1) times a stated factor.

No arithmetic of the method lives here; the only computation is drawing and
(for the flag-mix variant of the residual) rescaling random rows to a target
L2 norm, which is input construction.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

from . import (TID_CTX, TID_RESIDUAL, TID_WK, TID_WQ, TID_WV, h_rows_f16, h_rows_f16_into,
               normal_f16, normal_f64, row_id, u64)

FMT_FP16 = 0      # h stored as fp16
FMT_INT8 = 1      # int8 codes, one fp32 scale per row (per token)
FMT_INT4 = 2      # int4 codes, one fp16 scale per group of 64 along d


@dataclasses.dataclass
class Workload:
    name: str
    d: int
    H: int
    hd: int
    n_pre: int
    L_max: int
    fmt: int
    seed: int
    ctx: List[int]              # cached positions per lane (the new token sits at ctx[b])
    loops: List[int]            # loop count per lane (<= L_max)
    residual_scale: float
    threshold: float
    outlier_p: float = 0.0
    outlier_mul: float = 1.0
    forced_lanes: int = 0       # lanes forced above the threshold in the flag-mix variant
    lane_ids: Optional[List[int]] = None  # generator lane of each batch position (default: itself)

    def lane_id(self, b: int) -> int:
        return b if self.lane_ids is None else self.lane_ids[b]

    @property
    def B(self) -> int:
        return len(self.ctx)

    @property
    def n_layers(self) -> int:
        return self.n_pre + self.L_max

    @property
    def max_ctx(self) -> int:
        """Positions per (layer, lane) the cache must hold, counting the new token."""
        return max(self.ctx) + 1

    def cached_positions_per_step(self) -> int:
        """Sum over active (lane, iteration) of the lane's cached positions."""
        return int(sum(c * l for c, l in zip(self.ctx, self.loops)))

    # ------------------------------------------------------------ weights
    def weight(self, which: str) -> np.ndarray:
        tid = {"q": TID_WQ, "k": TID_WK, "v": TID_WV}[which]
        return normal_f16(self.seed, tid, 0, self.d * self.d, 1.0 / math.sqrt(self.d)).reshape(self.d, self.d)

    # ------------------------------------------------------------ h rows
    def h_rows(self, layer: int, b: int, pos0: int, n: int) -> np.ndarray:
        """h rows (fp16 [n, d]) of batch lane b at cache coordinate (layer, pos0 .. pos0+n-1)."""
        return h_rows_f16(self.seed, row_id(layer, self.lane_id(b), np.arange(pos0, pos0 + n)), self.d,
                          self.outlier_p, self.outlier_mul)

    def h_rows_into(self, out: np.ndarray, layer: int, b: int, pos0: int) -> None:
        n = out.shape[0]
        h_rows_f16_into(out, self.seed, row_id(layer, self.lane_id(b), np.arange(pos0, pos0 + n)), self.d,
                        self.outlier_p, self.outlier_mul)

    def h_new(self, it: int) -> np.ndarray:
        """New-token h for loop iteration ``it`` (fp16 [B, d]): the row at position ctx[b]
        of cache layer n_pre+it, so context rows and new rows share one stream."""
        layer = self.n_pre + it
        ids = np.array([row_id(layer, self.lane_id(b), self.ctx[b]) for b in range(self.B)], dtype=np.uint64)
        return h_rows_f16(self.seed, ids, self.d, self.outlier_p, self.outlier_mul)

    # ------------------------------------------------------------ residual
    def residual(self, it: int, flag_mix: bool = False) -> np.ndarray:
        """FP32 residual [B, d] checked after iteration ``it``.

        Literal: N(0,1) * residual_scale.  Flag-mix variant: each lane's draw is
        rescaled to L2 norm 0.5*threshold, and the first ``forced_lanes`` lanes
        (at least one) to 2*threshold, so both flag values occur and no lane sits
        near the threshold."""
        out = np.empty((self.B, self.d), dtype=np.float32)
        for b in range(self.B):
            lid = self.lane_id(b)
            z = normal_f64(self.seed, TID_RESIDUAL, (it * 256 + lid) * self.d, self.d)
            if not flag_mix:
                out[b] = (z * self.residual_scale).astype(np.float32)
            else:
                target = 2.0 * self.threshold if lid < max(1, self.forced_lanes) else 0.5 * self.threshold
                out[b] = (z * (target / np.sqrt(np.sum(z * z)))).astype(np.float32)
        return out


def _uniform_ctx(seed: int, n: int, lo: int, hi: int) -> List[int]:
    draws = u64(seed, TID_CTX, 0, n)
    span = hi - lo + 1
    return [int(lo + int(x) % span) for x in draws]


def get_workload(name: str) -> Workload:
    if name == "tiny_fp16":
        # d=256, 4 heads x 64, batch 1, 128 cached positions, n_pre=1, L=2
        return Workload(name, d=256, H=4, hd=64, n_pre=1, L_max=2, fmt=FMT_FP16, seed=0,
                        ctx=[128], loops=[2], residual_scale=1.0, threshold=50.0)
    if name == "fp16_407m":
        # 407M-like: d=1024, 16 heads x 64, batch 1, context 2048, n_pre=2, L=8
        return Workload(name, d=1024, H=16, hd=64, n_pre=2, L_max=8, fmt=FMT_FP16, seed=1,
                        ctx=[2048], loops=[8], residual_scale=4.0, threshold=50.0)
    if name == "int8_b16":
        # INT8-h per token: d=1024, 16 heads x 64, batch 16, context 4096, L=8, 1% outlier rows x8
        return Workload(name, d=1024, H=16, hd=64, n_pre=2, L_max=8, fmt=FMT_INT8, seed=2,
                        ctx=[4096] * 16, loops=[8] * 16, residual_scale=4.0, threshold=50.0,
                        outlier_p=0.01, outlier_mul=8.0)
    if name == "int4_2b":
        # 2B-like INT4-h g64: d=2048, 16 heads x 128, batch 32, context 4096, n_pre=2, L=8
        return Workload(name, d=2048, H=16, hd=128, n_pre=2, L_max=8, fmt=FMT_INT4, seed=3,
                        ctx=[4096] * 32, loops=[8] * 32, residual_scale=4.0, threshold=50.0,
                        forced_lanes=2)
    if name == "int4_mixed":
        # L-aware mixed batch: 48 lanes, 16 each at loops 4 / 16 / 32, ctx ~ U[1024, 8192], L_max=32
        return Workload(name, d=2048, H=16, hd=128, n_pre=2, L_max=32, fmt=FMT_INT4, seed=4,
                        ctx=_uniform_ctx(4, 48, 1024, 8192), loops=[4] * 16 + [16] * 16 + [32] * 16,
                        residual_scale=4.0, threshold=50.0, forced_lanes=2)
    raise KeyError(name)


WORKLOADS = ["tiny_fp16", "fp16_407m", "int8_b16", "int4_2b", "int4_mixed"]


def select_lanes(w: Workload, lanes: List[int]) -> Workload:
    """The same workload restricted to some of its lanes (each keeps its own rows and counts)."""
    w2 = dataclasses.replace(w)
    w2.ctx = [w.ctx[b] for b in lanes]
    w2.loops = [w.loops[b] for b in lanes]
    w2.lane_ids = [w.lane_id(b) for b in lanes]
    return w2


def small_variant(w: Workload, ctx: Optional[List[int]] = None, loops: Optional[List[int]] = None,
                  name: Optional[str] = None) -> Workload:
    """Same shapes/distributions and seed, different lane set (for parity at oracle-friendly sizes)."""
    w2 = dataclasses.replace(w)
    if ctx is not None:
        w2.ctx = list(ctx)
    if loops is not None:
        w2.loops = list(loops)
    if name is not None:
        w2.name = name
    return w2
