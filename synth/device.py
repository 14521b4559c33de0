"""Put a synthetic workload on the GPU: weights, per-lane counts, new-token rows,
residuals, and a store-h cache whose context rows are written through the
library's own append call.

Host rows come from the seeded generator (``synth.c``); nothing here computes
any part of the method.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

import store_kv_attention_b200 as tl

from .workloads import Workload


class DeviceWorkload:
    def __init__(self, w: Workload, device: str = "cuda", flag_mix: bool = False, fill: bool = True,
                 n_lanes_ws: Optional[int] = None, max_ctx: Optional[int] = None, split_rows: int = 0):
        self.w = w
        self.device = device
        self.desc = tl.StoreHDesc(w.d, w.H, w.hd, w.n_pre, w.L_max, w.B, max_ctx or w.max_ctx, w.fmt)
        self.cache = tl.StoreHCache(self.desc, device=device, n_lanes=n_lanes_ws, split_rows=split_rows)
        self.W = {k: self._f16(w.weight(k)).to(device) for k in "qkv"}
        self.loops = torch.tensor(w.loops, dtype=torch.int32, device=device)
        self.ctx = torch.tensor(w.ctx, dtype=torch.int32, device=device)
        self.h_new = torch.stack([self._f16(w.h_new(it)) for it in range(w.L_max)]).to(device)
        self.residual = torch.stack([torch.from_numpy(w.residual(it, flag_mix)) for it in range(w.L_max)]).to(device)
        self.out = torch.full((w.L_max, w.B, w.H, w.hd), float("nan"), dtype=torch.float32, device=device)
        self.reset_flags()
        if fill:
            self.fill_context()

    @staticmethod
    def _f16(a: np.ndarray) -> torch.Tensor:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16)

    def reset_flags(self) -> None:
        B = self.w.B
        if getattr(self, "flags", None) is None:
            self.flags = torch.zeros(B, dtype=torch.uint8, device=self.device)
            self.first = torch.full((B,), -1, dtype=torch.int32, device=self.device)
            self.norms = torch.full((self.w.L_max, B), float("nan"), dtype=torch.float32, device=self.device)
        else:
            self.flags.zero_()
            self.first.fill_(-1)
            self.norms.fill_(float("nan"))

    def fill_context(self, layers=None) -> None:
        """Write context positions 0..ctx[b]-1 of every loop layer a lane reads."""
        w = self.w
        max_rows = max(w.ctx)
        if max_rows == 0:
            return
        stage = torch.empty((w.B, max_rows, w.d), dtype=torch.float16, device=self.device)
        host = torch.empty((max_rows, w.d), dtype=torch.float16).pin_memory()
        host_np = host.numpy().view(np.float16)
        zeros = torch.zeros(w.B, dtype=torch.int32, device=self.device)
        for layer in (layers if layers is not None else range(w.n_pre, w.n_pre + w.L_max)):
            counts = []
            for b in range(w.B):
                active = layer < w.n_pre + w.loops[b]
                n = w.ctx[b] if active else 0
                counts.append(n)
                if n:
                    w.h_rows_into(host_np[:n], layer, b, 0)
                    stage[b, :n].copy_(host[:n], non_blocking=False)
            row_count = torch.tensor(counts, dtype=torch.int32, device=self.device)
            tl.append(self.cache, layer, stage, zeros, row_count=row_count)
        torch.cuda.synchronize()

    def append_new(self, it: int, stream=None) -> None:
        """Write the new token's row of iteration ``it`` at position ctx[b] (active lanes)."""
        tl.append(self.cache, self.w.n_pre + it, self.h_new[it].unsqueeze(1), self.ctx, loops=self.loops,
                  stream=stream)

    def decode(self, it: int, fused_check: bool = True, stream=None, append: bool = False) -> None:
        """Iteration `it` of the decode; with append=True the new token's row is written by the
        same call (tl_storeh_append_attn_decode) instead of a separate append_new."""
        w = self.w
        tl.attn_decode(self.cache, it, self.loops, self.ctx, self.h_new[it], self.W["q"], self.W["k"], self.W["v"],
                       self.out[it], residual=self.residual[it] if fused_check else None, threshold=w.threshold,
                       abort_flags=self.flags, first_abort_iter=self.first, norms_out=self.norms[it],
                       stream=stream, append=append)

    def step(self, stream=None, fused_append: bool = False) -> None:
        """One decode step: every loop iteration, append then attend (with the safety check),
        as two calls or (fused_append) as one."""
        for it in range(self.w.L_max):
            if fused_append:
                self.decode(it, stream=stream, append=True)
            else:
                self.append_new(it, stream)
                self.decode(it, stream=stream)
