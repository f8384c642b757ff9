"""The sharded-linear path composed from the C-ABI calls.

Layout helpers (views and one-time weight packing, done with torch as plain
data movement) and the block orchestration: RMSNorm -> column-parallel c_fc
with GELU -> row-parallel c_proj with the partial-sum reduction (and the
residual) fused in, per the nanotron "MLP Module" and the google-research
residual section.  Each step is one call into libtpl.so.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from ._tpl import (Partition, tpl_column_linear, tpl_partition_subparams, tpl_rmsnorm,
                   tpl_row_linear_reduce)


def shard_views(y: torch.Tensor, p: Partition, M: int) -> List[torch.Tensor]:
    """Rank r's ``[M, shard_width[r]]`` view of a column-linear output buffer."""
    out = []
    for r in range(p.tp_size):
        base, w = M * p.shard_base[r], p.shard_width[r]
        out.append(y.view(-1)[base:base + M * w].view(M, w))
    return out


def pack_row_weight(w2_full: torch.Tensor, k_w: Sequence[int]) -> torch.Tensor:
    """Rank-major packing of an unsharded ``[N, K]`` c_proj weight.

    Rank r's block ``[N, k_w[r]]`` holds columns ``sum(k_w[:r]) ..`` of the
    weight, i.e. the slice that rank holds in a row-parallel layout.
    """
    blocks, off = [], 0
    for k in k_w:
        blocks.append(w2_full[:, off:off + k].contiguous().view(-1))
        off += k
    return torch.cat(blocks)


class TPMLP:
    """One TP MLP block: ``[x +] c_proj(act(c_fc(rmsnorm(x))))``, all shards on one GPU."""

    def __init__(self, w1: torch.Tensor, w2_full: torch.Tensor, tp: int, act: str,
                 scale: Optional[torch.Tensor] = None, centered: bool = False,
                 norm: bool = True, residual: bool = False, eps: float = 1e-6):
        self.inter, self.hidden = w1.shape
        self.part = tpl_partition_subparams([self.inter], tp, 1)
        self.k_w = [self.part.shard_width[r] for r in range(tp)]
        self.w1 = w1.contiguous()
        self.w2 = pack_row_weight(w2_full, self.k_w)
        self.act, self.scale, self.centered = act, scale, centered
        self.norm, self.residual, self.eps = norm, residual, eps
        self._bufs = {}

    def _buf(self, name, numel, like):
        b = self._bufs.get(name)
        if b is None or b.numel() < numel or b.dtype != like.dtype or b.device != like.device:
            b = torch.empty(numel, dtype=like.dtype, device=like.device)
            self._bufs[name] = b
        return b[:numel]

    def __call__(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
        M = x.numel() // self.hidden
        xn = x
        if self.norm:
            xn = self._buf("xn", x.numel(), x).view(M, self.hidden)
            tpl_rmsnorm(x.view(M, self.hidden), self.scale, self.centered, self.eps, y=xn,
                        stream=stream)
        h = self._buf("h", M * self.inter, x)
        tpl_column_linear(self.part, xn.view(M, self.hidden), self.w1, None, self.act, y=h,
                          stream=stream)
        if out is None:
            out = torch.empty((M, self.hidden), dtype=x.dtype, device=x.device)
        tpl_row_linear_reduce(h, self.k_w, M, self.w2, None,
                              x.view(M, self.hidden) if self.residual else None, y=out,
                              stream=stream)
        return out


class TPStack:
    """``x <- x + MLP(RMSNorm(x))`` over several layers, in place on x."""

    def __init__(self, layers: Sequence[TPMLP]):
        self.layers = list(layers)

    def __call__(self, x: torch.Tensor, stream=None):
        for layer in self.layers:
            layer(x, out=x, stream=stream)
        return x
