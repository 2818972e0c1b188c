"""The LLM.int8() linear layer split by output channels across the ranks of a process group.

Each output channel of the layer depends only on X (the same on every rank) and on its own row
of W, scale and bias ([P5] "PyTorch 2.9 支持 LLM.int8()" items 1-3: per-channel weight scales,
per-row activation scales, outlier columns found from X alone), so an N-split needs no
exchange before the product: every rank finds the same outlier columns and activation scales
from its copy of X, runs the whole layer on its slice of channels with the library's kernels,
and one all-gather joins the slices of Y.  No other collective is involved, and nothing here
reads another GPU's memory outside the collective.

Shards have equal width (the last rank's slice is padded with zero weight rows, whose outputs
are dropped), a multiple of 16 channels, so that the gather moves one tensor of the same shape
from every rank.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist

import int8_mixed_precision_absmax_b200 as i8


@dataclass(frozen=True)
class Shard:
    rank: int
    world: int
    n_total: int      # output channels of the whole layer
    width: int        # channels per rank (padded), a multiple of 16
    lo: int           # first channel of this rank
    hi: int           # one past the last real channel of this rank (<= lo + width)

    @property
    def real(self) -> int:
        return self.hi - self.lo


def plan_shards(n_total: int, world: int) -> list[Shard]:
    """Equal-width slices of the output channels, each a multiple of 16 wide."""
    if n_total <= 0 or world <= 0:
        raise ValueError("n_total and world must be positive")
    width = -(-n_total // world)
    width = -(-width // 16) * 16
    shards = []
    for r in range(world):
        lo = min(r * width, n_total)
        hi = min(lo + width, n_total)
        shards.append(Shard(r, world, n_total, width, lo, hi))
    return shards


def shard_rows(t: torch.Tensor | None, shard: Shard) -> torch.Tensor | None:
    """Rows [lo, hi) of a per-channel tensor, zero-padded to the shard width."""
    if t is None:
        return None
    out = torch.zeros((shard.width,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    out[: shard.real] = t[shard.lo: shard.hi]
    return out


def gather_columns(y_local: torch.Tensor, shards: list[Shard], group=None) -> torch.Tensor:
    """Join the ranks' [M, width] slices of Y into [M, n_total] with one all-gather."""
    world = len(shards)
    M, width = y_local.shape
    stacked = torch.empty((world * M, width), dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(stacked, y_local.contiguous(), group=group)
    full = stacked.view(world, M, width).permute(1, 0, 2).reshape(M, world * width)
    n = shards[0].n_total
    return full[:, :n].contiguous()


LocalForward = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor | None, float],
                        torch.Tensor]


def _library_forward(X, Wq, w_scale, bias, threshold):
    return i8.int8_linear_forward(X, Wq, w_scale, bias, threshold)


class ColumnParallelInt8Linear:
    """An Int8Linear whose output channels are split across the ranks of `group`.

    `weight` and `bias` are the whole layer's (every rank passes the same tensors; each keeps
    only its slice).  `local_forward(X, Wq, w_scale, bias, threshold) -> Y` runs the layer on
    this rank's slice; by default the library's kernels on the current CUDA device.
    """

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None = None,
                 threshold: float = i8.DEFAULT_THRESHOLD, group=None,
                 local_forward: LocalForward | None = None,
                 quantize: Callable[[torch.Tensor], tuple[torch.Tensor, torch.Tensor]] | None = None):
        self.group = group
        world = dist.get_world_size(group)
        rank = dist.get_rank(group)
        self.shards = plan_shards(weight.shape[0], world)
        self.shard = self.shards[rank]
        self.in_features = weight.shape[1]
        self.threshold = float(threshold)
        w_local = shard_rows(weight.to(torch.float16), self.shard).contiguous()
        quantize = quantize or i8.int8_quant_weight
        self.Wq, self.w_scale = quantize(w_local)  # per-channel: the slice's own scales
        self.bias = shard_rows(None if bias is None else bias.to(torch.float16), self.shard)
        self.local_forward = local_forward or _library_forward

    def __call__(self, X: torch.Tensor) -> torch.Tensor:
        lead = X.shape[:-1]
        X2 = X.reshape(-1, self.in_features).contiguous()
        y_local = self.local_forward(X2, self.Wq, self.w_scale, self.bias, self.threshold)
        y = gather_columns(y_local, self.shards, self.group)
        return y.reshape(*lead, self.shards[0].n_total)
