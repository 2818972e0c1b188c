"""The LLM.int8() linear layer split by tokens (rows of X) across the ranks of a process group.

A row of Y depends on its own row of X and on the set O of outlier columns, and O depends on
every row of X: a column is an outlier when its |x| exceeds the threshold in any row ([P2]
"8位量化实战：离群值处理与显存优化避坑指南" section 2.3).  The per-row activation scale of
[P5] "PyTorch 2.9 支持 LLM.int8()" item 2 is then taken over the row's own regular columns.
So a row split needs one exchange before the product, and only one:

  1. every rank takes the column maxima of |X| over its rows (the library's statistics kernel),
  2. one all-reduce with MAX makes them the maxima over all rows (K floats),
  3. every rank appends one row to its X holding, in each column whose maximum exceeds the
     threshold, that maximum, and zero elsewhere (the library's int8_outlier_row), and runs
     the whole layer on it with the library's kernels.

The appended row makes the rank's own outlier set the global one (it exceeds the threshold
exactly in the global outlier columns, and no real row exceeds it anywhere else), and it leaves
the scale and the codes of every real row as the unsplit layer computes them; its output row is
dropped.  The weights are replicated on every rank.  The per-tensor activation scale (one scale
over all rows) is not offered here: it would need a second exchange.
"""
from __future__ import annotations

import math
from typing import Callable

import torch
import torch.distributed as dist

import int8_mixed_precision_absmax_b200 as i8

LocalForward = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor | None, float],
                        torch.Tensor]


def _library_forward(X, Wq, w_scale, bias, threshold):
    return i8.int8_linear_forward(X, Wq, w_scale, bias, threshold)


def _library_column_absmax(X: torch.Tensor) -> torch.Tensor:
    return i8.int8_activation_stats(X)[1]


def _library_outlier_row(col_max: torch.Tensor, threshold: float) -> torch.Tensor:
    return i8.int8_outlier_row(col_max.to(torch.float32).contiguous(), threshold)


class RowParallelInt8Linear:
    """An Int8Linear whose tokens are split across the ranks of `group`.

    Every rank passes the whole layer's `weight` and `bias` and its own rows of X (any number,
    zero included).  `local_forward(X, Wq, w_scale, bias, threshold) -> Y`,
    `column_absmax(X) -> float32 [K]` and `outlier_row(col_max, threshold) -> float16 [K]` run
    on this rank; by default the library's kernels on the current CUDA device.
    """

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None = None,
                 threshold: float = i8.DEFAULT_THRESHOLD, group=None,
                 local_forward: LocalForward | None = None,
                 quantize: Callable[[torch.Tensor], tuple[torch.Tensor, torch.Tensor]] | None = None,
                 column_absmax: Callable[[torch.Tensor], torch.Tensor] | None = None,
                 outlier_row: Callable[[torch.Tensor, float], torch.Tensor] | None = None):
        if math.isnan(threshold):
            raise ValueError("threshold is NaN")
        self.group = group
        self.out_features, self.in_features = weight.shape
        self.threshold = float(threshold)
        quantize = quantize or i8.int8_quant_weight
        self.Wq, self.w_scale = quantize(weight.to(torch.float16).contiguous())
        self.bias = None if bias is None else bias.to(torch.float16).contiguous()
        self.local_forward = local_forward or _library_forward
        self.column_absmax = column_absmax or _library_column_absmax
        self.outlier_row = outlier_row or _library_outlier_row

    def global_column_absmax(self, X2: torch.Tensor) -> torch.Tensor:
        """max over the rows of every rank of |X[:, j]| (the one exchange of the split)."""
        if X2.shape[0] > 0:
            col = self.column_absmax(X2).to(torch.float32).contiguous()
        else:
            col = torch.zeros(self.in_features, dtype=torch.float32, device=X2.device)
        dist.all_reduce(col, op=dist.ReduceOp.MAX, group=self.group)
        return col

    def __call__(self, X: torch.Tensor) -> torch.Tensor:
        lead = X.shape[:-1]
        X2 = X.reshape(-1, self.in_features).to(torch.float16).contiguous()
        M = X2.shape[0]
        extra = self.outlier_row(self.global_column_absmax(X2), self.threshold)
        if M == 0:
            return X2.new_empty(*lead, self.out_features)
        Xa = torch.cat([X2, extra.to(X2.device).view(1, -1)], dim=0)
        Y = self.local_forward(Xa, self.Wq, self.w_scale, self.bias, self.threshold)
        return Y[:M].reshape(*lead, self.out_features)
