"""Multi-GPU forms of the per-layer search: one process per GPU,
``torch.distributed`` for the plumbing.

The search shards naturally.  Layers are searched independently
(compassingai.com AWQ concept page, flow note: each layer searched on its own;
robocikowo.com AWQ page, "parallelism": layer by layer, parallel within a
layer), and within a layer each output column contributes its own terms to
L(alpha) = sum_n L_n(alpha) (its own groups, codes and output).  Two forms:

* layer sharding - every rank searches whole layers; no exchange is needed to
  compute anything, results are only collected;
* column sharding - every rank searches a slice of one layer's output columns
  (X replicated) and one all-reduce of the n_alpha fp64 partial losses gives
  every rank the layer's L(alpha), from which all take the same argmin.

The per-shard search is a callable, so the orchestration is the same for the
CUDA path (``awq.search`` on the rank's GPU, NCCL) and for the tests (gloo on
the CPU with an injected per-shard search).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced [start, end) slice of n items for one rank."""
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def column_shard(D_out: int, world: int, rank: int, align: int = 256) -> Tuple[int, int]:
    """Output-column slice of one rank, in whole multiples of `align` columns
    (the search's column tile), the remainder to the last ranks."""
    tiles = (D_out + align - 1) // align
    t0, t1 = shard_range(tiles, world, rank)
    return min(t0 * align, D_out), min(t1 * align, D_out)


def argmin_lowest(L: torch.Tensor) -> int:
    """Index of the smallest loss, the lowest index among exact ties."""
    best = 0
    vals = L.tolist()
    for i, v in enumerate(vals):
        if v < vals[best]:
            best = i
    return best


def column_sharded_search(shard_loss: Callable[[int, int], torch.Tensor], D_out: int,
                          group: Optional[dist.ProcessGroup] = None, align: int = 256,
                          device: Optional[torch.device] = None) -> Tuple[torch.Tensor, int]:
    """L(alpha) of a whole layer from per-rank column slices.

    shard_loss(c0, c1) returns this rank's fp64 partial losses [n_alpha] over
    output columns [c0, c1) (zeros for an empty slice).  One all-reduce (sum)
    combines them; every rank then holds the same L and takes the same argmin."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    c0, c1 = column_shard(D_out, world, rank, align)
    part = shard_loss(c0, c1).to(torch.float64)
    if device is not None:
        part = part.to(device)
    dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    return part, argmin_lowest(part.cpu())


def layer_sharded_search(n_layers: int, layer_search: Callable[[int], Tuple[torch.Tensor, int]],
                         n_alpha: int, group: Optional[dist.ProcessGroup] = None,
                         device: Optional[torch.device] = None) -> List[Tuple[torch.Tensor, int]]:
    """Independent searches of n_layers layers spread over the ranks.

    layer_search(i) returns (L [n_alpha] fp64, argmin) for layer i and is called
    only for this rank's layers.  The results are collected on every rank (a
    sum all-reduce of a table in which each layer's row is filled by its owner
    only), so every rank returns the full list."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    l0, l1 = shard_range(n_layers, world, rank)
    table = torch.zeros(n_layers, n_alpha + 1, dtype=torch.float64)
    for i in range(l0, l1):
        L, best = layer_search(i)
        table[i, :n_alpha] = L.detach().to("cpu", torch.float64)
        table[i, n_alpha] = float(best)
    if device is not None:
        table = table.to(device)
    dist.all_reduce(table, op=dist.ReduceOp.SUM, group=group)
    table = table.cpu()
    return [(table[i, :n_alpha].clone(), int(table[i, n_alpha].item())) for i in range(n_layers)]


def cuda_shard_loss(X: torch.Tensor, W: torch.Tensor, a: torch.Tensor, alpha_grid: Sequence[float],
                    bits: int = 4, group: int = 128, loss_form: int = 0) -> Callable[[int, int], torch.Tensor]:
    """The per-shard loss of :func:`column_sharded_search` on this rank's GPU:
    the search over columns [c0, c1) of W (X replicated), through the C ABI.
    The slice is searched in place: W + c0 with W's row stride, no copy (c0 is
    a multiple of the 256-column tile, so the slice stays 16-byte aligned)."""
    from . import awq

    def fn(c0: int, c1: int) -> torch.Tensor:
        if c1 <= c0:
            return torch.zeros(len(alpha_grid), dtype=torch.float64, device=X.device)
        Wc = W[:, c0:c1] if c1 - c0 < W.shape[1] else W
        res = awq.search(X, Wc, a, alpha_grid, bits, group, loss_form=loss_form)
        return res.L
    return fn
