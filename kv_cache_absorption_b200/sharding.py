"""Layer sharding of the warmup across GPUs (one process per GPU).

"Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption", technical summary section 2: each
layer's dual-stream attention, statistics, Delta W and reconstruction error
depend on that layer only, so the layers of a warmup split across ranks with
no exchange on the data path (layer l on rank l mod world). The one exchange
is the ranking: every rank needs every layer's error to know which K layers
become L-Layers, so the per-layer errors are all-gathered (L x 2 doubles) and
each rank ranks the full vector itself. Delta W stays on the rank that owns
the layer.
"""
from __future__ import annotations

from typing import List

import torch


def owned_layers(n_layers: int, world: int, rank: int) -> List[int]:
    """Layers of ``rank``: l with l mod world == rank, in ascending order."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    return list(range(rank, n_layers, world))


def gather_errors(err_local: torch.Tensor, n_layers: int, world: int, group=None) -> torch.Tensor:
    """All-gather the owned layers' errors ([n_owned, 2], float64, in
    ``owned_layers`` order) into the full [n_layers, 2] table, in layer
    order, on every rank. Works on any torch.distributed backend whose
    tensors live where ``err_local`` lives (gloo: CPU, nccl: CUDA)."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    if err_local.dtype != torch.float64 or err_local.dim() != 2 or err_local.shape[1] != 2:
        raise ValueError("err_local must be a float64 [n_owned, 2] tensor")
    if err_local.shape[0] != len(owned_layers(n_layers, world, rank)):
        raise ValueError("err_local does not match this rank's layers")
    per = -(-n_layers // world)                       # equal-size pieces for all_gather
    piece = torch.zeros(per, 2, dtype=torch.float64, device=err_local.device)
    piece[:err_local.shape[0]] = err_local
    pieces = [torch.empty_like(piece) for _ in range(world)]
    dist.all_gather(pieces, piece, group=group)
    full = torch.empty(n_layers, 2, dtype=torch.float64, device=err_local.device)
    for r in range(world):
        mine = owned_layers(n_layers, world, r)
        full[mine] = pieces[r][:len(mine)]
    return full
