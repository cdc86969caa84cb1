"""The allocation pass over several GPUs: matrices sharded by element count.

AQLoRA's allocation pass ("AQLoRA: A Zero-Search Recipe for Fast Quantized LoRA
Fine-Tuning", sections 3.1-3.2) scores every linear matrix by its NF4
reconstruction error and keeps the top K in 16-bit. A matrix's error needs only
that matrix, so with one process per GPU each rank scores the matrices it owns
(the library's error pass on its device), the per-matrix errors are combined with
one all-reduce of an fp64 vector that is zero outside each rank's own entries
(exact: every entry has a single nonzero contribution), and every rank ranks the
same vector with the library's ranking step, so all ranks get the same order and
keep mask. The exchange is L doubles (a few KB for hundreds of matrices).

`torch.distributed` is the plumbing (NCCL on GPUs); no arithmetic of the method
happens here.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def shard_by_numel(numel: Sequence[int], world: int) -> List[int]:
    """Owner rank of each matrix: largest matrices first, each to the rank with the
    fewest elements so far (ties to the lower rank; equal sizes by index), so the
    ranks' element counts differ by at most one matrix."""
    if world < 1:
        raise ValueError("world must be >= 1")
    load = [0] * world
    owner = [0] * len(numel)
    for i in sorted(range(len(numel)), key=lambda j: (-int(numel[j]), j)):
        r = min(range(world), key=lambda k: (load[k], k))
        owner[i] = r
        load[r] += int(numel[i])
    return owner


def sharded_layer_error_rank(weights: Dict[int, torch.Tensor], numel: Sequence[int], K: int,
                             double_quant: bool = False, group=None,
                             errors_fn: Optional[Callable[[List[torch.Tensor]], torch.Tensor]] = None,
                             rank_fn: Optional[Callable[[torch.Tensor, int], Tuple[torch.Tensor, torch.Tensor]]] = None):
    """(err, order, keep) of all len(numel) matrices, identical on every rank.

    weights   this rank's matrices by global index (exactly those shard_by_numel
              assigns to it; each a bf16 tensor on this rank's device)
    numel     element count of every matrix (all ranks pass the same list)
    errors_fn per-matrix fp64 errors of a list of matrices (default: the library's
              error pass); rank_fn (err, K) -> (order, keep) (default: the library's
              ranking step)
    """
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    owners = shard_by_numel(numel, world)
    mine = [i for i, o in enumerate(owners) if o == rank]
    if sorted(weights) != mine:
        raise ValueError(f"rank {rank} holds matrices {sorted(weights)}, its shard is {mine}")
    if errors_fn is None or rank_fn is None:
        from . import api
        if errors_fn is None:
            errors_fn = lambda Ws: api.layer_error_rank(Ws, 0, double_quant=double_quant)[0]  # noqa: E731
        if rank_fn is None:
            rank_fn = api.rank_errors
    device = next(iter(weights.values())).device if weights else (
        torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu"))
    full = torch.zeros(len(numel), dtype=torch.float64, device=device)
    if mine:
        full[torch.tensor(mine, device=device)] = errors_fn([weights[i] for i in mine]).to(torch.float64)
    if world > 1:
        dist.all_reduce(full, group=group)
    order, keep = rank_fn(full, K)
    return full, order, keep
