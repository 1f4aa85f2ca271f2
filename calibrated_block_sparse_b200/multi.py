"""Multi-GPU plumbing of the CalibAtt hot path (one process per GPU).

The path shards without data exchange except in one place:

* inference: heads (and videos) are independent; each rank runs its own
  attention calls;
* calibration: the calibration inputs are split across ranks; every rank
  folds its inputs' masks into a local count array, one integer sum over all
  ranks (all-reduce) gives the global counts, and every rank then binarises
  them at rho locally (the mean mask of all inputs, explainer §三).

Only torch.distributed is used here (NCCL on GPUs, gloo on CPU); the compute
stays in libcalibatt.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(n: int, rank: int, world: int):
    """Contiguous share [lo, hi) of n items for `rank` of `world` (sizes differ by at most one)."""
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def allreduce_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Sum uint16 mask counts over all ranks, in place (via int32 on the wire).

    The sum saturates at 65535 like the library's accumulation."""
    if counts.dtype != torch.uint16:
        raise TypeError("counts must be uint16")
    wide = counts.view(torch.int16).to(torch.int32) & 0xFFFF
    dist.all_reduce(wide, op=dist.ReduceOp.SUM, group=group)
    wide.clamp_(max=0xFFFF)
    counts.copy_(wide.to(torch.int16).view(torch.uint16).view(counts.shape))
    return counts


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Max of a scalar over all ranks (timing: the slowest rank sets the time)."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def calibrate_sharded(inputs, heads: int, nb: int, n_inputs: int, eps: float, rho: float = 0.5, group=None,
                      device=None):
    """Calibrate one (t, l) over n_inputs inputs split across the ranks.

    ``inputs(p)`` returns (q, k) bf16 CUDA tensors of input p. Each rank runs
    the single-pass block-energy + greedy-selection kernel on its share, the counts
    are summed over ranks, and the aggregated mask and skip list are built on
    every rank. Returns (mask, row_ptr, col_idx, nnz)."""
    from . import binding
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    lo, hi = shard_range(n_inputs, rank, world)
    counts = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=device)
    ws = None
    for p in range(lo, hi):
        q, k = inputs(p)
        if ws is None:  # single-pass energy: one S per tile; workspace reused over inputs
            ws = torch.empty(binding.energy_workspace_size(q.shape[0], q.shape[1]), dtype=torch.uint8,
                             device=q.device)
        binding.block_energy_1pass(q, k, eps=eps, energy=False, counts=counts, ws=ws)
    binding.check_status(what="calibration")
    if world > 1:
        allreduce_counts(counts, group)
    return binding.aggregate_masks(counts, n_inputs, rho)
