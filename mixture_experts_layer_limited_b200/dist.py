"""Multi-GPU plumbing for token-sharded replicas of the layer.

Each rank holds the full layer and routes, permutes, computes and combines
its own tokens; the only exchange is the sum of the per-expert token counts
before the aux-loss-free bias step (xxqk.cn digest §2.2), so that every
replica applies the same bias (loads are global, not per replica).
"""
import torch
import torch.distributed as dist


def world() -> int:
    return dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1


def allreduce_counts_(counts: torch.Tensor) -> torch.Tensor:
    """Sums expert counts over ranks in place (no-op on one rank)."""
    if world() > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM)
    return counts


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (e.g. the device time of the timed region)."""
    if world() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if world() > 1:
        dist.barrier()
