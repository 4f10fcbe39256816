"""Multi-GPU plumbing: the forward shards by (batch, head) with no exchange.

Every (b, h) head is an independent problem, so N GPUs each run fa_fwd on a
contiguous slice of the B*H heads and nothing crosses GPUs on the data path.
These helpers compute the slice, gather the per-rank outputs when a caller
wants them on every rank, and reduce timings as the max over ranks.  They
use torch.distributed only (NCCL on GPUs, gloo on CPU in the tests).
"""

from __future__ import annotations


def shard_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, end) slice of n items for `rank`; sizes differ by at most 1."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_heads(x, rank: int, world: int):
    """The rank's slice of a [B, H, N, d] (or [B, H, N]) tensor, as [1, h_local, N, ...]."""
    B, H = x.shape[0], x.shape[1]
    s, e = shard_range(B * H, rank, world)
    return x.reshape(B * H, *x.shape[2:])[s:e].unsqueeze(0).contiguous()


def gather_heads(local, B: int, H: int, group=None):
    """All-gather of per-rank head slices back into [B, H, ...] on every rank."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rest = tuple(local.shape[2:])
    sizes = [shard_range(B * H, r, world) for r in range(world)]
    bufs = [torch.empty((1, e - s) + rest, dtype=local.dtype, device=local.device) for s, e in sizes]
    dist.all_gather(bufs, local.contiguous(), group=group)
    return torch.cat(bufs, dim=1).reshape((B, H) + rest)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Max of a per-rank scalar (timings are reported as the slowest rank)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def aggregate_throughput(flops_per_rank_step: float, steps: int, world: int, t_max_ms: float) -> float:
    """Whole-job TFLOPS under weak scaling: every rank does the same work."""
    return world * flops_per_rank_step * steps / (t_max_ms * 1e-3) / 1e12
