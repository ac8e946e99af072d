"""Sharding verify work over ranks (one process per GPU).

Verify is independent per sequence, so a batch splits over ranks with no
collective on the data path: rank r verifies sequences [b0, b1) and passes
``seq_offset = b0`` so that its Philox draws are those of the unsharded call.
Collectives are only for bookkeeping: gathering the per-rank results and
taking the slowest rank's time.
"""
from __future__ import annotations


def shard(B: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced range of sequences [b0, b1) owned by `rank`."""
    if world < 1 or not 0 <= rank < world or B < 0:
        raise ValueError(f"bad shard request B={B} rank={rank} world={world}")
    base, extra = divmod(B, world)
    b0 = rank * base + min(rank, extra)
    return b0, b0 + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, group=None) -> float:
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def gather_rows(local, B: int, group=None):
    """All-gather per-rank row blocks (first axis = this rank's shard of B)
    into the full [B, ...] tensor on every rank."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    sizes = [shard(B, r, world)[1] - shard(B, r, world)[0] for r in range(world)]
    width = max(sizes)
    pad = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[: local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:n] for p, n in zip(parts, sizes)], dim=0)
