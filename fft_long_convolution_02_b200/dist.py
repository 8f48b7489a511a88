"""Multi-GPU plumbing for the operator (one process per GPU).

Rows (b, c) of the Hyena gated convolution are independent (depthwise
convolution, element-wise gates), so the work shards across ranks with no
exchange on the data path: `channel_shard` gives each rank a contiguous
channel range (its slice of u, the spectrum, D and the short-conv taps), and
the only collectives are host-side bookkeeping: a barrier and a max over
ranks of a timing.  The benchmark runs the per-GPU workload on every rank
(weak scaling); the tests run these helpers as gloo ranks on the CPU.
"""
from __future__ import annotations

import os
from datetime import timedelta


def env_ranks() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0, device=None) -> None:
    """Join the process group when WORLD_SIZE > 1 (MASTER_ADDR/PORT from the env)."""
    import torch.distributed as dist
    world, _, _ = env_ranks()
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if device is not None else {}
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank value (e.g. a time in ms) over all ranks."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def channel_shard(C: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous channel range [c0, c1) of `rank`: sizes differ by at most one,
    the ranges partition [0, C) in rank order."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("need 0 <= rank < world")
    base, extra = divmod(C, world)
    c0 = rank * base + min(rank, extra)
    return c0, c0 + base + (1 if rank < extra else 0)
