"""Multi-process helpers for running the recurrence on several GPUs.

Every (batch row, head) pair evolves on its own, so a batch shards across
ranks by rows with no exchange of data; the only cross-rank operations are
timing reductions.  One process per GPU, launched by torchrun.
"""

from __future__ import annotations

from typing import Tuple

import torch


def shard_rows(B: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [lo, hi) slice of B batch rows for `rank` of `world`; sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world or B < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(B, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's own synthetic batch (weak scaling: every rank draws its own rows)."""
    return int(base_seed) + 7919 * int(rank)


def max_over_ranks(x: float, group=None) -> float:
    """Maximum of a per-rank float (e.g. elapsed milliseconds) over the process group."""
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend(group) == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
