"""Instance sharding across GPUs (one process per GPU).

WildCat instances (batch x head) are independent: a batch of BH instances
splits into contiguous shards, one per rank, with no exchange on the data
path.  Each rank calls wildcat_forward on its shard with ``inst0`` = the
shard's first global instance, so its pivot draws -- Philox counter word 1
is the global instance index -- are exactly those of the unsharded batch.
The only collectives are host-side bookkeeping (timing and barriers), which
take whichever torch.distributed backend the caller initialised (NCCL on
GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

from typing import Tuple


def instance_range(BH: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) of the instances rank `rank` of `world` processes; shard
    sizes differ by at most one, lower ranks take the extra instances."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of world {world}")
    if BH < 0:
        raise ValueError("BH must be >= 0")
    base, extra = divmod(BH, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def shard(t, world: int, rank: int):
    """View of this rank's instances of a [BH, ...] tensor, plus inst0."""
    lo, hi = instance_range(t.shape[0], world, rank)
    return t[lo:hi], lo


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the initialised process group
    (the benchmark's time of a multi-GPU step); the value itself when no
    group is initialised."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def forward_shard(Q, K, V, beta: float, r: int, seed: int, eps: float, world: int, rank: int):
    """wildcat_forward on this rank's shard of full [BH, ...] device tensors.
    Returns (O_hat, S, rank, inst0) for the shard's instances."""
    from . import forward

    Qs, lo = shard(Q, world, rank)
    Ks, _ = shard(K, world, rank)
    Vs, _ = shard(V, world, rank)
    O, S, rk = forward(Qs.contiguous(), Ks.contiguous(), Vs.contiguous(), beta, r, seed, eps,
                       inst0=lo)
    return O, S, rk, lo
