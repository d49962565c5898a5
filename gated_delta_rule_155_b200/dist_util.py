"""Host-side multi-GPU plumbing for the KDA path: one process per GPU, no data-path collective.

Heads (b, h) of the gated delta rule are independent (each owns its own state), so
the work shards across ranks with nothing to exchange: a rank processes its own
batch of sequences (weak scaling) or its own slice of a global head list.  The only
communication is control: a barrier around timed regions and a max-reduction of
each rank's device time, so the reported time is the slowest rank's.
"""
from __future__ import annotations


def env():
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 when absent)."""
    import os

    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_range(n_units: int, rank: int, world: int):
    """Contiguous [lo, hi) share of `n_units` for `rank`: sizes differ by at most one and the
    shares of ranks 0..world-1 tile [0, n_units) exactly once."""
    if world < 1 or not (0 <= rank < world) or n_units < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Max of a per-rank scalar (e.g. milliseconds) over all ranks of the default group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, max_ms: float, world: int) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time (units/s)."""
    return world * units_per_rank / (max_ms / 1e3)
