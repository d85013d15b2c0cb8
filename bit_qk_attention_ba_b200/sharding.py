"""Data-parallel split of one forward over ranks (one process per GPU).

Every (batch, head) unit of the forward is independent given its own Q, K, V
and the bias (shared over the batch), so a job of B batch elements splits into
contiguous batch slices, one per rank, with no exchange on the data path:
each rank runs the whole hot path on its slice, and the outputs, concatenated
in rank order, are the output of the unsplit job.  Splitting along the batch
keeps every head of a batch element on one rank, so the bias, indexed by head,
needs no remapping.
"""
from __future__ import annotations


def shard_range(n_units: int, world: int, rank: int) -> tuple[int, int]:
    """Units [lo, hi) of rank `rank` when n_units are split into `world`
    contiguous slices whose sizes differ by at most one (the first
    n_units % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world or n_units < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, n_units >= 0")
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def batch_slice(x, world: int, rank: int):
    """This rank's contiguous batch slice of a [B, H, N, d] tensor (a view)."""
    lo, hi = shard_range(x.shape[0], world, rank)
    return x[lo:hi]
