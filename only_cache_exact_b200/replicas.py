"""Host logic for running the decode step as independent replicas, one process per GPU.

Every sequence attends only over its own K cache (Slim Attention article,
section "K-Cache is All You Need": the generation step reads q, the sequence's
cached K and W_KV), so N ranks run N disjoint batches with no collective on the
data path. The only collectives are the ones that time the job: a barrier
before the timed region and a max over ranks of its duration. Work per rank is
fixed as N grows (weak scaling): every rank keeps the same batch size and
length mix and draws its own token rows.
"""
from __future__ import annotations

from typing import Iterable


def global_sequence_ids(rank: int, world: int, batch: int) -> list[int]:
    """Global ids of the `batch` sequences rank `rank` owns: a contiguous, disjoint block."""
    if not (0 <= rank < world) or batch < 0:
        raise ValueError(f"bad rank/world/batch {rank}/{world}/{batch}")
    return list(range(rank * batch, (rank + 1) * batch))


def max_over_ranks(value: float, pg=None, device=None) -> float:
    """Largest `value` over all ranks of the default process group (identity without one).

    Every rank must call it at the same point: it is a collective.
    """
    if pg is None:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, elapsed_ms: float) -> float:
    """Units per second processed by the whole job: all ranks' units over the slowest rank's time."""
    if elapsed_ms <= 0:
        raise ValueError("elapsed time must be positive")
    return units_per_rank * world * 1e3 / elapsed_ms


def check_disjoint(blocks: Iterable[Iterable[int]]) -> bool:
    """True when no sequence id appears in two ranks' blocks."""
    seen: set[int] = set()
    for blk in blocks:
        for g in blk:
            if g in seen:
                return False
            seen.add(g)
    return True
