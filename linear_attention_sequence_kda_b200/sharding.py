"""Host-side multi-GPU helpers.

The KDA mixing step has no exchange between sequences or heads (each
(sequence, head) state evolves on its own), so a batch spreads over GPUs by
handing each rank a contiguous block of whole sequences: no collective is needed
on the data path.  Ranks only meet for timing (a barrier and the max of the
per-rank device times).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def split_varlen(cu_seqlens: Sequence[int], world: int) -> List[Tuple[int, int]]:
    """Contiguous split of the segments of a packed batch into `world` blocks
    [s_begin, s_end) with balanced token counts (greedy on the prefix sums:
    block r ends at the first segment boundary at or past (r+1)/world of the
    tokens).  Blocks may be empty when there are fewer segments than ranks."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    n = len(cu) - 1
    total = int(cu[-1])
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        s = int(np.searchsorted(cu, target, side="left"))
        s = min(max(s, bounds[-1]), n)
        bounds.append(s)
    bounds.append(n)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def local_batch(cu_seqlens: Sequence[int], block: Tuple[int, int]):
    """(token_begin, token_end, local cu_seqlens) of one rank's block; the
    rank's inputs are rows [token_begin, token_end) of the packed tensors and
    its states / conv tails are entries [s_begin, s_end)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    s0, s1 = block
    t0, t1 = int(cu[s0]), int(cu[s1])
    return t0, t1, (cu[s0:s1 + 1] - t0).astype(np.int32)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the default process group (identity when
    torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: Sequence[int], max_seconds: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return float(sum(units_per_rank)) / max_seconds
