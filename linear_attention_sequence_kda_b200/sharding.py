"""Host-side multi-GPU helpers.

The KDA mixing step has no exchange between sequences or heads (each
(sequence, head) state evolves on its own), so a batch spreads over GPUs by
handing each rank a contiguous block of whole sequences, or each rank its own
heads: no collective is needed on the data path.  Ranks only meet for timing (a
barrier and the max of the per-rank device times).

One long sequence split into contiguous segments, one per rank (context
parallelism), has one exchange step: the state handed from segment to segment.
Page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit
festem Zustand": the state is handed from chunk to chunk, and the hand-over is
linear in the state, so segment r maps its initial state as
S_out = A_r S_in + B_r.  context_parallel_prefill runs, on every rank:
  1. the conv halo: each rank's last three raw tokens, gathered, give the next
     rank its conv history;
  2. the carry: the segment entered from S = 0 (final state B_r) and from
     S = I with v = 0 (final state A_r).  On the chunked (bf16) path the chunk
     records, which depend on q, k, g and beta only, are prepared once: a
     record-keeping prefill gives B_r and two scans over the same records give
     A_r and, in step 5, the outputs.  On the fp32 path one prefill call runs
     the segment twice;
  3. the exchange: all ranks gather every (A_j, B_j);
  4. the composition S_in(r) = A_{r-1}(... (A_0 S_0 + B_0) ...) + B_{r-1};
  5. the segment's prefill from S_in(r): its outputs, and on the last rank the
     sequence's final state and conv tail.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

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


def conv_halo(q, k, v):
    """[1, 3 (q, k, v), 3 (time, oldest first), H * D]: the segment's last three
    raw tokens, the conv history of the segment after it (needs >= 3 tokens)."""
    if q.shape[0] < 3:
        raise ValueError("every segment but the last needs at least 3 tokens")
    import torch
    return torch.stack([x[-3:].reshape(3, -1) for x in (q, k, v)])[None].contiguous()


def compose_initial_state(S0, As, Bs, rank: int, affine: Callable):
    """S_in of segment `rank`: S0 carried through segments 0 .. rank - 1 by
    S <- A_j S + B_j (affine(A, S, B) computes one step)."""
    S = S0
    for j in range(rank):
        S = affine(As[j], S, Bs[j])
    return S


def segment_workspace(lib, q):
    """A workspace for the segment's chunk records (None where the call
    needs none: fp32 inputs)."""
    import torch
    T, H, _ = q.shape
    if q.dtype != torch.bfloat16:
        return None
    need = lib.workspace_size(1, T, H, T)
    return torch.empty(max(need, 16), dtype=torch.uint8, device=q.device) if need > 0 else None


def segment_carry(lib, q, k, v, g, beta, conv_w, prev_tail, act: int = 0, stream=None, workspace=None):
    """(A, B) of one segment, [1, H, D, D] fp32 each: the segment entered from
    S = 0 with the real inputs (final state B) and from S = I with v = 0 and a
    zero v history (final state A).  With a `workspace` (bf16 inputs) the chunk
    records are prepared once (a record-keeping prefill gives B, a scan over
    the same records A) and stay in `workspace` for the segment's final scan;
    otherwise one prefill call runs the segment twice."""
    import torch
    T, H, D = q.shape
    if workspace is not None:
        cu = np.array([0, T], dtype=np.int32)
        zero = torch.zeros((1, H, D, D), dtype=torch.float32, device=q.device)
        eye = torch.eye(D, dtype=torch.float32, device=q.device).expand(1, H, D, D).contiguous()
        hist0 = prev_tail.clone()
        hist0[:, 2] = 0
        _, B, _ = lib.prefill(q, k, v, g, beta, conv_w, cu, init_state=zero, init_conv=prev_tail, act=act,
                              stream=stream, workspace=workspace, mode="records")
        _, A, _ = lib.prefill(q, k, torch.zeros_like(v), g, beta, conv_w, cu, init_state=eye, init_conv=hist0,
                              act=act, stream=stream, workspace=workspace, mode="scan")
        return A, B
    two = lambda x, y=None: torch.cat([x, x if y is None else y]).contiguous()  # noqa: E731
    init = torch.zeros((2, H, D, D), dtype=torch.float32, device=q.device)
    init[1] = torch.eye(D, dtype=torch.float32, device=q.device)
    hist0 = prev_tail.clone()
    hist0[:, 2] = 0
    cu = np.array([0, T, 2 * T], dtype=np.int32)
    _, final, _ = lib.prefill(two(q), two(k), two(v, torch.zeros_like(v)), two(g), two(beta), conv_w, cu,
                              init_state=init, init_conv=torch.cat([prev_tail, hist0]).contiguous(), act=act,
                              stream=stream)
    return final[1:2].contiguous(), final[0:1].contiguous()


def context_parallel_prefill(lib, q, k, v, g, beta, conv_w, rank: int, world: int,
                             all_gather: Callable, init_state=None, init_conv=None, act: int = 0,
                             stream=None, o_dtype=None):
    """Prefill of segment `rank` of one sequence split over `world` ranks.
      q, k, v, g : [T_r, H, 128] this rank's tokens; beta [T_r, H].
      init_state : [1, H, 128, 128] the sequence's initial state (rank 0; None = 0).
      init_conv  : [1, 3, 3, H * 128] the sequence's conv history (rank 0; None = 0).
      all_gather : t -> list of every rank's t, in rank order (a collective).
      lib        : the library binding (prefill, state_affine).
    Returns (o, final_state, conv_tail) of this segment; on the last rank the
    final state and conv tail are those of the whole sequence."""
    import torch
    T, H, D = q.shape
    if T >= 3:
        halo = conv_halo(q, k, v)
    elif rank == world - 1:  # nobody reads the last segment's halo
        halo = torch.zeros((1, 3, 3, H * D), dtype=q.dtype, device=q.device)
    else:
        raise ValueError("every segment but the last needs at least 3 tokens")
    halos = all_gather(halo)
    if rank > 0:
        prev_tail = halos[rank - 1]
    elif init_conv is not None:
        prev_tail = init_conv
    else:
        prev_tail = torch.zeros((1, 3, 3, H * D), dtype=q.dtype, device=q.device)
    ws = segment_workspace(lib, q)
    A, B = segment_carry(lib, q, k, v, g, beta, conv_w, prev_tail, act, stream, workspace=ws)
    As, Bs = all_gather(A), all_gather(B)
    S0 = init_state if init_state is not None else torch.zeros((1, H, D, D), dtype=torch.float32, device=q.device)
    S_in = compose_initial_state(S0, As, Bs, rank, lib.state_affine)
    kw = {} if o_dtype is None else {"o_dtype": o_dtype}
    if ws is not None:  # the segment's records are in ws: its scan alone
        kw.update(workspace=ws, mode="scan")
    return lib.prefill(q, k, v, g, beta, conv_w, np.array([0, T], dtype=np.int32), init_state=S_in,
                       init_conv=prev_tail, act=act, stream=stream, **kw)
