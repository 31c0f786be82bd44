"""Multi-rank host logic on CPU with the gloo backend (world size 2): a packed
varlen batch split across ranks by whole sequences gives, gathered, exactly the
single-process result (no exchange between sequences), and the timing reduction
takes the max over ranks."""
import os
import socket

from hypothesis import given, settings
from hypothesis import strategies as st
import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from linear_attention_sequence_kda_b200.sharding import (local_batch, max_over_ranks, split_varlen,
                                                          whole_job_rate)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_split_varlen_balances_and_covers():
    cu = np.cumsum([0, 5, 70, 1, 130, 64, 3, 90])
    for world in (1, 2, 3, 4, 9):
        blocks = split_varlen(cu, world)
        assert len(blocks) == world
        assert blocks[0][0] == 0 and blocks[-1][1] == len(cu) - 1
        for (a, b), (c, d) in zip(blocks, blocks[1:]):
            assert b == c and a <= b
        sizes = [cu[b] - cu[a] for a, b in blocks]
        assert sum(sizes) == cu[-1]
        if world <= 3:
            assert max(sizes) <= cu[-1] / world + 130  # within one segment of balance
    t0, t1, lcu = local_batch(cu, (2, 5))
    assert (t0, t1) == (cu[2], cu[5]) and lcu[0] == 0 and lcu[-1] == t1 - t0
    assert whole_job_rate([100, 300], 2.0) == 200.0


def _worker(rank, world, port, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import kda_inputs as ki
        import oracle
        lens = [5, 70, 1, 130, 64, 3]
        inp = ki.make_prefill(lens, 2, torch.float32, 77, state_std=0.02, conv_history=True)
        block = split_varlen(inp.cu_seqlens, world)[rank]
        t0, t1, lcu = local_batch(inp.cu_seqlens, block)
        s0, s1 = block
        mine = ki.PrefillInputs(inp.q[t0:t1], inp.k[t0:t1], inp.v[t0:t1], inp.g[t0:t1], inp.beta[t0:t1],
                                inp.conv_w, inp.init_state[s0:s1], inp.init_conv[s0:s1], lcu)
        res = oracle.prefill(mine, nthreads=1) if s1 > s0 else {}
        local = {(n + s0, h): (p.o, p.final_state) for (n, h), p in res.items()}
        gathered = [None] * world
        dist.all_gather_object(gathered, local)
        slowest = max_over_ranks(1.0 + rank)
        if rank == 0:
            merged = {}
            for part in gathered:
                merged.update(part)
            full = oracle.prefill(inp, nthreads=1)
            ok = len(merged) == len(full) and all(
                np.array_equal(merged[key][0], p.o) and np.array_equal(merged[key][1], p.final_state)
                for key, p in full.items())
            with open(result_path, "w") as f:
                f.write(f"{int(ok)} {slowest}")
    finally:
        dist.destroy_process_group()


def test_sequence_sharding_over_two_gloo_ranks_matches_single_process(tmp_path):
    path = str(tmp_path / "result.txt")
    mp.start_processes(_worker, args=(2, _free_port(), path), nprocs=2, start_method="spawn", join=True)
    ok, slowest = open(path).read().split()
    assert ok == "1"
    assert float(slowest) == 2.0


@given(st.lists(st.integers(0, 300), min_size=1, max_size=40), st.integers(1, 10))
@settings(max_examples=200, deadline=None)
def test_split_varlen_properties(lengths, world):
    """Any batch (empty segments included) and any rank count: the blocks are
    contiguous and cover every segment once, and block r ends at the first
    segment boundary at or past (r + 1) / world of the tokens."""
    cu = np.cumsum([0] + lengths)
    blocks = split_varlen(cu, world)
    assert len(blocks) == world and blocks[0][0] == 0 and blocks[-1][1] == len(lengths)
    for (a, b), (c, d) in zip(blocks, blocks[1:]):
        assert b == c and a <= b
    total = int(cu[-1])
    for r, (_, end) in enumerate(blocks[:-1]):
        target = total * (r + 1) / world
        assert cu[end] >= target
        assert end == 0 or cu[end - 1] < target
