"""Context parallelism: one sequence split into contiguous segments over ranks,
joined by the affine state carry (linearity of the hand-over between chunks,
page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit
festem Zustand").  On the CPU, two gloo ranks run the orchestration with the
fp64 oracle standing in for the library: every segment's outputs and the last
rank's final state and conv tail equal the oracle run over the whole sequence.
The same building blocks on the GPU are in test_context_parallel_gpu.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

D = 128


class OracleLib:
    """prefill / state_affine of the library's binding, evaluated by the fp64
    oracle on the CPU (test stand-in).  Record-keeping and scan-only calls
    (`mode`, `workspace`) give what the library gives for them, the prefill of
    their arguments, so the oracle recomputes it; each call is logged, so that
    the driver's use of the modes can be checked."""
    calls = []

    @staticmethod
    def prefill(q, k, v, g, beta, conv_w, cu, init_state=None, init_conv=None, act=0, stream=None, **kw):
        import kda_inputs as ki
        import oracle
        OracleLib.calls.append(kw.get("mode", "full"))
        cu = np.asarray(cu, dtype=np.int32)
        N, (T, H, _) = len(cu) - 1, q.shape
        inp = ki.PrefillInputs(q, k, v, g, beta, conv_w, init_state, init_conv, cu)
        res = oracle.prefill(inp, act=act, nthreads=1)
        o = torch.zeros((T, H, D), dtype=torch.float64)
        S = torch.zeros((N, H, D, D), dtype=torch.float64)
        tail = torch.zeros((N, 3, 3, H * D), dtype=torch.float64)
        for (n, h), p in res.items():
            o[cu[n]:cu[n + 1], h] = torch.from_numpy(p.o)
            S[n, h] = torch.from_numpy(p.final_state)
            for x in range(3):
                tail[n, x, :, h * D:(h + 1) * D] = torch.from_numpy(p.tail[x])
        return o, S, tail

    @staticmethod
    def workspace_size(num_seqs, total_tokens, num_heads, max_seqlen, dtype=None):
        return 16  # a token workspace: the oracle keeps no records

    @staticmethod
    def state_affine(A, S, B, S_out=None, stream=None):
        return A.double() @ S.double() + B.double()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, bounds, result_path, dtype=torch.float32):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import kda_inputs as ki
        from linear_attention_sequence_kda_b200.sharding import context_parallel_prefill
        inp = ki.make_prefill([bounds[-1]], 2, dtype, 93, state_std=0.02, conv_history=True)
        t0, t1 = bounds[rank], bounds[rank + 1]

        def gather(t):
            out = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(out, t.contiguous())
            return out

        o, S, tail = context_parallel_prefill(
            OracleLib, inp.q[t0:t1], inp.k[t0:t1], inp.v[t0:t1], inp.g[t0:t1], inp.beta[t0:t1], inp.conv_w,
            rank, world, gather, init_state=inp.init_state if rank == 0 else None,
            init_conv=inp.init_conv if rank == 0 else None)
        outs = [None] * world
        dist.all_gather_object(outs, (o.numpy(), S.numpy(), tail.numpy()))
        if rank == 0:
            import oracle
            full = oracle.prefill(inp, nthreads=1)
            o_all = np.concatenate([x[0] for x in outs])
            err_o = max(np.abs(o_all[:, h] - full[(0, h)].o).max() for h in range(2))
            err_s = max(np.abs(outs[-1][1][0, h] - full[(0, h)].final_state).max() for h in range(2))
            tail_ok = all(np.array_equal(outs[-1][2][0, x, :, h * D:(h + 1) * D], full[(0, h)].tail[x])
                          for h in range(2) for x in range(3))
            with open(result_path, "w") as f:
                f.write(f"{err_o} {err_s} {int(tail_ok)} {','.join(OracleLib.calls)}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("bounds", [[0, 150, 280], [0, 70, 73, 230]])
def test_segments_over_gloo_equal_the_whole_sequence(tmp_path, bounds, dtype):
    """Two segments of 150 and 130 tokens (partial chunks at both ends of the
    boundary); three segments whose middle one has the minimum of 3 tokens, so
    that the last segment's conv history is that segment alone.  Nonzero
    initial state and conv history.  With bf16 inputs the driver prepares each
    segment's records once: one record-keeping call, then two scans."""
    path = str(tmp_path / "cp.txt")
    world = len(bounds) - 1
    mp.start_processes(_worker, args=(world, _free_port(), bounds, path, dtype), nprocs=world,
                       start_method="spawn", join=True)
    err_o, err_s, tail_ok, calls = open(path).read().split()
    assert float(err_o) < 1e-9 and float(err_s) < 1e-9 and tail_ok == "1"
    assert calls == ("records,scan,scan" if dtype == torch.bfloat16 else "full,full")


def test_conv_halo_needs_three_tokens():
    """A segment followed by another must hand over three raw tokens."""
    from linear_attention_sequence_kda_b200.sharding import conv_halo
    x = torch.zeros((2, 1, D))
    with pytest.raises(ValueError):
        conv_halo(x, x, x)
    halo = conv_halo(*(torch.arange(3 * D, dtype=torch.float32).view(3, 1, D) + 1000 * i for i in range(3)))
    assert halo.shape == (1, 3, 3, D) and halo[0, 2, 0, 0] == 2000 and halo[0, 0, 2, D - 1] == 3 * D - 1


def test_compose_order():
    """compose_initial_state applies the earlier segments first: S <- A_j S + B_j, j ascending."""
    from linear_attention_sequence_kda_b200.sharding import compose_initial_state
    r = np.random.default_rng(4)
    As = [torch.from_numpy(r.standard_normal((2, 3, 3))) for _ in range(3)]
    Bs = [torch.from_numpy(r.standard_normal((2, 3, 3))) for _ in range(3)]
    S0 = torch.from_numpy(r.standard_normal((2, 3, 3)))
    got = compose_initial_state(S0, As, Bs, 3, lambda A, S, B: A @ S + B)
    want = As[2] @ (As[1] @ (As[0] @ S0 + Bs[0]) + Bs[1]) + Bs[2]
    assert torch.allclose(got, want) and torch.equal(compose_initial_state(S0, As, Bs, 0, None), S0)
