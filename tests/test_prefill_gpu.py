"""GPU parity of kda_prefill / kda_prefill_recurrent against the fp64 oracle,
through the C ABI, on the five workloads' inputs and on edge cases."""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
import oracle
from parity import TOL, compare_prefill, rel_err, run_prefill, sample_pairs, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("recurrent", [False, True])
def test_workload0_tiny_fp32(recurrent):
    inp = ki.workload(0)
    eo, es = compare_prefill(inp, run_prefill(inp, recurrent=recurrent))
    assert eo <= 1e-4 and es <= 1e-4


def test_workload1_prefill_bf16_full_size():
    """4 x 4096 tokens, 64 heads: every (sequence, head) pair, o and final
    state element by element against the oracle."""
    inp = ki.workload(1)
    compare_prefill(inp, run_prefill(inp))


def test_workload2_long_context_full_size():
    """1 x 65,536 tokens, 64 heads: every head."""
    inp = ki.workload(2)
    compare_prefill(inp, run_prefill(inp))


def test_workload3_varlen_full_size():
    """16 packed segments (about 267k tokens), 64 heads: all 1,024 pairs."""
    inp = ki.workload(3)
    assert inp.num_seqs == 16
    compare_prefill(inp, run_prefill(inp), batch=16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("recurrent", [False, True])
def test_edge_lengths(dtype, recurrent):
    """Ragged lengths around the chunk size, segments shorter than the conv
    window, an empty segment, conv history and initial states."""
    lens = [1, 2, 3, 0, 63, 64, 65, 127, 130]
    inp = ki.make_prefill(lens, 2, dtype, 7, state_std=0.02, conv_history=True)
    compare_prefill(inp, run_prefill(inp, recurrent=recurrent))


@pytest.mark.parametrize("act", [0, 1])
def test_single_head_no_history_and_silu(act):
    inp = ki.make_prefill([200], 1, torch.bfloat16, 8)
    compare_prefill(inp, run_prefill(inp, act=act), act=act)


def test_gate_floor_and_beta_extremes():
    inp = ki.make_prefill([150, 70], 2, torch.bfloat16, 9, state_std=0.02, conv_history=True)
    inp.g[:, 0] = -5.0          # head 0: every channel at the floor
    inp.g[:40, 1, :64] = -7.0   # below the floor -> clamped
    inp.beta[:, 0] = 1.0
    inp.beta[100:, 1] = 0.0
    compare_prefill(inp, run_prefill(inp))


def test_bf16_output_is_rounded_fp32_output():
    """o_dt = bf16 gives exactly the fp32 result rounded to bf16."""
    inp = ki.make_prefill([130, 7], 2, torch.bfloat16, 15, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    o32 = run_prefill(inp, dev_inputs=d)[0]
    o16 = run_prefill(inp, dev_inputs=d, o_dtype=torch.bfloat16)[0]
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_all_segments_empty():
    inp = ki.make_prefill([0, 0], 2, torch.bfloat16, 10, state_std=0.02, conv_history=True)
    o, S, tail = run_prefill(inp)
    assert torch.equal(S.cpu(), inp.init_state)
    assert torch.equal(tail.cpu(), inp.init_conv)


def test_varlen_packed_equals_separate_calls_bitwise():
    lens = [70, 5, 129]
    inp = ki.make_prefill(lens, 2, torch.bfloat16, 11, state_std=0.02, conv_history=True)
    o, S, tail = [x.cpu() for x in run_prefill(inp)]
    for n, L in enumerate(lens):
        s0 = int(inp.cu_seqlens[n])
        one = ki.PrefillInputs(inp.q[s0:s0 + L], inp.k[s0:s0 + L], inp.v[s0:s0 + L], inp.g[s0:s0 + L],
                               inp.beta[s0:s0 + L], inp.conv_w, inp.init_state[n:n + 1],
                               inp.init_conv[n:n + 1], np.array([0, L], dtype=np.int32))
        o1, S1, t1 = [x.cpu() for x in run_prefill(one)]
        assert torch.equal(o1, o[s0:s0 + L]) and torch.equal(S1[0], S[n]) and torch.equal(t1[0], tail[n])


def test_split_and_decode_equivalence():
    """prefill(T) vs prefill(a) + prefill(T-a) carrying (state, tail) vs T
    decode steps, all on the GPU, each compared with the oracle's o."""
    T, a = 150, 67
    inp = ki.make_prefill([T], 2, torch.bfloat16, 12, state_std=0.02, conv_history=True)
    ref = oracle.prefill(inp)
    o_full, S_full, _ = run_prefill(inp)
    first = ki.PrefillInputs(inp.q[:a], inp.k[:a], inp.v[:a], inp.g[:a], inp.beta[:a], inp.conv_w,
                             inp.init_state, inp.init_conv, np.array([0, a], dtype=np.int32))
    o1, S1, t1 = run_prefill(first)
    second = ki.PrefillInputs(inp.q[a:], inp.k[a:], inp.v[a:], inp.g[a:], inp.beta[a:], inp.conv_w,
                              S1.cpu(), t1.cpu(), np.array([0, T - a], dtype=np.int32))
    o2, S2, _ = run_prefill(second)
    o_split = torch.cat([o1, o2]).cpu()
    # decode chain
    state = inp.init_state.clone().cuda()
    cache = inp.init_conv.clone().cuda()
    d = to_dev(inp)
    outs = []
    for t in range(T):
        outs.append(kda.decode_step(state, cache, d["q"][t:t + 1], d["k"][t:t + 1], d["v"][t:t + 1],
                                    d["g"][t:t + 1], d["beta"][t:t + 1], d["conv_w"]))
    o_dec = torch.cat(outs).cpu()
    for h in range(2):
        r = ref[(0, h)]
        for got in (o_full.cpu(), o_split, o_dec):
            assert rel_err(got[:, h].double().numpy(), r.o) <= TOL[torch.bfloat16]
        for st in (S_full, S2, state):
            assert rel_err(st.cpu()[0, h].double().numpy(), r.final_state) <= TOL[torch.bfloat16]


def test_determinism_and_in_place():
    inp = ki.make_prefill([300, 64], 3, torch.bfloat16, 13, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    a = [x.clone() for x in run_prefill(inp, dev_inputs=d)]
    b = [x.clone() for x in run_prefill(inp, dev_inputs=d)]
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    # final_state written over init_state, conv tail over init_conv
    st, cv = d["init_state"].clone(), d["init_conv"].clone()
    o, S, tail = kda.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], inp.cu_seqlens,
                             d["cu_dev"], st, cv, final_state=st, conv_tail=cv)
    torch.cuda.synchronize()
    assert torch.equal(st, a[1]) and torch.equal(cv, a[2]) and torch.equal(o, a[0])


def test_causality():
    inp = ki.make_prefill([200], 2, torch.bfloat16, 14)
    o1 = run_prefill(inp)[0].cpu()
    t0 = 130
    inp.q[t0] += 1
    inp.k[t0] -= 1
    inp.v[t0] += 2
    o2 = run_prefill(inp)[0].cpu()
    assert torch.equal(o1[:t0], o2[:t0])
    assert not torch.equal(o1[t0], o2[t0])


@pytest.mark.parametrize("heads", [96, 97])
def test_overlap_threshold_both_schedules(heads):
    """One sequence with 96 heads takes the overlapped schedule (the scan runs
    beside the prep and waits for each chunk's record), 97 heads the one after
    the other; both against the oracle on sampled heads, and both equal to the
    same heads run in a call of their own (4 heads, always overlapped): the
    schedule changes when records are read, never what is computed."""
    inp = ki.make_prefill([700], heads, torch.bfloat16, 91, state_std=0.02, conv_history=True)
    o, S, tail = run_prefill(inp)
    compare_prefill(inp, (o, S, tail), [(0, 0), (0, 45), (0, heads - 1)])
    sub = ki.make_prefill([700], 4, torch.bfloat16, 91, state_std=0.02, conv_history=True)
    hs = [0, 1, 2, 3]
    # the same inputs restricted to heads 0..3 (inputs are drawn per tensor, so slice them)
    D = 128
    pick = lambda t: t.view(t.shape[0], heads, -1)[:, hs].reshape(t.shape[0], 4, *t.shape[2:]).contiguous()  # noqa: E731
    sub.q, sub.k, sub.v, sub.g = pick(inp.q), pick(inp.k), pick(inp.v), pick(inp.g)
    sub.beta = inp.beta[:, hs].contiguous()
    sub.conv_w = inp.conv_w.view(3, heads, D, 4)[:, hs].reshape(3, 4 * D, 4).contiguous()
    sub.init_state = inp.init_state[:, hs].contiguous()
    sub.init_conv = inp.init_conv.view(1, 3, 3, heads, D)[:, :, :, hs].reshape(1, 3, 3, 4 * D).contiguous()
    o4, S4, _ = run_prefill(sub)
    assert torch.equal(o4, o[:, hs]) and torch.equal(S4, S[:, hs])
