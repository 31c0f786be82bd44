"""Out-of-bounds writes through the C ABI.  Every output, in-place buffer and
workspace of a call sits inside a larger allocation whose margins hold a fixed
bit pattern (guard.py).  After the call every margin is unchanged, and the
results equal, bit for bit, those of the same call on plain buffers.  Sizes
are chosen so that no grid divides the work evenly: partial last chunks,
(sequence, head) counts that are not multiples of the persistent grid."""
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
from guard import guarded
from parity import to_dev

pytestmark = pytest.mark.gpu
BF = torch.bfloat16
D = 128


def _done():
    torch.cuda.synchronize()
    assert kda.check_async_status() == 0


@pytest.mark.parametrize("recurrent", [False, True])
@pytest.mark.parametrize("state_dtype", [torch.float32, BF])
def test_prefill_writes_stay_in_bounds(recurrent, state_dtype):
    inp = ki.make_prefill([300, 64, 1, 130], 4, BF, 95, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    N, H, T = 4, 4, int(inp.cu_seqlens[-1])
    init = d["init_state"].to(state_dtype)
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], inp.cu_seqlens, d["cu_dev"])
    want = kda.prefill(*args, init.clone(), d["init_conv"], recurrent=recurrent, state_dtype=state_dtype)
    _done()

    o, o_ok = guarded((T, H, D), torch.float32)
    S, s_ok = guarded((N, H, D, D), state_dtype)
    tail, t_ok = guarded((N, 3, 3, H * D), BF)
    S0, s0_ok = guarded(init.shape, state_dtype, fill=init)
    ws, ws_ok = None, lambda: True
    if not recurrent:
        ws, ws_ok = guarded((kda.workspace_size(N, T, H, 300, BF),), torch.uint8)
    kda.prefill(*args, S0, d["init_conv"], o=o, final_state=S, conv_tail=tail, workspace=ws,
                recurrent=recurrent)
    _done()
    assert o_ok() and s_ok() and t_ok() and s0_ok() and ws_ok()
    assert torch.equal(S0, init)  # the initial state is only read
    assert torch.equal(o, want[0]) and torch.equal(S, want[1]) and torch.equal(tail, want[2])


@pytest.mark.parametrize("state_dtype", [torch.float32, BF])
def test_decode_step_writes_stay_in_bounds(state_dtype):
    inp = ki.make_decode(37, 3, BF, 96)  # 111 (sequence, head) items
    d = {n: getattr(inp, n).cuda() for n in ("state", "conv_cache", "q", "k", "v", "g", "beta", "conv_w")}
    st0 = d["state"].to(state_dtype)
    rows = (d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"])
    ref_state, ref_cache = st0.clone(), d["conv_cache"].clone()
    ref_o = kda.decode_step(ref_state, ref_cache, *rows)
    _done()

    state, s_ok = guarded(st0.shape, state_dtype, fill=st0)
    cache, c_ok = guarded(d["conv_cache"].shape, BF, fill=d["conv_cache"])
    o, o_ok = guarded(d["q"].shape, torch.float32)
    kda.decode_step(state, cache, *rows, o=o)
    _done()
    assert s_ok() and c_ok() and o_ok()
    assert torch.equal(o, ref_o) and torch.equal(state, ref_state) and torch.equal(cache, ref_cache)


@pytest.mark.parametrize("state_dtype", [torch.float32, BF])
def test_multi_token_writes_stay_in_bounds(state_dtype):
    step1 = ki.make_decode_rows(19, 6, 3, BF, 97)  # 57 items; n_accept from 0 to 6
    step2 = ki.make_decode_rows(19, 6, 3, BF, 98)
    d1 = {n: getattr(step1, n).cuda() for n in ("state", "conv_cache", "q", "k", "v", "g", "beta", "conv_w")}
    d2 = {n: getattr(step2, n).cuda() for n in ("q", "k", "v", "g", "beta")}
    na = torch.from_numpy(step1.n_accept).cuda()
    st0, cache0, w = d1["state"].to(state_dtype), d1["conv_cache"], d1["conv_w"]
    rows1 = (d1["q"], d1["k"], d1["v"], d1["g"], d1["beta"], w)
    rows2 = (d2["q"], d2["k"], d2["v"], d2["g"], d2["beta"], w)
    nd = kda.deltas_size(19, 6, 3) // 4

    # plain buffers: verify, commit, then the fused commit + verify of a second step
    ref_state, ref_cache = st0.clone(), cache0.clone()
    ref_o1, ref_dl1 = kda.decode_verify(ref_state, ref_cache, *rows1)
    kda.decode_commit(ref_state, ref_cache, d1["q"], d1["k"], d1["v"], ref_dl1, na)
    fused_state, fused_cache = st0.clone(), cache0.clone()
    ref_o2, ref_dl2 = kda.decode_commit_verify(fused_state, fused_cache, (d1["q"], d1["k"], d1["v"], ref_dl1, na),
                                               *rows2)
    _done()

    # guarded buffers
    state, s_ok = guarded(st0.shape, state_dtype, fill=st0)
    cache, c_ok = guarded(cache0.shape, BF, fill=cache0)
    o1, o1_ok = guarded(d1["q"].shape, torch.float32)
    dl1, dl1_ok = guarded((nd,), torch.float32)
    kda.decode_verify(state, cache, *rows1, o=o1, deltas=dl1)
    _done()
    assert s_ok() and c_ok() and o1_ok() and dl1_ok()
    assert torch.equal(state, st0) and torch.equal(cache, cache0)  # verify changes neither
    assert torch.equal(o1, ref_o1) and torch.equal(dl1, ref_dl1)
    kda.decode_commit(state, cache, d1["q"], d1["k"], d1["v"], dl1, na)
    _done()
    assert s_ok() and c_ok() and dl1_ok()
    assert torch.equal(state, ref_state) and torch.equal(cache, ref_cache)

    state2, s2_ok = guarded(st0.shape, state_dtype, fill=st0)
    cache2, c2_ok = guarded(cache0.shape, BF, fill=cache0)
    o2, o2_ok = guarded(d2["q"].shape, torch.float32)
    dl2, dl2_ok = guarded((nd,), torch.float32)
    kda.decode_commit_verify(state2, cache2, (d1["q"], d1["k"], d1["v"], dl1, na), *rows2, o=o2, deltas=dl2)
    _done()
    assert s2_ok() and c2_ok() and o2_ok() and dl2_ok() and dl1_ok()
    assert torch.equal(o2, ref_o2) and torch.equal(dl2, ref_dl2)
    assert torch.equal(state2, fused_state) and torch.equal(cache2, fused_cache)


def test_state_affine_writes_stay_in_bounds():
    g = torch.Generator().manual_seed(99)
    A = (torch.randn((5, D, D), generator=g) * 0.05).cuda()
    B = torch.randn((5, D, D), generator=g).cuda()
    S_in = torch.randn((5, D, D), generator=g).cuda()
    want = kda.state_affine(A, S_in, B)
    _done()
    out, ok = guarded((5, D, D), torch.float32)
    kda.state_affine(A, S_in, B, S_out=out)
    _done()
    assert ok() and torch.equal(out, want)
