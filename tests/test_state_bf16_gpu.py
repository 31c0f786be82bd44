"""GPU parity of bf16 state storage (state_dt = KDA_BF16) through the C ABI.

All state arithmetic stays fp32; a bf16 state is rounded (nearest, ties to
even) where it is stored.  Checked here:
  * bit for bit: a call on a bf16 state equals the same call on an fp32 state
    holding the same values, with the stored state equal to the fp32 result
    rounded once (decode step, chunked and recurrent prefill);
  * bit for bit: verify / commit equal chained single steps on a bf16 state;
  * against the fp64 oracle whose state is rounded to bf16 at the same storage
    points (after every decode step / kept row, at the end of a prefill)."""
import dataclasses

import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
import oracle
from parity import TOL, rel_err, run_prefill, to_dev

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _state_close(got, ref):
    """A stored bf16 state against the oracle's: the GPU rounds an fp32 result
    and the oracle an exact one, so an element whose exact value lies near a
    rounding boundary may land on the neighbouring bf16 value (one ulp, at most
    2^-7 of the value), and such a difference can spread a little through
    later steps.  Every element within 2^-7 of its value (plus 2^-12 of the
    rms for elements near zero); returns the fraction that is exactly equal."""
    err = np.abs(got - ref)
    rms = float(np.sqrt((ref ** 2).mean()))
    assert np.all(err <= 2.0 ** -7 * np.abs(ref) + 2.0 ** -12 * rms), float((err / (np.abs(ref) + rms)).max())
    return float((err == 0).mean())


def _bf16_state(inp):
    """The same inputs with the state stored in bf16 (the values both sides use)."""
    return dataclasses.replace(inp, state=inp.state.to(BF))


def _decode(inp, state_dtype, act=0):
    state = inp.state.to(state_dtype).cuda()
    cache = inp.conv_cache.clone().cuda()
    o = kda.decode_step(state, cache, inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.g.cuda(), inp.beta.cuda(),
                        inp.conv_w.cuda(), act=act)
    torch.cuda.synchronize()
    return o.cpu(), state.cpu(), cache.cpu()


@pytest.mark.parametrize("dtype,act", [(BF, 0), (torch.float32, 0), (BF, 1)])
def test_decode_bf16_state_is_fp32_step_rounded_once(dtype, act):
    inp = _bf16_state(ki.make_decode(7, 3, dtype, 81 + act))
    o16, s16, c16 = _decode(inp, BF, act)
    o32, s32, c32 = _decode(inp, torch.float32, act)  # fp32 storage of the same (bf16) values
    assert torch.equal(o16, o32) and torch.equal(c16, c32)
    assert torch.equal(s16, s32.to(BF))


def test_decode_bf16_state_full_size_against_oracle():
    """256 sequences x 64 heads (the decode workload's shape) with a bf16 state."""
    inp = _bf16_state(ki.make_decode(256, 64, BF, ki.BASE_SEED + 4))
    o, S, cache = _decode(inp, BF)
    ref = oracle.decode(inp, state_round=oracle.STATE_BF16_AT_END)
    cv = cache.view(256, 3, 3, 64, 128)
    equal = []
    for (n, h), p in ref.items():
        assert rel_err(o[n, h].double().numpy(), p.o[0]) <= TOL[BF], (n, h)
        equal.append(_state_close(S[n, h].double().numpy(), p.final_state))
        if (n * 64 + h) % 97 == 0:
            for x in range(3):
                assert np.array_equal(cv[n, x, :, h].double().numpy(), p.tail[x])
    assert np.mean(equal) > 0.99


def test_chained_decode_steps_bf16_state_against_oracle():
    """Eight single-token steps carrying a bf16 state and the conv cache equal
    the oracle that rounds the state after every step."""
    inp = _bf16_state(ki.make_decode_rows(4, 8, 2, BF, 83, accept=(8, 8)))
    state = inp.state.cuda()
    cache = inp.conv_cache.clone().cuda()
    outs = []
    for t in range(8):
        outs.append(kda.decode_step(state, cache, inp.q[:, t].contiguous().cuda(), inp.k[:, t].contiguous().cuda(),
                                    inp.v[:, t].contiguous().cuda(), inp.g[:, t].contiguous().cuda(),
                                    inp.beta[:, t].contiguous().cuda(), inp.conv_w.cuda()).cpu())
    torch.cuda.synchronize()
    o = torch.stack(outs, 1)
    for n in range(4):
        for h in range(2):
            p = oracle.decode_rows_problem(inp, n, h, 8, state_round=oracle.STATE_BF16_EACH_TOKEN)
            oracle.run_problems([p], 1)
            assert rel_err(o[n, :, h].double().numpy(), p.o) <= TOL[BF], (n, h)
            _state_close(state[n, h].cpu().double().numpy(), p.final_state)


def _verify_commit(inp, n_accept=None):
    d = {n: getattr(inp, n).cuda() for n in ("state", "conv_cache", "q", "k", "v", "g", "beta", "conv_w")}
    state, cache = d["state"].clone(), d["conv_cache"].clone()
    o, deltas = kda.decode_verify(state, cache, d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"])
    torch.cuda.synchronize()
    assert torch.equal(state, d["state"]) and torch.equal(cache, d["conv_cache"])
    na = torch.from_numpy(inp.n_accept if n_accept is None else n_accept).cuda()
    kda.decode_commit(state, cache, d["q"], d["k"], d["v"], deltas, na)
    torch.cuda.synchronize()
    assert kda.check_async_status() == 0
    return o.cpu(), state.cpu(), cache.cpu()


def test_verify_commit_bf16_state_bitwise_equal_to_single_steps():
    inp = _bf16_state(ki.make_decode_rows(9, 6, 3, BF, 84))
    o, S, cache = _verify_commit(inp)
    state = inp.state.cuda()
    c = inp.conv_cache.clone().cuda()
    snaps, outs = [(state.cpu(), c.cpu())], []
    for t in range(6):
        outs.append(kda.decode_step(state, c, inp.q[:, t].contiguous().cuda(), inp.k[:, t].contiguous().cuda(),
                                    inp.v[:, t].contiguous().cuda(), inp.g[:, t].contiguous().cuda(),
                                    inp.beta[:, t].contiguous().cuda(), inp.conv_w.cuda()).cpu())
        torch.cuda.synchronize()
        snaps.append((state.cpu(), c.cpu()))
    assert torch.equal(o, torch.stack(outs, 1))
    for n, na in enumerate(inp.n_accept):
        assert torch.equal(S[n], snaps[int(na)][0][n]) and torch.equal(cache[n], snaps[int(na)][1][n]), (n, na)


def test_mtp_bf16_state_against_oracle():
    """256 sequences x 6 rows x 64 heads with about four rows kept: sampled
    (sequence, head) pairs against the oracle rounding after every row."""
    inp = _bf16_state(ki.make_decode_rows(256, 6, 64, BF, ki.BASE_SEED + 6, accept=(2, 6)))
    o, S, cache = _verify_commit(inp)
    rng = np.random.default_rng(6)
    pairs = [(int(rng.integers(256)), int(rng.integers(64))) for _ in range(16)] + [(0, 0), (255, 63)]
    for n, h in pairs:
        full = oracle.decode_rows_problem(inp, n, h, 6, state_round=oracle.STATE_BF16_EACH_TOKEN)
        kept = oracle.decode_rows_problem(inp, n, h, int(inp.n_accept[n]), state_round=oracle.STATE_BF16_EACH_TOKEN)
        oracle.run_problems([full, kept])
        assert rel_err(o[n, :, h].double().numpy(), full.o) <= TOL[BF], (n, h)
        _state_close(S[n, h].double().numpy(), kept.final_state)


@pytest.mark.parametrize("recurrent", [False, True])
def test_prefill_bf16_state(recurrent):
    """Varlen prefill (partial last chunks, conv history) on a bf16 initial
    state: bit for bit the fp32-state call rounded once at the end, and the
    oracle rounding its final state once."""
    inp = ki.make_prefill([300, 64, 1, 130], 4, BF, 85, state_std=0.02, conv_history=True)
    inp = dataclasses.replace(inp, init_state=inp.init_state.to(BF))
    d = to_dev(inp)
    o16, s16, t16 = run_prefill(inp, recurrent=recurrent, dev_inputs=d)
    d32 = dict(d, init_state=d["init_state"].float())
    o32, s32, t32 = run_prefill(inp, recurrent=recurrent, dev_inputs=d32)
    assert s16.dtype == BF and s32.dtype == torch.float32
    assert torch.equal(o16, o32) and torch.equal(t16, t32) and torch.equal(s16, s32.to(BF))
    ref = oracle.prefill(inp, state_round=oracle.STATE_BF16_AT_END)
    o, S = o16.cpu(), s16.cpu()
    for (n, h), p in ref.items():
        s0, s1 = int(inp.cu_seqlens[n]), int(inp.cu_seqlens[n + 1])
        assert rel_err(o[s0:s1, h].double().numpy(), p.o) <= TOL[BF], (n, h)
        # the fp32-state bar plus one bf16 ulp: rounding the GPU's fp32 state and
        # rounding the exact one may land on neighbouring bf16 values, and one
        # ulp (at most 2^-7 relative) of the largest elements is already a few
        # percent of the state's rms
        got, want = S[n, h].double().numpy(), p.final_state
        rms = float(np.sqrt((want ** 2).mean()))
        assert np.all(np.abs(got - want) <= TOL[BF] * rms + 2.0 ** -7 * np.abs(want)), (n, h)
