"""GPU parity of the multi-token decode (kda_decode_verify + kda_decode_commit)
through the C ABI: against the fp64 oracle (the recurrence over the kept rows,
from the sequence's state and conv cache), and bit for bit against the same
rows fed one at a time to kda_decode_step."""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
import oracle
from parity import TOL, rel_err

pytestmark = pytest.mark.gpu


def _dev(inp):
    return {n: getattr(inp, n).cuda() for n in ("state", "conv_cache", "q", "k", "v", "g", "beta", "conv_w")}


def _verify_commit(inp, act=0, n_accept=None, o_dtype=torch.float32):
    d = _dev(inp)
    state, cache = d["state"].clone(), d["conv_cache"].clone()
    o, deltas = kda.decode_verify(state, cache, d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], act=act,
                                  o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert torch.equal(state, d["state"]) and torch.equal(cache, d["conv_cache"])  # verify changes neither
    na = torch.from_numpy(inp.n_accept if n_accept is None else n_accept).cuda()
    kda.decode_commit(state, cache, d["q"], d["k"], d["v"], deltas, na)
    torch.cuda.synchronize()
    return o.cpu(), state.cpu(), cache.cpu()


def _single_steps(inp, act=0):
    """Every row through kda_decode_step in turn; returns per-row outputs and
    the (state, cache) after each number of kept rows."""
    d = _dev(inp)
    state, cache = d["state"].clone(), d["conv_cache"].clone()
    outs, snaps = [], [(state.cpu(), cache.cpu())]
    for t in range(inp.num_rows):
        o = kda.decode_step(state, cache, d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                            d["v"][:, t].contiguous(), d["g"][:, t].contiguous(), d["beta"][:, t].contiguous(),
                            d["conv_w"], act=act)
        torch.cuda.synchronize()
        outs.append(o.cpu())
        snaps.append((state.cpu(), cache.cpu()))
    return torch.stack(outs, 1), snaps


@pytest.mark.parametrize("dtype,act", [(torch.bfloat16, 0), (torch.float32, 0), (torch.bfloat16, 1)])
def test_verify_commit_bitwise_equal_to_single_steps(dtype, act):
    inp = ki.make_decode_rows(9, 6, 3, dtype, 41 + act)
    o, S, cache = _verify_commit(inp, act)
    o_ref, snaps = _single_steps(inp, act)
    assert torch.equal(o, o_ref)
    for n, na in enumerate(inp.n_accept):
        S_ref, c_ref = snaps[int(na)]
        assert torch.equal(S[n], S_ref[n]), (n, na)
        assert torch.equal(cache[n], c_ref[n]), (n, na)


def test_mtp_workload_against_oracle():
    """256 sequences x 6 rows (5 drafts + 1) x 64 heads, about four rows kept;
    sampled (sequence, head) pairs against the oracle, every row's output."""
    inp = ki.make_decode_rows(256, 6, 64, torch.bfloat16, ki.BASE_SEED + 5, accept=(2, 6))
    o, S, cache = _verify_commit(inp)
    tol = TOL[torch.bfloat16]
    rng = np.random.default_rng(5)
    pairs = [(int(rng.integers(256)), int(rng.integers(64))) for _ in range(24)] + [(0, 0), (255, 63)]
    D = 128
    cv = cache.view(256, 3, 3, 64, D)
    for n, h in pairs:
        full = oracle.decode_rows_problem(inp, n, h, 6)
        kept = oracle.decode_rows_problem(inp, n, h, int(inp.n_accept[n]))
        oracle.run_problems([full, kept])
        assert rel_err(o[n, :, h].double().numpy(), full.o) <= tol, (n, h)
        assert rel_err(S[n, h].double().numpy(), kept.final_state) <= tol, (n, h)
        for x in range(3):
            assert np.array_equal(cv[n, x, :, h].double().numpy(), kept.tail[x])


def test_fp32_rows_against_oracle_tight():
    inp = ki.make_decode_rows(4, 5, 2, torch.float32, 47)
    o, S, cache = _verify_commit(inp)
    for n in range(4):
        for h in range(2):
            full = oracle.decode_rows_problem(inp, n, h, 5)
            kept = oracle.decode_rows_problem(inp, n, h, int(inp.n_accept[n]))
            oracle.run_problems([full, kept])
            assert rel_err(o[n, :, h].double().numpy(), full.o) <= 1e-4
            assert rel_err(S[n, h].double().numpy(), kept.final_state) <= 1e-4


def test_commit_nothing_and_everything():
    inp = ki.make_decode_rows(5, 8, 2, torch.bfloat16, 43)
    _, snaps = _single_steps(inp)
    for na in (0, 8):
        _, S, cache = _verify_commit(inp, n_accept=np.full(5, na, dtype=np.int32))
        assert torch.equal(S, snaps[na][0]) and torch.equal(cache, snaps[na][1])


def test_single_row_verify_equals_decode_step():
    inp = ki.make_decode_rows(6, 1, 4, torch.bfloat16, 44, accept=(1, 1))
    o, S, cache = _verify_commit(inp)
    o_ref, snaps = _single_steps(inp)
    assert torch.equal(o, o_ref) and torch.equal(S, snaps[1][0]) and torch.equal(cache, snaps[1][1])


def test_bf16_output_is_rounded_fp32_output():
    inp = ki.make_decode_rows(3, 4, 2, torch.bfloat16, 45)
    o32, _, _ = _verify_commit(inp)
    o16, _, _ = _verify_commit(inp, o_dtype=torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_out_of_range_accept_is_clamped_and_reported():
    inp = ki.make_decode_rows(3, 4, 2, torch.bfloat16, 46)
    assert kda.check_async_status() == 0
    _, snaps = _single_steps(inp)
    _, S, cache = _verify_commit(inp, n_accept=np.array([5, -1, 2], dtype=np.int32))
    assert kda.check_async_status() == 1  # KDA_ERR_INVALID_ARG, then cleared
    assert kda.check_async_status() == 0
    assert torch.equal(S[0], snaps[4][0][0]) and torch.equal(S[1], snaps[0][0][1])
    assert torch.equal(S[2], snaps[2][0][2]) and torch.equal(cache[2], snaps[2][1][2])


@pytest.mark.parametrize("state_dtype", [torch.float32, torch.bfloat16])
def test_commit_verify_equals_commit_then_verify(state_dtype):
    """Three speculative steps of 6, 4 and 6 rows (0..R rows kept, so steps
    that keep nothing occur): verify, then commit_verify per later step, equals
    verify / commit / verify / commit / verify bit for bit (outputs of every
    step, deltas, and the state and cache after committing the last step)."""
    steps = [ki.make_decode_rows(9, R, 3, torch.bfloat16, 90 + i, accept=(0, R)) for i, R in enumerate((6, 4, 6))]
    assert any(int(x) == 0 for st in steps for x in st.n_accept)
    first = steps[0]
    rows = [{n: getattr(st, n).cuda() for n in ("q", "k", "v", "g", "beta")} for st in steps]
    accept = [torch.from_numpy(st.n_accept).cuda() for st in steps]
    conv_w = first.conv_w.cuda()

    def fresh():
        return first.state.to(state_dtype).cuda(), first.conv_cache.clone().cuda()

    # separate calls
    S, C = fresh()
    outs_a = []
    for i, r in enumerate(rows):
        o, dl = kda.decode_verify(S, C, r["q"], r["k"], r["v"], r["g"], r["beta"], conv_w)
        kda.decode_commit(S, C, r["q"], r["k"], r["v"], dl, accept[i])
        outs_a.append(o)
    # fused: one pass per step after the first
    S2, C2 = fresh()
    r = rows[0]
    o, dl = kda.decode_verify(S2, C2, r["q"], r["k"], r["v"], r["g"], r["beta"], conv_w)
    outs_b = [o]
    bufs = [dl, torch.empty_like(dl)]
    for i in (1, 2):
        p, r = rows[i - 1], rows[i]
        out_buf = torch.empty(kda.deltas_size(9, r["q"].shape[1], 3) // 4, dtype=torch.float32, device="cuda")
        o, dl_new = kda.decode_commit_verify(S2, C2, (p["q"], p["k"], p["v"], dl, accept[i - 1]), r["q"], r["k"],
                                             r["v"], r["g"], r["beta"], conv_w, deltas=out_buf)
        outs_b.append(o)
        dl = dl_new
    kda.decode_commit(S2, C2, rows[2]["q"], rows[2]["k"], rows[2]["v"], dl, accept[2])
    torch.cuda.synchronize()
    assert kda.check_async_status() == 0
    for a, b in zip(outs_a, outs_b):
        assert torch.equal(a, b)
    assert torch.equal(S, S2) and torch.equal(C, C2)
