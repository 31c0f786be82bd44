"""Context parallelism on the GPU, emulated on one device: one sequence split
into 4 contiguous segments, each taken through the steps a rank takes
(conv halo, the segment's affine carry (A, B) from one prefill call,
composition of its initial state with kda_state_affine, its prefill), equals
one prefill call over the whole sequence and the oracle."""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
import oracle
from linear_attention_sequence_kda_b200.sharding import (compose_initial_state, conv_halo, segment_carry,
                                                         segment_workspace)
from parity import TOL, rel_err, run_prefill, to_dev

pytestmark = pytest.mark.gpu


def test_state_affine_matches_fp64_product():
    r = np.random.default_rng(8)
    A = torch.from_numpy(r.standard_normal((5, 128, 128)) * 0.1).float()
    S = torch.from_numpy(r.standard_normal((5, 128, 128)) * 0.02).float()
    B = torch.from_numpy(r.standard_normal((5, 128, 128)) * 0.02).float()
    want = A.double() @ S.double() + B.double()
    got = kda.state_affine(A.cuda(), S.cuda(), B.cuda()).cpu()
    assert (got.double() - want).abs().max() <= 1e-5 * want.abs().max()
    Sd = S.cuda()
    kda.state_affine(A.cuda(), Sd, B.cuda(), S_out=Sd)  # in place
    assert torch.equal(Sd.cpu(), got)
    S16 = S.to(torch.bfloat16).cuda()
    got16 = kda.state_affine(A.cuda(), S16, B.cuda()).cpu()
    assert got16.dtype == torch.bfloat16
    want16 = A.double() @ S.to(torch.bfloat16).double() + B.double()
    assert ((got16.double() - want16).abs() <= 2.0 ** -7 * want16.abs() + 1e-6).all()


@pytest.mark.parametrize("dtype,records", [(torch.bfloat16, False), (torch.bfloat16, True), (torch.float32, False)])
def test_four_segments_equal_one_call(dtype, records):
    bounds = [0, 700, 1100, 1950, 2300]  # segments of 700, 400, 850, 350 tokens
    H = 4
    inp = ki.make_prefill([bounds[-1]], H, dtype, 95, state_std=0.02, conv_history=True)
    dev = {n: getattr(inp, n).cuda() for n in ("q", "k", "v", "g", "beta", "conv_w", "init_state", "init_conv")}
    whole_o, whole_S, whole_tail = run_prefill(inp)
    seg = [{n: dev[n][t0:t1].contiguous() for n in ("q", "k", "v", "g", "beta")}
           for t0, t1 in zip(bounds[:-1], bounds[1:])]
    halos = [conv_halo(s["q"], s["k"], s["v"]) for s in seg]
    As, Bs, wss = [], [], []
    for r, s in enumerate(seg):
        prev = dev["init_conv"] if r == 0 else halos[r - 1]
        ws = segment_workspace(kda, s["q"]) if records else None  # records prepared once per segment
        A, B = segment_carry(kda, s["q"], s["k"], s["v"], s["g"], s["beta"], dev["conv_w"], prev, workspace=ws)
        As.append(A)
        Bs.append(B)
        wss.append(ws)
    outs = []
    for r, s in enumerate(seg):
        S_in = compose_initial_state(dev["init_state"], As, Bs, r, kda.state_affine)
        prev = dev["init_conv"] if r == 0 else halos[r - 1]
        T = s["q"].shape[0]
        kw = {"workspace": wss[r], "mode": "scan"} if records else {}
        outs.append(kda.prefill(s["q"], s["k"], s["v"], s["g"], s["beta"], dev["conv_w"],
                                np.array([0, T], dtype=np.int32), init_state=S_in, init_conv=prev, **kw))
    torch.cuda.synchronize()
    assert kda.check_async_status() == 0
    o = torch.cat([x[0] for x in outs]).cpu()
    S, tail = outs[-1][1].cpu(), outs[-1][2].cpu()
    assert torch.equal(tail, whole_tail.cpu())
    ref = oracle.prefill(inp)
    tol = TOL[dtype] if dtype == torch.bfloat16 else 1e-4
    for h in range(H):
        # against the oracle: the composition adds the error of A and B to the state's
        assert rel_err(o[:, h].double().numpy(), ref[(0, h)].o) <= tol, h
        assert rel_err(S[0, h].double().numpy(), ref[(0, h)].final_state) <= tol, h
        # against one call on the GPU
        assert rel_err(o[:, h].double().numpy(), whole_o[:, h].cpu().double().numpy()) <= tol, h


@pytest.mark.parametrize("lens,H,sdt", [([700, 130, 5], 4, torch.float32), ([300, 300], 64, torch.float32),
                                        ([500, 64], 4, torch.bfloat16)])
def test_scan_over_kept_records_equals_prefill(lens, H, sdt):
    """kda_prefill_scan over the records of a kda_prefill_records call equals
    kda_prefill of its own arguments bit for bit, with other values, initial
    states, v history and output type, and again on a second scan; the
    records call itself equals kda_prefill.  12 chains (the overlapped
    schedule) and 128 chains (prep, then the scan)."""
    inp = ki.make_prefill(lens, H, torch.bfloat16, 96, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    d["init_state"] = d["init_state"].to(sdt)
    ws = torch.empty(kda.workspace_size(len(lens), sum(lens), H, max(lens)), dtype=torch.uint8, device="cuda")
    cu = inp.cu_seqlens
    args = lambda dd: (dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["conv_w"], cu, dd["cu_dev"])  # noqa: E731
    o1, S1, t1 = kda.prefill(*args(d), d["init_state"], d["init_conv"], workspace=ws, mode="records")
    o1f, S1f, t1f = kda.prefill(*args(d), d["init_state"], d["init_conv"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o1f) and torch.equal(S1, S1f) and torch.equal(t1, t1f)
    # other v, v history and initial state: the records do not depend on them
    d2 = dict(d)
    d2["v"] = ki.randn(tuple(inp.v.shape), 97, 1, dtype=torch.bfloat16).cuda()
    hist = d["init_conv"].clone()
    hist[:, 2] = ki.randn(tuple(hist[:, 2].shape), 97, 2, dtype=torch.bfloat16).cuda()
    S0 = ki.randn(tuple(inp.init_state.shape), 97, 3, std=0.05).cuda().to(sdt)
    want = kda.prefill(*args(d2), S0, hist, o_dtype=torch.bfloat16)
    for _ in range(2):
        got = kda.prefill(*args(d2), S0, hist, workspace=ws, mode="scan", o_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert kda.check_async_status() == 0
        for x, y in zip(got, want):
            assert torch.equal(x, y)
