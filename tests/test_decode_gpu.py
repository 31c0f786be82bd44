"""GPU parity of kda_decode_step against the fp64 oracle through the C ABI."""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
import oracle
from parity import TOL, rel_err

pytestmark = pytest.mark.gpu


def _run(inp, act=0):
    state = inp.state.clone().cuda()
    cache = inp.conv_cache.clone().cuda()
    o = kda.decode_step(state, cache, inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.g.cuda(),
                        inp.beta.cuda(), inp.conv_w.cuda(), act=act)
    torch.cuda.synchronize()
    return o.cpu(), state.cpu(), cache.cpu()


def _compare(inp, outs, act=0):
    o, S, cache = outs
    tol = TOL[inp.dtype]
    ref = oracle.decode(inp, act=act)
    D, H = inp.q.shape[2], inp.num_heads
    cv = cache.view(inp.num_seqs, 3, 3, H, D)
    worst = 0.0
    for (n, h), p in ref.items():
        eo = rel_err(o[n, h].double().numpy(), p.o[0])
        es = rel_err(S[n, h].double().numpy(), p.final_state)
        worst = max(worst, eo, es)
        assert eo <= tol and es <= tol, (n, h, eo, es)
        for x in range(3):
            assert np.array_equal(cv[n, x, :, h].double().numpy(), p.tail[x])
    return worst


def test_workload4_decode_full_size():
    inp = ki.workload(4)
    _compare(inp, _run(inp))


@pytest.mark.parametrize("act", [0, 1])
def test_decode_fp32(act):
    inp = ki.make_decode(5, 3, torch.float32, 21)
    assert _compare(inp, _run(inp, act), act) <= 1e-4


def test_decode_bf16_output_is_rounded_fp32_output():
    inp = ki.make_decode(6, 4, torch.bfloat16, 23)
    outs = []
    for od in (torch.float32, torch.bfloat16):
        state = inp.state.clone().cuda()
        cache = inp.conv_cache.clone().cuda()
        outs.append(kda.decode_step(state, cache, inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.g.cuda(),
                                    inp.beta.cuda(), inp.conv_w.cuda(), o_dtype=od))
    assert torch.equal(outs[1], outs[0].to(torch.bfloat16))


def test_decode_bf16_silu_single_head():
    inp = ki.make_decode(7, 1, torch.bfloat16, 22)
    _compare(inp, _run(inp, 1), 1)
