"""GPU parity of the output epilogue (gated RMS normalisation of each head's
output row) against the fp64 oracle, through the C ABI: fused into the chunked
prefill (kda_prefill_gated) and on its own (kda_output_norm).

Tolerance: the epilogue's reference is the oracle epilogue applied to the
oracle's mixer output.  Per element |y - y_ref| <= tol * rms(y_ref) + 2^-7 |y_ref|
per (sequence, head): the mixer's own bar (tol = 2e-2 for bf16 inputs, 1e-4 for
fp32) plus the bf16 rounding of y (at most 2^-9 relative) with margin for the
fp32 normalisation."""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
import oracle
from oracle import epilogue
from parity import run_prefill, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _check(y, ref, tol, what):
    rms = float(np.sqrt((ref ** 2).mean()))
    err = np.abs(y - ref)
    bound = tol * rms + 2.0 ** -7 * np.abs(ref)
    worst = float((err / np.maximum(bound, 1e-30)).max())
    assert worst <= 1.0, f"{what}: worst error {worst:.3f} of the bound"
    return worst


def _gated(inp, seed, pairs=None, dev_inputs=None):
    d = dev_inputs or to_dev(inp)
    T, H = inp.q.shape[0], inp.q.shape[1]
    z, w = ki.make_output_norm(T, H, seed)
    y, S, tail = run_prefill(inp, dev_inputs=d, gate=z.cuda(), norm_weight=w.cuda(), norm_eps=EPS)
    assert y.dtype == torch.bfloat16
    if pairs is None:
        pairs = [(n, h) for n in range(inp.num_seqs) for h in range(H)]
    ref = oracle.prefill(inp, pairs)
    yc, zc = y.float().cpu().numpy(), z.float().numpy()
    worst = 0.0
    for (n, h), p in ref.items():
        s0, s1 = int(inp.cu_seqlens[n]), int(inp.cu_seqlens[n + 1])
        if s1 == s0:
            continue
        yr = epilogue.gated_rmsnorm(p.o, zc[s0:s1, h], w.double().numpy(), EPS)
        worst = max(worst, _check(yc[s0:s1, h], yr, 2e-2, f"seq {n} head {h}"))
    return y, S, tail, z, w, worst


def test_gated_prefill_edge_lengths():
    """Ragged lengths around the chunk size, segments shorter than the conv
    window, an empty segment, conv history and initial states; the state and
    conv tails equal those of the plain call bit for bit."""
    lens = [1, 2, 3, 0, 63, 64, 65, 127, 130]
    inp = ki.make_prefill(lens, 2, torch.bfloat16, 31, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    y, S, tail, _, _, _ = _gated(inp, 31, dev_inputs=d)
    _, S0, tail0 = run_prefill(inp, dev_inputs=d)
    assert torch.equal(S, S0) and torch.equal(tail, tail0)


def test_gated_prefill_equals_two_step():
    """The fused epilogue against the plain prefill (fp32 o) followed by
    kda_output_norm: the same arithmetic up to the summation order of the
    mean square, so at most a few bf16 units apart."""
    inp = ki.make_prefill([300, 64, 7], 3, torch.bfloat16, 32, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    T, H = inp.q.shape[0], inp.q.shape[1]
    z, w = ki.make_output_norm(T, H, 32)
    zd, wd = z.cuda(), w.cuda()
    y, _, _ = run_prefill(inp, dev_inputs=d, gate=zd, norm_weight=wd, norm_eps=EPS)
    o, _, _ = run_prefill(inp, dev_inputs=d)
    y2 = kda.output_norm(o, zd, wd, EPS)
    torch.cuda.synchronize()
    a, b = y.float(), y2.float()
    assert torch.all((a - b).abs() <= 2.0 ** -7 * b.abs() + 1e-6), float((a - b).abs().max())


@pytest.mark.parametrize("silu", [0, 1])
def test_gated_prefill_several_chunks(silu):
    """Several chunks per segment with a ragged tail, both conv activations."""
    inp = ki.make_prefill([1000, 333], 2, torch.bfloat16, 33 + silu, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    T, H = inp.q.shape[0], inp.q.shape[1]
    z, w = ki.make_output_norm(T, H, 33)
    y, _, _ = run_prefill(inp, dev_inputs=d, act=silu, gate=z.cuda(), norm_weight=w.cuda(), norm_eps=EPS)
    ref = oracle.prefill(inp, act=silu)
    for (n, h), p in ref.items():
        s0, s1 = int(inp.cu_seqlens[n]), int(inp.cu_seqlens[n + 1])
        yr = epilogue.gated_rmsnorm(p.o, z[s0:s1, h].double().numpy(), w.double().numpy(), EPS)
        _check(y[s0:s1, h].float().cpu().numpy(), yr, 2e-2, f"seq {n} head {h}")


@pytest.mark.parametrize("silu", [0, 1])
def test_gated_prefill_many_chains(silu):
    """More than 96 (segment, head) chains: the preparation and the scan run one
    after the other (the schedule of the multi-sequence workloads), with the
    epilogue instance of the scan; ragged lengths, conv history and initial
    states.  Every pair against the oracle; state and conv tails bit-identical
    to the plain call."""
    lens = [300, 64, 1, 190, 65, 7, 128, 250]
    inp = ki.make_prefill(lens, 16, torch.bfloat16, 39 + silu, state_std=0.02, conv_history=True)
    assert inp.num_seqs * inp.num_heads > 96
    d = to_dev(inp)
    T, H = inp.q.shape[0], inp.q.shape[1]
    z, w = ki.make_output_norm(T, H, 39)
    y, S, tail = run_prefill(inp, dev_inputs=d, act=silu, gate=z.cuda(), norm_weight=w.cuda(), norm_eps=EPS)
    _, S0, tail0 = run_prefill(inp, dev_inputs=d, act=silu)
    assert torch.equal(S, S0) and torch.equal(tail, tail0)
    ref = oracle.prefill(inp, act=silu)
    yc, zc = y.float().cpu().numpy(), z.double().numpy()
    for (n, h), p in ref.items():
        s0, s1 = int(inp.cu_seqlens[n]), int(inp.cu_seqlens[n + 1])
        yr = epilogue.gated_rmsnorm(p.o, zc[s0:s1, h], w.double().numpy(), EPS)
        _check(yc[s0:s1, h], yr, 2e-2, f"seq {n} head {h}")


def test_gated_prefill_long_context_full_size():
    """1 x 65,536 tokens, 64 heads, with the epilogue: every head against the
    oracle, in the launch configuration the benchmark times (overlapped)."""
    inp = ki.workload(2)
    _gated(inp, 34)


def test_gated_prefill_extreme_gates():
    """Gates far in both tails (sigmoid 1 in fp32, and all but closed) and a zero eps."""
    inp = ki.make_prefill([130], 2, torch.bfloat16, 35, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    T, H = inp.q.shape[0], inp.q.shape[1]
    _, w = ki.make_output_norm(T, H, 35)
    z = torch.full((T, H, 128), 100.0, dtype=torch.bfloat16)
    z[::2] = -100.0
    y, _, _ = run_prefill(inp, dev_inputs=d, gate=z.cuda(), norm_weight=w.cuda(), norm_eps=0.0)
    assert torch.all(torch.isfinite(y.float()))
    ref = oracle.prefill(inp)
    for (n, h), p in ref.items():
        yr = epilogue.gated_rmsnorm(p.o, z[:, h].double().numpy(), w.double().numpy(), 0.0)
        _check(y[:, h].float().cpu().numpy(), yr, 2e-2, f"head {h}")
    # a closed gate: sigmoid(-100) = 3.7e-44 (the kernel's sigmoid saturates at 2^-64 there)
    assert torch.all(y[::2].float().abs() < 1e-15)


@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16])
def test_output_norm_standalone(odt):
    """kda_output_norm on exact inputs: only fp32 arithmetic and the bf16
    rounding of y separate it from the oracle; bf16 o also in place."""
    rows, H = 1000, 3
    o = ki.randn((rows, H, 128), 36, 1, std=3.0, dtype=odt)
    z, w = ki.make_output_norm(rows, H, 36)
    y = kda.output_norm(o.cuda(), z.cuda(), w.cuda(), 1e-5)
    ref = epilogue.gated_rmsnorm(o.double().numpy(), z.double().numpy(), w.double().numpy(), 1e-5)
    err = np.abs(y.float().cpu().numpy() - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6), float(err.max())
    if odt == torch.bfloat16:
        od = o.cuda()
        y2 = kda.output_norm(od, z.cuda(), w.cuda(), 1e-5, y=od)
        torch.cuda.synchronize()
        assert torch.equal(y2.cpu(), y.cpu())


def test_output_norm_after_decode():
    """A decode step's output through the standalone epilogue, against the
    oracle's decode output through the oracle epilogue."""
    inp = ki.make_decode(16, 4, torch.bfloat16, 37)
    st, cc = inp.state.cuda(), inp.conv_cache.cuda()
    o = kda.decode_step(st, cc, inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.g.cuda(), inp.beta.cuda(),
                        inp.conv_w.cuda())
    z, w = ki.make_output_norm(16, 4, 37)
    y = kda.output_norm(o, z.cuda(), w.cuda(), EPS)
    ref = oracle.decode(inp)
    yc = y.float().cpu().numpy()
    for (n, h), p in ref.items():
        yr = epilogue.gated_rmsnorm(p.o[0], z[n, h].double().numpy(), w.double().numpy(), EPS)
        _check(yc[n, h], yr, 1e-4, f"seq {n} head {h}")


@pytest.mark.parametrize("silu", [0, 1])
def test_gated_prefill_bf16_state(silu):
    """The epilogue instance with bf16 state storage and both conv activations:
    the final state equals the plain call's bit for bit, and the output the
    plain call's output through the standalone epilogue within 2^-7."""
    inp = ki.make_prefill([400, 90], 3, torch.bfloat16, 38 + silu, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    d["init_state"] = d["init_state"].to(torch.bfloat16)
    T, H = inp.q.shape[0], inp.q.shape[1]
    z, w = ki.make_output_norm(T, H, 38)
    zd, wd = z.cuda(), w.cuda()
    y, S, tail = run_prefill(inp, dev_inputs=d, act=silu, gate=zd, norm_weight=wd, norm_eps=EPS)
    o, S0, tail0 = run_prefill(inp, dev_inputs=d, act=silu)
    assert S.dtype == torch.bfloat16 and torch.equal(S, S0) and torch.equal(tail, tail0)
    y2 = kda.output_norm(o, zd, wd, EPS)
    torch.cuda.synchronize()
    a, b = y.float(), y2.float()
    assert torch.all((a - b).abs() <= 2.0 ** -7 * b.abs() + 1e-6), float((a - b).abs().max())
