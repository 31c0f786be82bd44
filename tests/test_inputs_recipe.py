"""The seeded input generators follow the stated recipe: bit-identical for the
same seed whatever the thread count, the stated distributions and structure,
and bf16 workloads equal to the fp32 draws rounded once (nearest, ties to even)."""
import numpy as np
import pytest
import torch

import kda_inputs as ki


def test_same_seed_same_bits_whatever_the_thread_count(monkeypatch):
    a = ki.make_prefill([3000, 1200], 4, torch.float32, 11, state_std=0.02, conv_history=True)
    monkeypatch.setattr(ki, "_threads", lambda: 1)
    b = ki.make_prefill([3000, 1200], 4, torch.float32, 11, state_std=0.02, conv_history=True)
    for name in ("q", "k", "v", "g", "beta", "conv_w", "init_state", "init_conv"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    c = ki.make_prefill([3000, 1200], 4, torch.float32, 12)
    assert not torch.equal(a.q, c.q)
    assert not torch.equal(a.q, a.k) and not torch.equal(a.k, a.v)  # each tensor its own stream


def test_distributions():
    inp = ki.make_prefill([8192], 8, torch.float32, 13, state_std=0.02, conv_history=True)
    for name in ("q", "k", "v", "init_conv"):
        x = getattr(inp, name).double()
        assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01, name
    assert abs(inp.conv_w.double().std().item() - 0.5) < 0.01      # variance 1/4
    assert abs(inp.init_state.double().std().item() - 0.02) < 0.001
    g = inp.g.double()
    assert g.max().item() < 0.0 and g.min().item() > -5.0          # -5 sigmoid(N(0,1))
    assert abs(g.median().item() + 2.5) < 0.02
    b = inp.beta.double()
    assert b.min().item() > 0.0 and b.max().item() < 1.0 and abs(b.median().item() - 0.5) < 0.01


def test_bimodal_gate_structure():
    T, H, D = 512, 8, 128
    g = ki.gate_bimodal(T, H, D, 14).view(T, H * D)
    low = g[0] < -4.0
    assert int(low.sum()) == round(0.1 * H * D)                    # a seeded 10 % of (head, channel)
    assert torch.equal(g < -4.0, low.expand(T, -1))                 # the same pairs for every token
    sel, rest = g[:, low], g[:, ~low]
    assert sel.min().item() >= -5.0 and sel.max().item() <= -4.9   # -5 + 0.1 U(0,1)
    assert rest.min().item() >= -0.05 and rest.max().item() <= 0.0  # -0.05 U(0,1)


def test_bf16_workloads_are_the_fp32_draws_rounded_once():
    a = ki.make_prefill([700], 3, torch.float32, 15, conv_history=True)
    b = ki.make_prefill([700], 3, torch.bfloat16, 15, conv_history=True)
    for name in ("q", "k", "v", "g", "beta", "init_conv"):
        assert getattr(b, name).dtype == torch.bfloat16
        assert torch.equal(getattr(a, name).to(torch.bfloat16), getattr(b, name)), name
    assert b.conv_w.dtype == torch.float32 and torch.equal(a.conv_w, b.conv_w)


def test_workload_shapes_and_lengths():
    lens = ki.varlen_lengths(ki.BASE_SEED + 3)
    assert len(lens) == 16 and all(1024 <= n <= 32768 for n in lens)
    w0 = ki.workload(0)
    assert w0.q.shape == (256, 2, 128) and w0.dtype == torch.float32 and list(w0.cu_seqlens) == [0, 256]
    rows = ki.make_decode_rows(64, 6, 2, torch.bfloat16, 16, accept=(2, 6))
    assert rows.q.shape == (64, 6, 2, 128) and rows.beta.shape == (64, 6, 2)
    assert rows.n_accept.min() >= 2 and rows.n_accept.max() <= 6
    dec = ki.make_decode(5, 3, torch.bfloat16, 17)
    assert dec.state.shape == (5, 3, 128, 128) and dec.state.dtype == torch.float32
    assert dec.conv_cache.shape == (5, 3, 3, 3 * 128)


@pytest.mark.parametrize("seed", [0, 1, 2**40 + 3])
def test_stream_seeds_are_distinct(seed):
    seeds = {ki._mix(seed, s, b) for s in range(1, 13) for b in range(4)}
    assert len(seeds) == 12 * 4
