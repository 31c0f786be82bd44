"""Helpers shared by the GPU parity tests: run the CUDA library through the
C ABI on seeded inputs and compare with the fp64 oracle element by element.

Tolerance (max|err| / rms(reference), per (sequence, head) pair, for the output
o and for the final state):  1e-4 when the inputs are fp32, 2e-2 when they are
bf16.  Conv tails are copies of raw inputs and must match bit for bit."""
from __future__ import annotations

import numpy as np
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
import oracle

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def to_dev(inp, dev="cuda"):
    f = lambda t: None if t is None else t.to(dev, non_blocking=False)  # noqa: E731
    return {"q": f(inp.q), "k": f(inp.k), "v": f(inp.v), "g": f(inp.g), "beta": f(inp.beta),
            "conv_w": f(inp.conv_w), "init_state": f(inp.init_state), "init_conv": f(inp.init_conv),
            "cu_dev": torch.from_numpy(inp.cu_seqlens).to(dev)}


def run_prefill(inp, recurrent=False, act=0, dev_inputs=None, **kw):
    d = dev_inputs or to_dev(inp)
    o, S, tail = kda.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], inp.cu_seqlens,
                             d["cu_dev"], d["init_state"], d["init_conv"], act=act, recurrent=recurrent,
                             **kw)
    torch.cuda.synchronize()
    assert kda.check_async_status() == 0
    return o, S, tail


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    rms = float(np.sqrt((ref ** 2).mean())) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.abs(got - ref).max() / max(rms, 1e-30))


def compare_prefill(inp, outs, pairs=None, act=0, tol=None, check_tail=True, batch=64):
    """Compares GPU (o, final_state, conv_tail) with the oracle on `pairs`
    (every (sequence, head) pair by default), `batch` pairs per oracle run so
    that host memory stays bounded on the large workloads.  Returns the worst
    (o, state) relative errors."""
    tol = tol or TOL[inp.dtype]
    o, S, tail = [x.cpu() for x in outs]
    if pairs is None:
        pairs = [(n, h) for n in range(inp.num_seqs) for h in range(inp.num_heads)]
    pairs = list(pairs)
    worst_o = worst_s = 0.0
    D = inp.q.shape[2]
    H = inp.num_heads
    for b in range(0, len(pairs), batch):
        wo, ws = _compare_batch(inp, o, S, tail, pairs[b:b + batch], act, tol, check_tail, D, H)
        worst_o, worst_s = max(worst_o, wo), max(worst_s, ws)
    return worst_o, worst_s


def _compare_batch(inp, o, S, tail, pairs, act, tol, check_tail, D, H):
    ref = oracle.prefill(inp, pairs, act=act)
    worst_o = worst_s = 0.0
    for (n, h), p in ref.items():
        s0, s1 = int(inp.cu_seqlens[n]), int(inp.cu_seqlens[n + 1])
        eo = rel_err(o[s0:s1, h].double().numpy(), p.o)
        es = rel_err(S[n, h].double().numpy(), p.final_state)
        worst_o, worst_s = max(worst_o, eo), max(worst_s, es)
        assert eo <= tol, f"o mismatch at seq {n} head {h}: {eo:.3e} > {tol}"
        assert es <= tol, f"state mismatch at seq {n} head {h}: {es:.3e} > {tol}"
        if check_tail:
            t = tail.view(inp.num_seqs, 3, 3, H, D)[n, :, :, h].double().numpy()
            for x in range(3):
                assert np.array_equal(t[x], p.tail[x]), f"conv tail mismatch seq {n} head {h} x {x}"
    return worst_o, worst_s


def sample_pairs(inp, count, seed=0):
    rng = np.random.default_rng(seed)
    N, H = inp.num_seqs, inp.num_heads
    lens = np.diff(inp.cu_seqlens)
    pairs = {(int(np.argmax(lens)), 0), (int(np.argmin(lens)), H - 1)}
    while len(pairs) < min(count, N * H):
        pairs.add((int(rng.integers(N)), int(rng.integers(H))))
    return sorted(pairs)
