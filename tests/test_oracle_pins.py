"""Pins for the fp64 oracle: closed forms, invariants, library routines and brute
force that the KDA definition fixes (page "GLM-5.3-Flash im Detail", section
"Sequenz-Mixing: 34 KDA-Schichten mit festem Zustand").  None of these retypes
the recurrence; each checks it against something independent of it."""
import os

import numpy as np
import pytest
import torch

import kda_inputs as ki
import oracle
from oracle import HeadProblem, forms

EPS = 1e-6  # L2-norm epsilon (inside the square root)
D = 128
IDENT = np.tile(np.array([0.0, 0.0, 0.0, 1.0]), (D, 1))  # conv taps that pass the current token


def _rng(seed):
    return np.random.default_rng(seed)


def _solve(p):
    oracle.run_problems([p], 1)
    return p


def _rel(a, b):
    return np.abs(a - b).max() / max(np.sqrt((b ** 2).mean()), 1e-300)


def _np_conv_norm(x, w, hist=None, norm=True, act=0):
    """Causal depthwise conv by numpy.convolve (kernel flipped: tap 3 = current
    token), optional SiLU, optional L2 normalisation."""
    T, d = x.shape
    h = np.zeros((3, d)) if hist is None else hist
    xs = np.concatenate([h, x], axis=0)
    y = np.stack([np.convolve(xs[:, c], w[c][::-1], mode="valid") for c in range(d)], axis=1)
    assert y.shape == (T, d)
    if act == 1:
        y = y * (1.0 / (1.0 + np.exp(-y)))
    if norm:
        y = y / np.sqrt((y ** 2).sum(axis=1, keepdims=True) + EPS)
    return y


def _random_problem(seed, T, d=D, beta=None, g=None, S0=True, hist=True, act=0):
    r = _rng(seed)
    q, k, v = r.standard_normal((3, T, d))
    gg = -5.0 / (1.0 + np.exp(-r.standard_normal((T, d)))) if g is None else g
    bb = 1.0 / (1.0 + np.exp(-r.standard_normal(T))) if beta is None else beta
    w = r.standard_normal((3, d, 4)) * 0.5
    st = r.standard_normal((d, d)) * 0.02 if S0 else None
    hh = list(r.standard_normal((3, 3, d))) if hist else None
    return HeadProblem(q, k, v, gg, bb, w[0], w[1], w[2], st, hh, act)


# ---------------------------------------------------------------- closed forms

def test_beta_zero_is_pure_channel_decay():
    """beta = 0: S_T = diag(exp(sum_t max(g_t,-5))) S_0 and
    o_t = (diag(exp(sum_{s<=t} g'_s)) S_0)^T q_hat_t.  Gates below -5 test the floor."""
    r = _rng(1)
    T = 50
    q = r.standard_normal((T, D))
    g = -6.0 * r.random((T, D))  # about 1/6 of them below the floor
    S0 = r.standard_normal((D, D))
    p = _solve(HeadProblem(q, r.standard_normal((T, D)), r.standard_normal((T, D)), g, np.zeros(T),
                           IDENT, IDENT, IDENT, S0, None))
    decay = np.exp(np.cumsum(np.maximum(g, -5.0), axis=0))  # [T][D]
    qn = q / np.sqrt((q ** 2).sum(1, keepdims=True) + EPS)
    o_ref = np.einsum("tk,kv,tk->tv", decay, S0, qn)
    # elementwise relative: T chained exp/multiply roundings vs one exp of the sum
    assert np.all(np.abs(p.o - o_ref) <= 1e-12 * np.abs(decay[:, :, None] * S0[None] * qn[:, :, None]).sum(1))
    S_ref = decay[-1][:, None] * S0
    assert np.all(np.abs(p.final_state - S_ref) <= 1e-12 * np.abs(S_ref))
    # zero state and beta = 0 -> identically zero output
    p0 = _solve(HeadProblem(q, q, q, g, np.zeros(T), IDENT, IDENT, IDENT, None, None))
    assert np.all(p0.o == 0.0) and np.all(p0.final_state == 0.0)


def test_orthonormal_keys_store_then_recall():
    """g = 0, beta = 1, identity conv, orthonormal keys: writing (k_i, v_i) then
    querying q = k_i returns v_i * s^2 with s^2 = 1/(1+eps) (the norm epsilon);
    rewriting a key replaces its value up to the same factor."""
    r = _rng(2)
    n = 40
    Qm, _ = np.linalg.qr(r.standard_normal((D, D)))
    keys = Qm[:n]  # orthonormal rows
    vals = r.standard_normal((n, D))
    # tokens 0..n-1 write, tokens n..2n-1 query with beta = 0
    k_in = np.concatenate([keys, keys])
    q_in = np.concatenate([keys, keys])
    v_in = np.concatenate([vals, np.zeros((n, D))])
    beta = np.concatenate([np.ones(n), np.zeros(n)])
    p = _solve(HeadProblem(q_in, k_in, v_in, np.zeros((2 * n, D)), beta, IDENT, IDENT, IDENT, None, None))
    s2 = 1.0 / (1.0 + EPS)
    assert np.abs(p.o[n:] - s2 * vals).max() < 1e-12
    # the state is the sum of outer products s * k_i v_i^T
    assert np.abs(p.final_state - np.sqrt(s2) * keys.T @ vals).max() < 1e-12
    # rewrite key 0 with a new value, then query it
    vnew = r.standard_normal(D)
    p2 = _solve(HeadProblem(np.stack([keys[0], keys[0], keys[0]]), np.stack([keys[0], keys[0], keys[0]]),
                            np.stack([vals[0], vnew, np.zeros(D)]), np.zeros((3, D)), np.array([1.0, 1.0, 0.0]),
                            IDENT, IDENT, IDENT, None, None))
    expect = s2 * ((1.0 - s2) * vals[0] + vnew)
    assert np.abs(p2.o[2] - expect).max() < 1e-12


def test_beta_one_recalls_last_write():
    """beta = 1 and q = k: o_t = S_t^T k_t = v_t for any gates and any S_0
    (keys of norm ~1e3 make the epsilon term ~1e-12)."""
    r = _rng(3)
    T = 30
    x = r.standard_normal((T, D)) * 1e3
    v = r.standard_normal((T, D))
    g = -5.0 * r.random((T, D))
    p = _solve(HeadProblem(x, x, v, g, np.ones(T), IDENT, IDENT, IDENT, r.standard_normal((D, D)), None))
    assert np.abs(p.o - v).max() < 1e-9


def test_conv_matches_numpy_convolve_and_tap_order():
    """g = 0, beta = 0, S_0 = I: o_t = q_hat_t, so the oracle's conv + norm on q
    must equal numpy.convolve with the flipped kernel (tap 3 = current token),
    including the 3-token history; and the SiLU variant."""
    r = _rng(4)
    T = 9
    q = r.standard_normal((T, D))
    w = r.standard_normal((D, 4))
    hist = r.standard_normal((3, D))
    for act in (0, 1):
        p = _solve(HeadProblem(q, q, q, np.zeros((T, D)), np.zeros(T), w, w, w, np.eye(D),
                               [hist, hist, hist], act))
        assert _rel(p.o, _np_conv_norm(q, w, hist, act=act)) < 1e-13
    # impulse response on v through the beta = 1, q = k recall: o_t = conv(v)_t
    x = r.standard_normal((T, D)) * 1e3
    imp = np.zeros((T, D))
    imp[2, 5] = 1.0
    wv = r.standard_normal((D, 4))
    p = _solve(HeadProblem(x, x, imp, np.zeros((T, D)), np.ones(T), IDENT, IDENT, wv, None, None))
    expect = np.zeros(T)
    for t in range(2, min(T, 6)):
        expect[t] = wv[5, 3 - (t - 2)]  # token t sees the impulse through tap 3-(t-2)
    assert np.abs(p.o[:, 5] - expect).max() < 1e-9
    assert np.abs(np.delete(p.o, 5, axis=1)).max() < 1e-9


def test_silu_closed_form_through_recall():
    """The SiLU activation of the conv (act = 1), pinned by values rather than by
    its formula: with identity taps, beta = 1 and q = k of norm ~1e3, o_t = v'_t,
    the activated value.  At x = ln a the sigmoid is a / (1 + a), so
    SiLU(ln a) = ln a * a / (1 + a); and SiLU(x) - SiLU(-x) = x,
    SiLU(x) + SiLU(-x) = x tanh(x / 2) (numpy's tanh)."""
    r = _rng(41)
    T = 8
    x = r.standard_normal((T, D)) * 1e3
    a = np.exp(r.uniform(-4.0, 4.0, (T, D)))
    lv = np.log(a)
    lv[:, 0] = 0.0  # SiLU(0) = 0
    outs = []
    for sign in (1.0, -1.0):
        p = _solve(HeadProblem(x, x, sign * lv, np.zeros((T, D)), np.ones(T), IDENT, IDENT, IDENT, None, None, 1))
        outs.append(p.o)
    assert np.abs(outs[0] - lv * a / (1.0 + a)).max() < 1e-9
    assert np.abs(outs[0][:, 0]).max() < 1e-12
    assert np.abs((outs[0] - outs[1]) - lv).max() < 1e-9
    assert np.abs((outs[0] + outs[1]) - lv * np.tanh(lv / 2.0)).max() < 1e-9


def test_key_conv_and_single_write():
    """One write at t = 0 (beta = 1, S_0 = 0, g = 0), then beta = 0: o_t =
    v_0 * (k_hat_0 . q_hat_t), with k_hat_0, q_hat_t, v_0 from numpy.convolve."""
    r = _rng(5)
    T = 6
    q, k, v = r.standard_normal((3, T, D))
    wq, wk, wv = r.standard_normal((3, D, 4))
    beta = np.zeros(T)
    beta[0] = 1.0
    p = _solve(HeadProblem(q, k, v, np.zeros((T, D)), beta, wq, wk, wv, None, None))
    qh = _np_conv_norm(q, wq)
    kh = _np_conv_norm(k, wk)
    vc = _np_conv_norm(v, wv, norm=False)
    expect = (qh @ kh[0])[:, None] * vc[0][None, :]
    assert _rel(p.o, expect) < 1e-12


# ----------------------------------------------------------------- invariants

def test_linearity_in_values_and_state():
    p1 = _solve(_random_problem(10, 70))
    p2 = _random_problem(10, 70)
    c = -2.5
    p2.v *= c
    p2.init_state *= c
    p2.hist[2] *= c
    _solve(p2)
    assert _rel(p2.o, c * p1.o) < 1e-13
    assert _rel(p2.final_state, c * p1.final_state) < 1e-13


def test_value_column_permutation():
    perm = _rng(11).permutation(D)
    p1 = _solve(_random_problem(11, 40))
    p2 = _random_problem(11, 40)
    p2.v = np.ascontiguousarray(p2.v[:, perm])
    p2.wv = np.ascontiguousarray(p2.wv[perm])
    p2.init_state = np.ascontiguousarray(p2.init_state[:, perm])
    p2.hist[2] = np.ascontiguousarray(p2.hist[2][:, perm])
    _solve(p2)
    assert np.array_equal(p2.o, p1.o[:, perm])
    assert np.array_equal(p2.final_state, p1.final_state[:, perm])


def test_causality():
    p1 = _solve(_random_problem(12, 60))
    p2 = _random_problem(12, 60)
    t0 = 33
    p2.q[t0] += 1.0
    p2.k[t0] -= 1.0
    p2.v[t0] += 3.0
    p2.g[t0] *= 0.5
    p2.beta[t0] = 0.3
    _solve(p2)
    assert np.array_equal(p1.o[:t0], p2.o[:t0])
    assert not np.array_equal(p1.o[t0], p2.o[t0])


def test_gate_floor_is_minus_five():
    p1 = _random_problem(13, 20)
    p1.g[:] = -5.0
    p2 = _random_problem(13, 20)
    p2.g[:] = -11.0
    _solve(p1), _solve(p2)
    assert np.array_equal(p1.o, p2.o) and np.array_equal(p1.final_state, p2.final_state)


def test_contraction_bound():
    """|k_hat| <= 1 and beta in [0,1] make (I - beta k k^T) Diag(alpha) a
    contraction: ||S_t||_2 <= ||S_{t-1}||_2 + beta_t ||v_t||."""
    base = _random_problem(14, 25)
    S = base.init_state.copy()
    hist = [h.copy() for h in base.hist]
    for t in range(base.T):
        p = _solve(HeadProblem(base.q[t:t + 1], base.k[t:t + 1], base.v[t:t + 1], base.g[t:t + 1],
                               base.beta[t:t + 1], base.wq, base.wk, base.wv, S, hist))
        vconv = _np_conv_norm(np.concatenate([hist[2], base.v[t:t + 1]])[-1:], base.wv,
                              hist[2], norm=False)[0]
        assert np.linalg.norm(p.final_state, 2) <= np.linalg.norm(S, 2) + base.beta[t] * np.linalg.norm(vconv) + 1e-12
        S, hist = p.final_state.copy(), [x.copy() for x in p.tail]


def test_varlen_packed_equals_separate():
    inp = ki.make_prefill([5, 70, 1, 130], 3, torch.float32, 99, state_std=0.02, conv_history=True)
    packed = oracle.prefill(inp)
    for n, L in enumerate([5, 70, 1, 130]):
        s0 = int(inp.cu_seqlens[n])
        single = ki.PrefillInputs(inp.q[s0:s0 + L], inp.k[s0:s0 + L], inp.v[s0:s0 + L], inp.g[s0:s0 + L],
                                  inp.beta[s0:s0 + L], inp.conv_w, inp.init_state[n:n + 1],
                                  inp.init_conv[n:n + 1], np.array([0, L], dtype=np.int32))
        res = oracle.prefill(single)
        for h in range(3):
            a, b = packed[(n, h)], res[(0, h)]
            assert np.array_equal(a.o, b.o) and np.array_equal(a.final_state, b.final_state)
            for x in range(3):
                assert np.array_equal(a.tail[x], b.tail[x])


def test_split_and_decode_equivalence():
    """prefill(T) == prefill(a) then prefill(T-a) carrying (state, conv tail)
    == T single-token decode steps."""
    full = _solve(_random_problem(15, 77))
    for a in (1, 2, 3, 40, 76):
        base = _random_problem(15, 77)
        p1 = HeadProblem(base.q[:a], base.k[:a], base.v[:a], base.g[:a], base.beta[:a],
                         base.wq, base.wk, base.wv, base.init_state, base.hist)
        _solve(p1)
        p2 = HeadProblem(base.q[a:], base.k[a:], base.v[a:], base.g[a:], base.beta[a:],
                         base.wq, base.wk, base.wv, p1.final_state, p1.tail)
        _solve(p2)
        assert _rel(np.concatenate([p1.o, p2.o]), full.o) < 1e-13
        assert _rel(p2.final_state, full.final_state) < 1e-13
    base = _random_problem(15, 77)
    S, hist, outs = base.init_state, base.hist, []
    for t in range(base.T):
        p = _solve(HeadProblem(base.q[t:t + 1], base.k[t:t + 1], base.v[t:t + 1], base.g[t:t + 1],
                               base.beta[t:t + 1], base.wq, base.wk, base.wv, S, hist))
        outs.append(p.o[0])
        S, hist = p.final_state, p.tail
    assert _rel(np.stack(outs), full.o) < 1e-13
    assert _rel(S, full.final_state) < 1e-13


def test_conv_tail_short_segments():
    """The tail is the last 3 raw tokens of history + segment, for T = 0, 1, 2, 3, 5."""
    r = _rng(16)
    hist = list(r.standard_normal((3, 3, D)))
    for T in (0, 1, 2, 3, 5):
        x = r.standard_normal((T, D))
        p = _solve(HeadProblem(x, x, x, np.zeros((T, D)), np.zeros(T), IDENT, IDENT, IDENT, None,
                               [h.copy() for h in hist]))
        for c in range(3):
            expect = np.concatenate([hist[c], x])[-3:]
            assert np.array_equal(p.tail[c], expect)


# ------------------------------------------------- independent forms / brute force

@pytest.mark.parametrize("d,T", [(2, 1), (2, 4), (4, 3), (4, 4), (128, 9)])
def test_literal_matrix_form_equals_recurrence(d, T):
    for seed in range(3):
        p = _solve(_random_problem(100 + seed, T, d=d))
        o, S = forms.literal_head(p)
        assert _rel(p.o, o) < 1e-12 and _rel(p.final_state, S) < 1e-12


@pytest.mark.parametrize("C", [1, 7, 16, 64])
def test_chunked_form_equals_recurrence(C):
    p = _solve(_random_problem(200 + C, 150))
    o, S = forms.chunked_head(p, C)
    assert _rel(p.o, o) < 1e-12 and _rel(p.final_state, S) < 1e-12


def test_chunked_partial_last_chunks_and_floor_gates():
    """Chunk 64 with every partial-last-chunk length class and gates pinned at
    the -5 floor for whole chunks (Gamma reaches -320 inside a chunk)."""
    for T in (1, 2, 3, 63, 64, 65, 127, 128, 131):
        p = _random_problem(300 + T, T)
        p.g[:, :16] = -5.0
        _solve(p)
        o, S = forms.chunked_head(p, 64)
        assert _rel(p.o, o) < 1e-12 and _rel(p.final_state, S) < 1e-12


def test_workload_zero_decode_matches_prefill():
    """The decode wrapper (conv cache as history, T = 1) equals one prefill token."""
    dec = ki.make_decode(3, 2, torch.float32, 7)
    res = oracle.decode(dec)
    for (n, h), p in res.items():
        c = dec.conv_cache.view(3, 3, 3, 2, D)[n, :, :, h].double().numpy()
        w = dec.conv_w.view(3, 2, D, 4)[:, h].double().numpy()
        ref = _solve(HeadProblem(dec.q[n, h][None], dec.k[n, h][None], dec.v[n, h][None],
                                 dec.g[n, h][None], dec.beta[n, h].reshape(1), w[0], w[1], w[2],
                                 dec.state[n, h], [c[0], c[1], c[2]]))
        assert np.array_equal(p.o, ref.o)
        # literal form on the same single step
        o, S = forms.literal_head(p)
        assert _rel(p.o, o) < 1e-12 and _rel(p.final_state, S) < 1e-12


def test_decode_rows_wrapper_equals_chained_single_steps():
    """The multi-row decode wrapper (rows of sequence n, head h of [N, R, H, D]
    inputs, cache as history) keeping r rows equals r single-token steps that
    carry the state and the conv cache; r = 0 keeps state and cache as given."""
    inp = ki.make_decode_rows(3, 6, 2, torch.float32, 31)
    for n in range(3):
        for h in range(2):
            c = inp.conv_cache.view(3, 3, 3, 2, D)[n, :, :, h].double().numpy()
            w = inp.conv_w.view(3, 2, D, 4)[:, h].double().numpy()
            S, hist, outs = inp.state[n, h].double().numpy(), [c[0], c[1], c[2]], []
            for r in range(7):
                p = oracle.decode_rows_problem(inp, n, h, r)
                _solve(p)
                assert np.array_equal(p.final_state, S) and np.array_equal(p.o, np.array(outs).reshape(r, D))
                for x in range(3):
                    assert np.array_equal(p.tail[x], hist[x])
                if r < 6:
                    step = _solve(HeadProblem(inp.q[n, r, h][None], inp.k[n, r, h][None], inp.v[n, r, h][None],
                                              inp.g[n, r, h][None], inp.beta[n, r, h].reshape(1), w[0], w[1], w[2],
                                              S, hist))
                    outs.append(step.o[0])
                    S, hist = step.final_state, step.tail


# ---------------------------------------------------------------- bf16 state storage

def _bf16_neighbours(x):
    """The two bf16 values around double x (truncation toward zero and the next
    one away from zero), from frexp: 8 significant bits, fp32 exponent range."""
    m, e = np.frexp(x)
    ulp = np.ldexp(1.0, np.maximum(e - 8, -133))
    lo = np.trunc(x / ulp) * ulp
    return lo, lo + np.sign(x) * ulp, ulp


def test_bf16_rounding_is_nearest_ties_to_even():
    """Brute force on random doubles of every magnitude (and exact ties): the
    result is one of the two neighbouring bf16 values, the nearer one, and on a
    tie the one with an even last mantissa bit; it is representable as bf16
    (an fp32 whose low 16 bits are zero)."""
    r = _rng(5)
    x = r.standard_normal(20000) * np.ldexp(1.0, r.integers(-140, 40, 20000))
    lo, hi, ulp = _bf16_neighbours(x)
    ties = lo[:2000] + np.sign(x[:2000]) * ulp[:2000] / 2  # exactly halfway
    x = np.concatenate([x, ties, [0.0, 1.0, -2.5, 1 + 2 ** -8, 1 + 3 * 2 ** -8]])
    lo, hi, ulp = _bf16_neighbours(x)
    y = oracle.round_bf16(x)
    assert np.all((y == lo) | (y == hi))
    d_lo, d_hi = np.abs(x - lo), np.abs(x - hi)
    nearer = np.where(d_lo < d_hi, lo, hi)
    tie = d_lo == d_hi
    assert np.array_equal(y[~tie], nearer[~tie])
    even = np.where(np.round(lo / ulp) % 2 == 0, lo, hi)
    assert np.array_equal(y[tie], even[tie]) and tie.sum() >= 2000
    f = y.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), y) and not np.any(f.view(np.uint32) & 0xFFFF)


def test_state_rounded_at_end_changes_only_the_stored_state():
    """Storage in bf16 at the end of a call: outputs are those of the exact
    recurrence and the final state is the exact final state rounded once."""
    for seed, T in ((70, 1), (71, 37)):
        a, b = _random_problem(seed, T), _random_problem(seed, T)
        b.state_round = oracle.STATE_BF16_AT_END
        _solve(a); _solve(b)
        assert np.array_equal(a.o, b.o)
        assert np.array_equal(b.final_state, oracle.round_bf16(a.final_state))


def test_state_rounded_each_token_equals_chained_stored_steps():
    """Storage in bf16 after every token = T single-token decode steps, each
    starting from the previous step's stored (rounded) state and conv cache and
    rounding its own final state once; the readout of a step uses the state
    before storage.  The rounding does change the result (it is not a no-op)."""
    T = 9
    full = _random_problem(72, T)
    full.state_round = oracle.STATE_BF16_EACH_TOKEN
    _solve(full)
    exact = _random_problem(72, T)
    _solve(exact)
    S, hist = full.init_state, full.hist
    for t in range(T):
        step = HeadProblem(full.q[t:t + 1], full.k[t:t + 1], full.v[t:t + 1], full.g[t:t + 1], full.beta[t:t + 1],
                           full.wq, full.wk, full.wv, S, hist, 0, oracle.STATE_BF16_AT_END)
        _solve(step)
        assert np.array_equal(step.o[0], full.o[t]), t
        S, hist = step.final_state, step.tail
    assert np.array_equal(S, full.final_state)
    # storage drift from the exact state: rounding moves each stored element by
    # at most half a bf16 ulp (2^-9 relative) per step, and the largest
    # elements are several rms, so after 9 steps max|err|/rms is about 2 %
    drift = _rel(full.final_state, exact.final_state)
    assert 2 ** -9 < drift < 0.05


# ---------------------------------------------------------------- page numbers

def test_page_dimensions():
    vals = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "kda_dims.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, val = line.split()
                vals[key] = float(val)
    H, Dh = int(vals["heads"]), int(vals["head_dim"])
    dec = ki.make_decode(1, H, torch.bfloat16, 0)
    per_layer = dec.state[0].numel()
    assert per_layer == vals["state_scalars_per_layer"] == H * Dh * Dh
    assert per_layer * vals["kda_layers"] == vals["state_scalars_per_request"]
    mib = per_layer * vals["kda_layers"] * dec.state.element_size() / 2 ** 20
    assert round(mib) == vals["state_fp32_mib_per_request"]
    assert dec.conv_w.shape[-1] == vals["conv_width"]
