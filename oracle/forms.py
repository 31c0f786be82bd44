"""Two further fp64 evaluations of the KDA step, written independently of the C
recurrence so that agreement between them pins the algebra (test
infrastructure only).

Source: page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34
KDA-Schichten mit festem Zustand" (conv width 4 on q/k/v, channel-wise forget
gate with log-decay floor -5, scalar-beta delta rule, readout of the updated
state; prefill evaluates tokens in parallel inside a chunk and hands a state
from chunk to chunk).

* ``literal_head``: S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1}
  + beta_t k_t v_t^T with the d x d update matrix formed explicitly, then
  o_t = S_t^T q_t.
* ``chunked_head``: the chunk form.  Inside a chunk of C tokens, with
  Gamma_i = sum_{s<=i} g'_s (per key channel, g' = max(g, -5)):
      M_ij = sum_c k_ic k_jc exp(Gamma_ic - Gamma_jc)        (i > j)
      P_ij = sum_c q_ic k_jc exp(Gamma_ic - Gamma_jc)        (j <= i)
      T    = (I + diag(beta) M)^-1 diag(beta)                (forward substitution)
      W    = T (exp(Gamma) * K),   U~ = T V,   U = U~ - W S
      O    = (exp(Gamma) * Q) S + P U
      S   <- diag(exp(Gamma_C)) S + sum_j (exp(Gamma_C - Gamma_j) * k_j) u_j^T
  It follows from expanding S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T with
  u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t): an exact rearrangement,
  every exponential taken of a difference <= 0.
"""
from __future__ import annotations

import numpy as np

LOG_DECAY_FLOOR = -5.0
NORM_EPS = 1e-6


def _conv(x: np.ndarray, w: np.ndarray, hist, act: int) -> np.ndarray:
    """x [T][d], w [d][4], hist [3][d] or None -> y [T][d]; tap 3 = current."""
    T, d = x.shape[0], w.shape[0]
    h = np.zeros((3, d)) if hist is None else np.asarray(hist, dtype=np.float64)
    xs = np.concatenate([h, x.reshape(T, d)], axis=0)  # [T+3][d]
    y = np.zeros((T, d))
    for j in range(4):
        y += w[:, j][None, :] * xs[j:j + T]
    if act == 1:
        y = y / (1.0 + np.exp(-y))
    return y


def prologue(p):
    """conv + L2 norm (q, k) + clamped log-decay, from a HeadProblem's raw arrays."""
    hist = p.hist if p.hist is not None else [None, None, None]
    q = _conv(p.q, p.wq, hist[0], p.act)
    k = _conv(p.k, p.wk, hist[1], p.act)
    v = _conv(p.v, p.wv, hist[2], p.act)
    q = q / np.sqrt((q * q).sum(axis=1, keepdims=True) + NORM_EPS)
    k = k / np.sqrt((k * k).sum(axis=1, keepdims=True) + NORM_EPS)
    gl = np.maximum(p.g.reshape(p.T, -1), LOG_DECAY_FLOOR)
    return q, k, v, gl, p.beta.reshape(-1)


def _init_state(p) -> np.ndarray:
    return np.zeros((p.dk, p.dv)) if p.init_state is None else np.array(p.init_state, dtype=np.float64)


def literal_head(p):
    """Returns (o [T][dv], S_T [dk][dv]) with explicit update matrices."""
    q, k, v, gl, beta = prologue(p)
    S = _init_state(p)
    eye = np.eye(p.dk)
    o = np.zeros((p.T, p.dv))
    for t in range(p.T):
        A = (eye - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(gl[t]))
        S = A @ S + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def chunked_head(p, C: int = 64):
    """Returns (o [T][dv], S_T [dk][dv]) via the chunk form with chunk size C."""
    q, k, v, gl, beta = prologue(p)
    S = _init_state(p)
    o = np.zeros((p.T, p.dv))
    for s0 in range(0, p.T, C):
        s1 = min(p.T, s0 + C)
        n = s1 - s0
        Q, K, V, b = q[s0:s1], k[s0:s1], v[s0:s1], beta[s0:s1]
        G = np.cumsum(gl[s0:s1], axis=0)  # Gamma_i, [n][dk]
        ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        lower_eq = (ii >= jj)[:, :, None]
        # exp(Gamma_i - Gamma_j) only where i >= j (difference <= 0); zero elsewhere
        E = np.exp(np.where(lower_eq, G[:, None, :] - G[None, :, :], -np.inf))
        M = np.einsum("ic,jc,ijc->ij", K, K, E) * (ii > jj)
        P = np.einsum("ic,jc,ijc->ij", Q, K, E)
        # T = (I + diag(b) M)^-1 diag(b) by forward substitution, row by row
        L = b[:, None] * M
        Tm = np.zeros((n, n))
        for i in range(n):
            row = np.zeros(n)
            row[i] = b[i]
            for j in range(i):
                row -= L[i, j] * Tm[j]
            Tm[i] = row
        Kt = np.exp(G) * K
        W = Tm @ Kt
        U = Tm @ V - W @ S
        o[s0:s1] = (np.exp(G) * Q) @ S + P @ U
        Kbar = np.exp(G[-1][None, :] - G) * K
        S = np.exp(G[-1])[:, None] * S + Kbar.T @ U
    return o, S
