"""Seeded synthetic inputs for the KDA sequence-mixing step.

This module only draws random tensors and lays them out; it contains none of the
method's arithmetic (no convolution, normalisation, gating or state update).  It
is the one module that both the fp64 oracle and the CUDA library are fed from,
so that both see bit-identical inputs.

Layouts (all per-token tensors packed token-major, channel contiguous):
  q, k, v, g     [total_T, H, D]      float32 or bfloat16
  beta           [total_T, H]         same dtype
  conv_w         [3, H*D, 4]          float32  (q, k, v taps; tap 3 = current token)
  init_state     [N, H, D, D]         float32  (row = key channel, column = value channel)
  init_conv      [N, 3, 3, H*D]       input dtype (q/k/v, 3 tokens oldest first)
  cu_seqlens     [N+1]                int32 offsets of each segment
Decode inputs use [N, H, D] for q, k, v, g and [N, H] for beta.

Distributions follow the five workload descriptions of the KDA mixing step
(64 heads x 128, chunk 64):  q, k, v ~ N(0, 1); conv taps ~ N(0, variance 1/4);
g = -5 * sigmoid(N(0, 1)); beta = sigmoid(N(0, 1)); states ~ N(0, std 0.02);
conv history ~ N(0, 1).  The long-context workload draws g near the -5 floor
(-5 + 0.1 U(0,1)) on a seeded 10 % of (head, key channel) pairs and near zero
(-0.05 U(0,1)) elsewhere.  Values are drawn in fp32 and rounded to bf16
(round-to-nearest-even) where the workload is bf16.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

D_HEAD = 128
BASE_SEED = 20261202
_BLOCK = 1 << 22  # elements per independently seeded block

# stream ids: each tensor draws from its own substream
_Q, _K, _V, _G, _BETA, _CONVW, _STATE, _CONV, _GSEL, _GU, _LEN, _ACC, _Z, _NW = range(1, 15)


def _mix(seed: int, stream: int, block: int) -> int:
    """splitmix64 finaliser over (seed, stream, block) -> a 63-bit torch seed."""
    z = (seed * 0x9E3779B97F4A7C15 + stream * 0xBF58476D1CE4E5B9 + block * 0x94D049BB133111EB) & (2**64 - 1)
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & (2**64 - 1)
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & (2**64 - 1)
    z ^= z >> 31
    return z & (2**63 - 1)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _draw(shape, seed: int, stream: int, kind: str, dtype: torch.dtype = torch.float32,
          scale: float = 1.0, fn=None) -> torch.Tensor:
    """Tensor of N(0,1) ('n') or U[0,1) ('u') draws, optionally mapped by
    fn(x, first_index), then scaled; generated in fp32 blocks with their own
    seeds (the result does not depend on the thread count) and stored as
    `dtype` (round-to-nearest-even for bf16) block by block."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(n, dtype=dtype)
    nblocks = (n + _BLOCK - 1) // _BLOCK

    def fill(b: int) -> None:
        gen = torch.Generator().manual_seed(_mix(seed, stream, b))
        lo, hi = b * _BLOCK, min(n, (b + 1) * _BLOCK)
        x = torch.randn(hi - lo, generator=gen) if kind == "n" else torch.rand(hi - lo, generator=gen)
        if fn is not None:
            x = fn(x, lo)
        if scale != 1.0:
            x = x * scale
        out[lo:hi] = x

    if nblocks <= 1:
        for b in range(nblocks):
            fill(b)
    else:
        with ThreadPoolExecutor(max_workers=_threads()) as ex:
            list(ex.map(fill, range(nblocks)))
    return out.view(*shape)


def randn(shape, seed: int, stream: int, std: float = 1.0,
          dtype: torch.dtype = torch.float32) -> torch.Tensor:
    return _draw(shape, seed, stream, "n", dtype, std)


def rand(shape, seed: int, stream: int) -> torch.Tensor:
    return _draw(shape, seed, stream, "u")


def _sigmoid(x: torch.Tensor, lo: int) -> torch.Tensor:
    return torch.sigmoid(x)


def _neg5_sigmoid(x: torch.Tensor, lo: int) -> torch.Tensor:
    return torch.sigmoid(x).mul_(-5.0)


@dataclasses.dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    conv_w: torch.Tensor
    init_state: Optional[torch.Tensor]
    init_conv: Optional[torch.Tensor]
    cu_seqlens: np.ndarray  # int32 [N+1]
    name: str = ""

    @property
    def num_seqs(self) -> int:
        return len(self.cu_seqlens) - 1

    @property
    def num_heads(self) -> int:
        return self.q.shape[1]

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def dtype(self) -> torch.dtype:
        return self.q.dtype


@dataclasses.dataclass
class DecodeInputs:
    state: torch.Tensor      # [N, H, D, D] fp32
    conv_cache: torch.Tensor  # [N, 3, 3, H*D]
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    conv_w: torch.Tensor
    name: str = ""

    @property
    def num_seqs(self) -> int:
        return self.q.shape[0]

    @property
    def num_heads(self) -> int:
        return self.q.shape[1]

    @property
    def dtype(self) -> torch.dtype:
        return self.q.dtype


def gate_sigmoid(shape, seed: int, dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """g = -5 * sigmoid(N(0,1))."""
    return _draw(shape, seed, _G, "n", dtype, fn=_neg5_sigmoid)


def gate_bimodal(total_t: int, H: int, D: int, seed: int, frac: float = 0.1,
                 dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """Long-context gate mix: a seeded `frac` of (head, key channel) pairs get
    g = -5 + 0.1 U(0,1) for every token, the rest g = -0.05 U(0,1)."""
    rng = np.random.default_rng(_mix(seed, _GSEL, 0))
    HD = H * D
    nsel = int(round(frac * HD))
    sel = np.zeros(HD, dtype=bool)
    sel[rng.permutation(HD)[:nsel]] = True
    sel_t = torch.from_numpy(sel)

    def mix(u: torch.Tensor, lo: int) -> torch.Tensor:
        chan = (torch.arange(lo, lo + u.numel(), dtype=torch.int64) % HD)
        return torch.where(sel_t[chan], -5.0 + 0.1 * u, -0.05 * u)

    return _draw((total_t, H, D), seed, _GU, "u", dtype, fn=mix)


def make_prefill(seqlens: Sequence[int], H: int, dtype: torch.dtype, seed: int, *,
                 D: int = D_HEAD, gate: str = "sigmoid", state_std: Optional[float] = None,
                 conv_history: bool = False, name: str = "") -> PrefillInputs:
    seqlens = [int(s) for s in seqlens]
    N = len(seqlens)
    cu = np.zeros(N + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    T = int(cu[-1])
    q = randn((T, H, D), seed, _Q, dtype=dtype)
    k = randn((T, H, D), seed, _K, dtype=dtype)
    v = randn((T, H, D), seed, _V, dtype=dtype)
    if gate == "sigmoid":
        g = gate_sigmoid((T, H, D), seed, dtype)
    elif gate == "bimodal":
        g = gate_bimodal(T, H, D, seed, dtype=dtype)
    else:
        raise ValueError(gate)
    beta = _draw((T, H), seed, _BETA, "n", dtype, fn=_sigmoid)
    conv_w = randn((3, H * D, 4), seed, _CONVW, std=0.5)
    init_state = randn((N, H, D, D), seed, _STATE, std=state_std) if state_std else None
    init_conv = randn((N, 3, 3, H * D), seed, _CONV, dtype=dtype) if conv_history else None
    return PrefillInputs(q, k, v, g, beta, conv_w, init_state, init_conv, cu, name)


def make_decode(N: int, H: int, dtype: torch.dtype, seed: int, *, D: int = D_HEAD,
                state_std: float = 0.02, name: str = "") -> DecodeInputs:
    state = randn((N, H, D, D), seed, _STATE, std=state_std)
    conv_cache = randn((N, 3, 3, H * D), seed, _CONV, dtype=dtype)
    q = randn((N, H, D), seed, _Q, dtype=dtype)
    k = randn((N, H, D), seed, _K, dtype=dtype)
    v = randn((N, H, D), seed, _V, dtype=dtype)
    g = gate_sigmoid((N, H, D), seed, dtype)
    beta = _draw((N, H), seed, _BETA, "n", dtype, fn=_sigmoid)
    conv_w = randn((3, H * D, 4), seed, _CONVW, std=0.5)
    return DecodeInputs(state, conv_cache, q, k, v, g, beta, conv_w, name)


@dataclasses.dataclass
class DecodeRowsInputs:
    """R new rows per sequence for a multi-token (verify / commit) decode step,
    with the number of rows each sequence keeps."""
    state: torch.Tensor       # [N, H, D, D] fp32
    conv_cache: torch.Tensor  # [N, 3, 3, H*D]
    q: torch.Tensor           # [N, R, H, D]
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor        # [N, R, H]
    conv_w: torch.Tensor
    n_accept: np.ndarray      # int32 [N], each in [0, R]
    name: str = ""

    @property
    def num_seqs(self) -> int:
        return self.q.shape[0]

    @property
    def num_rows(self) -> int:
        return self.q.shape[1]

    @property
    def num_heads(self) -> int:
        return self.q.shape[2]


def make_decode_rows(N: int, R: int, H: int, dtype: torch.dtype, seed: int, *, D: int = D_HEAD,
                     state_std: float = 0.02, accept: Tuple[int, int] = (0, -1),
                     name: str = "") -> DecodeRowsInputs:
    """Distributions as the single-token decode workload; n_accept uniform on
    the integers [accept[0], accept[1]] (accept[1] = -1 means R)."""
    state = randn((N, H, D, D), seed, _STATE, std=state_std)
    conv_cache = randn((N, 3, 3, H * D), seed, _CONV, dtype=dtype)
    q = randn((N, R, H, D), seed, _Q, dtype=dtype)
    k = randn((N, R, H, D), seed, _K, dtype=dtype)
    v = randn((N, R, H, D), seed, _V, dtype=dtype)
    g = gate_sigmoid((N, R, H, D), seed, dtype)
    beta = _draw((N, R, H), seed, _BETA, "n", dtype, fn=_sigmoid)
    conv_w = randn((3, H * D, 4), seed, _CONVW, std=0.5)
    lo, hi = accept[0], (R if accept[1] < 0 else accept[1])
    rng = np.random.default_rng(_mix(seed, _ACC, 0))
    n_accept = rng.integers(lo, hi, size=N, endpoint=True).astype(np.int32)
    return DecodeRowsInputs(state, conv_cache, q, k, v, g, beta, conv_w, n_accept, name)


def varlen_lengths(seed: int, n: int = 16, lo: int = 1024, hi: int = 32768) -> List[int]:
    rng = np.random.default_rng(_mix(seed, _LEN, 0))
    return [int(x) for x in rng.integers(lo, hi, size=n, endpoint=True)]


# The five workloads of the KDA mixing step.  Index i uses seed BASE_SEED + i.
WORKLOADS = {
    0: "KDA tiny fp32: 1 x T=256, 2 heads x 128, chunk 64",
    1: "KDA prefill bf16: 4 x T=4096, 64 heads x 128, fp32 init state, conv history",
    2: "KDA long-context prefill bf16: 1 x T=65536, 64 heads x 128, bimodal gates",
    3: "KDA varlen packed prefill bf16: 16 x T~U[1024,32768], 64 heads x 128",
    4: "KDA decode step bf16: 256 sequences x 1 token, 64 heads x 128, fp32 states",
}


def workload(i: int, heads: Optional[int] = None):
    """Inputs of workload i (0..4).  `heads` overrides the head count (used to
    build reduced cases with the same per-head statistics)."""
    seed = BASE_SEED + i
    if i == 0:
        return make_prefill([256], heads or 2, torch.float32, seed, name="tiny_fp32")
    if i == 1:
        return make_prefill([4096] * 4, heads or 64, torch.bfloat16, seed, state_std=0.02,
                            conv_history=True, name="prefill_bf16_4x4096")
    if i == 2:
        return make_prefill([65536], heads or 64, torch.bfloat16, seed, gate="bimodal",
                            name="longctx_bf16_65536")
    if i == 3:
        return make_prefill(varlen_lengths(seed), heads or 64, torch.bfloat16, seed,
                            state_std=0.02, name="varlen_bf16_16seq")
    if i == 4:
        return make_decode(256, heads or 64, torch.bfloat16, seed, name="decode_bf16_256")
    raise ValueError(i)


def make_output_norm(rows: int, H: int, seed: int, D: int = D_HEAD):
    """Synthetic inputs of the output epilogue (no trained weights exist here):
    the gate z [rows, H, D] bf16 ~ N(0, 2^2), as logits of a sigmoid gate that
    spans closed to open; the norm weight w [D] fp32 ~ 1 + 0.25 N(0, 1)."""
    z = randn((rows, H, D), seed, _Z, std=2.0, dtype=torch.bfloat16)
    w = 1.0 + randn((D,), seed, _NW, std=0.25)
    return z, w
