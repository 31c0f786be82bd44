"""fp64 CPU oracle for the KDA sequence-mixing step -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check in ``__graft_entry__`` and the CPU-baseline leg of
``bench.py`` may import or execute anything in this package.  The CUDA library
never calls it and shares no code with it; both sides are fed from
``kda_inputs``.

Three independent evaluations of the same definition (page "GLM-5.3-Flash im
Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit festem Zustand": causal
depthwise conv of width 4 on q/k/v, per-channel forget gate with log-decay floor
-5, scalar-beta delta-rule write, query readout of the updated state):

* ``kda_oracle.c`` -- the token-by-token recurrence in fp64 C (the reference the
  GPU is compared with; threaded over (sequence, head) pairs);
* ``forms.literal_head`` -- the same recurrence with the update matrix
  (I - beta k k^T) Diag(alpha) formed explicitly (numpy, tiny cases);
* ``forms.chunked_head`` -- the chunk-parallel rearrangement (chunk C tokens in
  parallel, state handed from chunk to chunk), fp64 numpy.

Parity status: the recurrence is pinned by closed forms and invariants in
``tests/test_oracle_pins.py`` (beta = 0 pure decay, exact store/recall with
orthonormal keys, last-write recall at beta = 1, linearity, column
permutation, conv impulse response, causality, varlen isolation, split and
decode equivalence, chunked == recurrent, literal == expanded).
``tests/test_oracle_mutants.py`` plants plausible mistakes in a copy of
``kda_oracle.c`` (wrong sign, dropped term, wrong operand, transposed index,
reversed order, wrong rounding) and checks that a pin catches each one.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Iterable, Optional, Tuple

import numpy as np
import torch

from . import epilogue  # noqa: F401  (re-exported)
from . import forms  # noqa: F401  (re-exported)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


class _Job(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("dk", ctypes.c_int),
        ("dv", ctypes.c_int),
        ("q", _dp), ("k", _dp), ("v", _dp), ("g", _dp), ("beta", _dp),
        ("wq", _dp), ("wk", _dp), ("wv", _dp),
        ("init_state", _dp),
        ("cq", _dp), ("ck", _dp), ("cv", _dp),
        ("act", ctypes.c_int),
        ("o", _dp), ("final_state", _dp),
        ("tq", _dp), ("tk", _dp), ("tv", _dp),
        ("state_round", ctypes.c_int),
    ]

# state storage modes of a HeadProblem (how the state is stored, see kda_oracle.c)
STATE_EXACT, STATE_BF16_EACH_TOKEN, STATE_BF16_AT_END = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc into oracle/libkda_oracle.so."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.kda_oracle_run_jobs.argtypes = [ctypes.POINTER(_Job), ctypes.c_int, ctypes.c_int]
        lib.kda_oracle_run_jobs.restype = ctypes.c_int
        lib.kda_oracle_job_size.restype = ctypes.c_int
        lib.kda_oracle_round_bf16.argtypes = [_dp, _dp, ctypes.c_int64]
        assert lib.kda_oracle_job_size() == ctypes.sizeof(_Job), "oracle job struct mismatch"
        _lib = lib
    return _lib


def round_bf16(x) -> np.ndarray:
    """The oracle's state-storage rounding: each double to the nearest bf16
    value, ties to even, without passing through float."""
    a = _f64(x)
    out = np.empty_like(a)
    _load().kda_oracle_round_bf16(_ptr(a), _ptr(out), a.size)
    return out


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.cast(None, _dp)
    return a.ctypes.data_as(_dp)


class HeadProblem:
    """One (sequence, head) problem in fp64: raw q/k/v/g/beta, conv taps,
    initial state and conv history; `run` fills o, final_state and the tails."""

    def __init__(self, q, k, v, g, beta, wq, wk, wv, init_state=None, hist=None, act=0,
                 state_round=STATE_EXACT):
        self.q, self.k, self.v, self.g = _f64(q), _f64(k), _f64(v), _f64(g)
        self.beta = _f64(beta).reshape(-1)
        self.wq, self.wk, self.wv = _f64(wq), _f64(wk), _f64(wv)
        self.T = self.q.shape[0]
        self.dk = self.q.shape[1] if self.q.ndim == 2 and self.T else int(self.wq.shape[0])
        self.dv = self.v.shape[1] if self.v.ndim == 2 and self.T else int(self.wv.shape[0])
        if self.T == 0:
            self.q = np.zeros((0, self.dk)); self.k = np.zeros((0, self.dk))
            self.v = np.zeros((0, self.dv)); self.g = np.zeros((0, self.dk))
        self.init_state = None if init_state is None else _f64(init_state)
        self.hist = None if hist is None else [_f64(h) for h in hist]  # 3 x [3][d]
        self.act = int(act)
        self.state_round = int(state_round)
        self.o = np.zeros((self.T, self.dv))
        self.final_state = np.zeros((self.dk, self.dv))
        self.tail = [np.zeros((3, self.dk)), np.zeros((3, self.dk)), np.zeros((3, self.dv))]

    def job(self) -> _Job:
        h = self.hist
        return _Job(self.T, self.dk, self.dv, _ptr(self.q), _ptr(self.k), _ptr(self.v), _ptr(self.g),
                    _ptr(self.beta), _ptr(self.wq), _ptr(self.wk), _ptr(self.wv), _ptr(self.init_state),
                    _ptr(h[0] if h else None), _ptr(h[1] if h else None), _ptr(h[2] if h else None),
                    self.act, _ptr(self.o), _ptr(self.final_state),
                    _ptr(self.tail[0]), _ptr(self.tail[1]), _ptr(self.tail[2]), self.state_round)


def run_problems(problems, nthreads: Optional[int] = None) -> int:
    """Evaluate HeadProblems in place on up to `nthreads` threads (default: all
    cores).  Returns the thread count used."""
    problems = list(problems)
    if not problems:
        return 0
    lib = _load()
    jobs = (_Job * len(problems))(*[p.job() for p in problems])
    return lib.kda_oracle_run_jobs(jobs, len(problems), int(nthreads or os.cpu_count() or 1))


def prefill_problem(inp, n: int, h: int, act: int = 0, state_round: int = STATE_EXACT) -> HeadProblem:
    """Extract (sequence n, head h) of packed PrefillInputs as a HeadProblem."""
    s0, s1 = int(inp.cu_seqlens[n]), int(inp.cu_seqlens[n + 1])
    D = inp.q.shape[2]
    w = inp.conv_w.view(3, -1, D, 4)[:, h]  # [3][D][4]
    hist = None
    if inp.init_conv is not None:
        c = inp.init_conv.view(inp.num_seqs, 3, 3, -1, D)[n, :, :, h]  # [3 x][3 t][D]
        hist = [c[0], c[1], c[2]]
    st = None if inp.init_state is None else inp.init_state[n, h]
    return HeadProblem(inp.q[s0:s1, h], inp.k[s0:s1, h], inp.v[s0:s1, h], inp.g[s0:s1, h],
                       inp.beta[s0:s1, h], w[0], w[1], w[2], st, hist, act, state_round)


def prefill(inp, pairs: Optional[Iterable[Tuple[int, int]]] = None, act: int = 0,
            nthreads: Optional[int] = None, state_round: int = STATE_EXACT) -> Dict[Tuple[int, int], HeadProblem]:
    """Run the oracle on (sequence, head) pairs of a packed prefill (all pairs
    by default).  Returns {(n, h): solved HeadProblem}."""
    if pairs is None:
        pairs = [(n, h) for n in range(inp.num_seqs) for h in range(inp.num_heads)]
    probs = {p: prefill_problem(inp, p[0], p[1], act, state_round) for p in pairs}
    run_problems(probs.values(), nthreads)
    return probs


def decode_problem(inp, n: int, h: int, act: int = 0, state_round: int = STATE_EXACT) -> HeadProblem:
    D = inp.q.shape[2]
    w = inp.conv_w.view(3, -1, D, 4)[:, h]
    c = inp.conv_cache.view(inp.num_seqs, 3, 3, -1, D)[n, :, :, h]
    return HeadProblem(inp.q[n, h][None], inp.k[n, h][None], inp.v[n, h][None], inp.g[n, h][None],
                       inp.beta[n, h].reshape(1), w[0], w[1], w[2], inp.state[n, h],
                       [c[0], c[1], c[2]], act, state_round)


def decode_rows_problem(inp, n: int, h: int, rows: int, act: int = 0,
                        state_round: int = STATE_EXACT) -> HeadProblem:
    """The first `rows` rows of sequence n, head h of a multi-row decode
    (DecodeRowsInputs), decoded one after another from the sequence's state
    and conv cache: the recurrence with T = rows and the cache as history.  Its
    o holds the outputs of those rows, its final_state and tails the state and
    cache after them."""
    D = inp.q.shape[3]
    w = inp.conv_w.view(3, -1, D, 4)[:, h]
    c = inp.conv_cache.view(inp.num_seqs, 3, 3, -1, D)[n, :, :, h]
    return HeadProblem(inp.q[n, :rows, h], inp.k[n, :rows, h], inp.v[n, :rows, h], inp.g[n, :rows, h],
                       inp.beta[n, :rows, h], w[0], w[1], w[2], inp.state[n, h], [c[0], c[1], c[2]], act,
                       state_round)


def decode(inp, pairs: Optional[Iterable[Tuple[int, int]]] = None, act: int = 0,
           nthreads: Optional[int] = None, state_round: int = STATE_EXACT) -> Dict[Tuple[int, int], HeadProblem]:
    """One decode step = the recurrence with T = 1 and the conv cache as
    history; the updated cache is the problem's tail."""
    if pairs is None:
        pairs = [(n, h) for n in range(inp.num_seqs) for h in range(inp.num_heads)]
    probs = {p: decode_problem(inp, p[0], p[1], act, state_round) for p in pairs}
    run_problems(probs.values(), nthreads)
    return probs
