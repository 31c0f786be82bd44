"""Python binding of libkda.so (the B200 KDA sequence-mixing library).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI of ``include/kda.h``.  PyTorch is used for device
memory, streams and dtype plumbing.  If ``libkda.so`` has not been built the
import fails loudly; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda.so")
HEAD_DIM = 128
CHUNK = 64

KDA_F32, KDA_BF16 = 0, 1
KDA_CONV_NONE, KDA_CONV_SILU = 0, 1
STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_ALIGNMENT",
          4: "KDA_ERR_WORKSPACE", 5: "KDA_ERR_CUDA", 6: "KDA_ERR_TIMEOUT"}

# every entry point declared in include/kda.h
EXPORTS = ("kda_prefill_workspace_size", "kda_prefill", "kda_prefill_recurrent",
           "kda_decode_step", "kda_status_string", "kda_check_async_status", "kda_version",
           "kda_prefill_noalloc", "kda_decode_deltas_size", "kda_decode_verify", "kda_decode_commit",
           "kda_decode_commit_verify", "kda_state_affine", "kda_inject_fault", "kda_last_cuda_error",
           "kda_prefill_gated", "kda_output_norm", "kda_prefill_records", "kda_prefill_scan")
MAX_VERIFY_ROWS = 8  # KDA_MAX_VERIFY_ROWS

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python "
                      "linear_attention_sequence_kda_b200/build.py` (nvcc, sm_100a)")

_vp, _i32p, _f32p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
lib = ctypes.CDLL(LIB_PATH)
lib.kda_last_cuda_error.restype = ctypes.c_int
lib.kda_last_cuda_error.argtypes = []
lib.kda_prefill_workspace_size.restype = ctypes.c_size_t
lib.kda_prefill_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int]
_PREFILL_ARGS = [_vp, _vp, _vp, _vp, _vp, _f32p, _vp, _vp, _i32p, _i32p, ctypes.c_int, ctypes.c_int,
                 ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp]
lib.kda_prefill.restype = ctypes.c_int
lib.kda_prefill.argtypes = _PREFILL_ARGS + [_vp, ctypes.c_size_t, _vp]
for _name in ("kda_prefill_records", "kda_prefill_scan"):
    getattr(lib, _name).restype = ctypes.c_int
    getattr(lib, _name).argtypes = _PREFILL_ARGS + [_vp, ctypes.c_size_t, _vp]
lib.kda_prefill_recurrent.restype = ctypes.c_int
lib.kda_prefill_recurrent.argtypes = _PREFILL_ARGS + [_vp]
lib.kda_prefill_gated.restype = ctypes.c_int
lib.kda_prefill_gated.argtypes = _PREFILL_ARGS + [_vp, ctypes.c_size_t, _vp, _f32p, ctypes.c_float, _vp]
lib.kda_output_norm.restype = ctypes.c_int
lib.kda_output_norm.argtypes = [_vp, ctypes.c_int, _vp, _f32p, ctypes.c_float, _vp, ctypes.c_int64, ctypes.c_int,
                                _vp]
lib.kda_prefill_noalloc.restype = ctypes.c_int
lib.kda_prefill_noalloc.argtypes = _PREFILL_ARGS + [_vp]
NOALLOC_SCRATCH_BYTES = 128 << 20  # KDA_NOALLOC_SCRATCH_BYTES
lib.kda_decode_step.restype = ctypes.c_int
lib.kda_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _f32p, ctypes.c_int, ctypes.c_int,
                                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp]
lib.kda_decode_deltas_size.restype = ctypes.c_size_t
lib.kda_decode_deltas_size.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
lib.kda_decode_verify.restype = ctypes.c_int
lib.kda_decode_verify.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _f32p, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _f32p,
                                  _vp]
lib.kda_decode_commit.restype = ctypes.c_int
lib.kda_decode_commit.argtypes = [_vp, _vp, _vp, _vp, _vp, _f32p, _i32p, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp]
lib.kda_decode_commit_verify.restype = ctypes.c_int
lib.kda_decode_commit_verify.argtypes = [_vp, _vp, _vp, _vp, _vp, _f32p, _i32p, ctypes.c_int, _vp, _vp, _vp, _vp,
                                         _vp, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _f32p, _vp]
lib.kda_state_affine.restype = ctypes.c_int
lib.kda_state_affine.argtypes = [_f32p, _vp, _f32p, _vp, ctypes.c_int, ctypes.c_int, _vp]
lib.kda_status_string.restype = ctypes.c_char_p
lib.kda_status_string.argtypes = [ctypes.c_int]
lib.kda_check_async_status.restype = ctypes.c_int
lib.kda_check_async_status.argtypes = [_vp]
lib.kda_version.restype = ctypes.c_int
lib.kda_inject_fault.restype = ctypes.c_int
lib.kda_inject_fault.argtypes = [ctypes.c_int]
KDA_FAULT_NONE, KDA_FAULT_DROP_READY = 0, 1


class KdaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {STATUS.get(code, code)} ({lib.kda_status_string(code).decode()})"
        if code == 5:  # KDA_ERR_CUDA: name the CUDA runtime error behind it
            self.cuda_error = int(lib.kda_last_cuda_error())
            msg += f" [cudaError_t {self.cuda_error}]"
        super().__init__(msg)


def _check(code: int, where: str) -> None:
    if code != 0:
        raise KdaError(code, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream if isinstance(stream, int) else stream.cuda_stream


def workspace_size(num_seqs: int, total_tokens: int, num_heads: int, max_seqlen: int,
                   dtype: torch.dtype = torch.bfloat16) -> int:
    return int(lib.kda_prefill_workspace_size(num_seqs, total_tokens, num_heads, max_seqlen,
                                              KDA_F32 if dtype == torch.float32 else KDA_BF16))


def _state_code(final_state, init_state) -> int:
    """state_dt of a call: the element type of its state tensors (which agree)."""
    if init_state is not None and init_state.dtype != final_state.dtype:
        raise ValueError("init_state and final_state must have the same element type")
    return _dtype_code(final_state)


def prefill(q, k, v, g, beta, conv_w, cu_seqlens_host, cu_seqlens_dev=None, init_state=None,
            init_conv=None, act: int = KDA_CONV_NONE, o=None, final_state=None, conv_tail=None,
            workspace=None, stream=None, recurrent: bool = False, o_dtype=torch.float32,
            state_dtype=None, gate=None, norm_weight=None, norm_eps: float = 1e-6, mode: str = "full"):
    """kda_prefill (or kda_prefill_recurrent) on device tensors.  Returns
    (o, final_state, conv_tail); outputs are allocated when not given (o in
    `o_dtype`, fp32 by default; the final state in `state_dtype`, default the
    init state's type, else fp32).  The state element type of the call is that
    of final_state.  With `gate` ([T, H, 128] bf16) and `norm_weight` ([128]
    fp32) the call is kda_prefill_gated: o holds the gated RMS-normalised
    output, in bf16.  `mode` "records" calls kda_prefill_records (the chunk
    records stay valid in `workspace`), "scan" kda_prefill_scan (the scan over
    records a "records" call left in `workspace`; see include/kda.h)."""
    if mode not in ("full", "records", "scan"):
        raise ValueError(f"unknown prefill mode {mode!r}")
    if mode != "full" and (recurrent or gate is not None):
        raise ValueError("record-keeping and scan-only calls run the plain chunked path")
    if mode == "scan" and workspace is None:
        raise ValueError("a scan-only call reads the records of an earlier call from its workspace")
    if gate is not None:
        if recurrent:
            raise ValueError("the fused output epilogue runs on the chunked path only")
        o_dtype = torch.bfloat16
    cu_h = np.ascontiguousarray(np.asarray(cu_seqlens_host, dtype=np.int32))
    N = len(cu_h) - 1
    T, H = q.shape[0], q.shape[1]
    dev = q.device
    if cu_seqlens_dev is None:
        cu_seqlens_dev = torch.from_numpy(cu_h).to(dev)
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype, device=dev)
    if final_state is None:
        sdt = state_dtype or (init_state.dtype if init_state is not None else torch.float32)
        final_state = torch.empty((N, H, HEAD_DIM, HEAD_DIM), dtype=sdt, device=dev)
    if conv_tail is None:
        conv_tail = torch.empty((N, 3, 3, H * HEAD_DIM), dtype=q.dtype, device=dev)
    dt = _dtype_code(q)
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(conv_w), _ptr(init_state),
            _ptr(init_conv), _ptr(cu_seqlens_dev), _ptr(cu_h), N, H, dt, int(act), _dtype_code(o),
            _state_code(final_state, init_state), _ptr(o), _ptr(final_state), _ptr(conv_tail)]
    if recurrent:
        _check(lib.kda_prefill_recurrent(*args, _stream(stream)), "kda_prefill_recurrent")
    else:
        need = workspace_size(N, int(cu_h[-1]), H, int(np.diff(cu_h).max()) if N else 0, q.dtype)
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        if gate is not None:
            _check(lib.kda_prefill_gated(*args, _ptr(workspace), wbytes, _ptr(gate), _ptr(norm_weight),
                                         float(norm_eps), _stream(stream)), "kda_prefill_gated")
        elif mode != "full":
            name = "kda_prefill_records" if mode == "records" else "kda_prefill_scan"
            _check(getattr(lib, name)(*args, _ptr(workspace), wbytes, _stream(stream)), name)
        else:
            _check(lib.kda_prefill(*args, _ptr(workspace), wbytes, _stream(stream)), "kda_prefill")
    return o, final_state, conv_tail


def output_norm(o, gate, norm_weight, norm_eps: float = 1e-6, y=None, stream=None):
    """kda_output_norm: y = o / sqrt(mean o^2 + eps) * norm_weight * sigmoid(gate)
    over each head's 128 channels; o [rows, H, 128] fp32 or bf16, gate bf16,
    y bf16 (allocated when not given; may be o itself when o is bf16)."""
    rows, H = o.shape[0], o.shape[1]
    if y is None:
        y = torch.empty(o.shape, dtype=torch.bfloat16, device=o.device)
    _check(lib.kda_output_norm(_ptr(o), _dtype_code(o), _ptr(gate), _ptr(norm_weight), float(norm_eps),
                               _ptr(y), rows, H, _stream(stream)), "kda_output_norm")
    return y


def prefill_noalloc(q, k, v, g, beta, conv_w, cu_seqlens_host, cu_seqlens_dev=None, init_state=None,
                    init_conv=None, act: int = KDA_CONV_NONE, o=None, final_state=None, conv_tail=None,
                    stream=None, o_dtype=torch.float32, state_dtype=None):
    """kda_prefill_noalloc: like prefill() but the library uses its own static
    device scratch instead of a workspace.  Returns (o, final_state, conv_tail)."""
    cu_h = np.ascontiguousarray(np.asarray(cu_seqlens_host, dtype=np.int32))
    N = len(cu_h) - 1
    H = q.shape[1]
    dev = q.device
    if cu_seqlens_dev is None:
        cu_seqlens_dev = torch.from_numpy(cu_h).to(dev)
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype, device=dev)
    if final_state is None:
        sdt = state_dtype or (init_state.dtype if init_state is not None else torch.float32)
        final_state = torch.empty((N, H, HEAD_DIM, HEAD_DIM), dtype=sdt, device=dev)
    if conv_tail is None:
        conv_tail = torch.empty((N, 3, 3, H * HEAD_DIM), dtype=q.dtype, device=dev)
    _check(lib.kda_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(conv_w),
                                   _ptr(init_state), _ptr(init_conv), _ptr(cu_seqlens_dev), _ptr(cu_h), N, H,
                                   _dtype_code(q), int(act), _dtype_code(o), _state_code(final_state, init_state),
                                   _ptr(o), _ptr(final_state), _ptr(conv_tail), _stream(stream)),
           "kda_prefill_noalloc")
    return o, final_state, conv_tail


def decode_step(state, conv_cache, q, k, v, g, beta, conv_w, act: int = KDA_CONV_NONE, o=None,
                stream=None, o_dtype=torch.float32):
    """kda_decode_step in place on `state` (fp32 or bf16 storage) and
    `conv_cache`; returns o (allocated in `o_dtype` when not given)."""
    N, H = q.shape[0], q.shape[1]
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype, device=q.device)
    _check(lib.kda_decode_step(_ptr(state), _ptr(conv_cache), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                               _ptr(beta), _ptr(conv_w), N, H, _dtype_code(q), int(act), _dtype_code(o),
                               _dtype_code(state), _ptr(o), _stream(stream)), "kda_decode_step")
    return o


def deltas_size(num_seqs: int, num_rows: int, num_heads: int) -> int:
    return int(lib.kda_decode_deltas_size(num_seqs, num_rows, num_heads))


def decode_verify(state, conv_cache, q, k, v, g, beta, conv_w, act: int = KDA_CONV_NONE, o=None,
                  deltas=None, stream=None, o_dtype=torch.float32):
    """kda_decode_verify: rows [N, R, H, 128] decoded in turn from `state` and
    `conv_cache` (neither modified).  Returns (o [N, R, H, 128], deltas)."""
    N, R, H = q.shape[0], q.shape[1], q.shape[2]
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype, device=q.device)
    if deltas is None:
        deltas = torch.empty(deltas_size(N, R, H) // 4, dtype=torch.float32, device=q.device)
    _check(lib.kda_decode_verify(_ptr(state), _ptr(conv_cache), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(conv_w), N, R, H, _dtype_code(q), int(act), _dtype_code(o),
                                 _dtype_code(state), _ptr(o), _ptr(deltas), _stream(stream)), "kda_decode_verify")
    return o, deltas


def decode_commit(state, conv_cache, q, k, v, deltas, n_accept, stream=None):
    """kda_decode_commit: keep the first n_accept[n] verified rows of each
    sequence (n_accept: int32 device tensor [N]); state and conv_cache are
    updated in place."""
    N, R, H = q.shape[0], q.shape[1], q.shape[2]
    _check(lib.kda_decode_commit(_ptr(state), _ptr(conv_cache), _ptr(q), _ptr(k), _ptr(v), _ptr(deltas),
                                 _ptr(n_accept), N, R, H, _dtype_code(q), _dtype_code(state), _stream(stream)),
           "kda_decode_commit")


def decode_commit_verify(state, conv_cache, prev, q, k, v, g, beta, conv_w, act: int = KDA_CONV_NONE, o=None,
                         deltas=None, stream=None, o_dtype=torch.float32):
    """kda_decode_commit_verify: keep the first prev.n_accept[n] rows of the
    previous step (`prev` = (prev_q, prev_k, prev_v, prev_deltas, n_accept) as
    given to and returned by the previous verify), then verify the new rows
    [N, R, H, 128] from the updated state and cache.  Returns (o, deltas);
    `deltas` must not be the previous step's buffer."""
    pq, pk, pv, pdeltas, pn = prev
    N, R, H = q.shape[0], q.shape[1], q.shape[2]
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype, device=q.device)
    if deltas is None:
        deltas = torch.empty(deltas_size(N, R, H) // 4, dtype=torch.float32, device=q.device)
    _check(lib.kda_decode_commit_verify(_ptr(state), _ptr(conv_cache), _ptr(pq), _ptr(pk), _ptr(pv), _ptr(pdeltas),
                                        _ptr(pn), pq.shape[1], _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                        _ptr(conv_w), N, R, H, _dtype_code(q), int(act), _dtype_code(o),
                                        _dtype_code(state), _ptr(o), _ptr(deltas), _stream(stream)),
           "kda_decode_commit_verify")
    return o, deltas


def state_affine(A, S_in, B, S_out=None, stream=None):
    """kda_state_affine: S_out = A S_in + B per (sequence, head); A and B fp32
    [..., 128, 128], S_in in the state storage type (S_out defaults to a new
    tensor of that type; it may be S_in)."""
    if S_out is None:
        S_out = torch.empty_like(S_in)
    count = S_in.numel() // (HEAD_DIM * HEAD_DIM)
    _check(lib.kda_state_affine(_ptr(A), _ptr(S_in), _ptr(B), _ptr(S_out), count, _dtype_code(S_in),
                                _stream(stream)), "kda_state_affine")
    return S_out


def check_async_status(stream=None) -> int:
    return int(lib.kda_check_async_status(_stream(stream)))


def inject_fault(kind: int) -> None:
    """Test hook: arm a host-side fault for the next call that can apply it
    (KDA_FAULT_DROP_READY) or clear a pending one (KDA_FAULT_NONE)."""
    _check(lib.kda_inject_fault(int(kind)), "kda_inject_fault")
