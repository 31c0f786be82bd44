"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/kda.h declares, and rejects bad arguments on the host before any launch
(fake device addresses are never dereferenced on these paths)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import linear_attention_sequence_kda_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

# distinct, 16-byte aligned fake device addresses
Q, K, V, G, B, W, O, FS, CT, CU, WS = [(i + 1) << 20 for i in range(11)]


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_]+)\s*\(", txt)))


def test_header_declarations_are_exported():
    names = _declared()
    assert set(names) == set(kda.EXPORTS), names
    out = subprocess.run(["nm", "-D", "--defined-only", kda.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for n in names:
        assert n in exported, n
        assert hasattr(kda.lib, n)


def test_version_and_status_strings():
    assert kda.lib.kda_version() >> 16 == 2
    for code in range(7):
        s = kda.lib.kda_status_string(code)
        assert s and s.decode()
    assert kda.lib.kda_status_string(99).decode() == "unknown status"


def test_inject_fault_host_validation():
    """Arming and clearing the host-side fault is pure host work; an unknown
    kind is rejected."""
    assert kda.lib.kda_inject_fault(7) == 1
    assert kda.lib.kda_inject_fault(-1) == 1
    assert kda.lib.kda_inject_fault(kda.KDA_FAULT_DROP_READY) == 0
    assert kda.lib.kda_inject_fault(kda.KDA_FAULT_NONE) == 0


def test_workspace_size_invalid_is_zero():
    assert kda.lib.kda_prefill_workspace_size(-1, 10, 4, 10, 1) == 0
    assert kda.lib.kda_prefill_workspace_size(1, 10, 0, 10, 1) == 0
    assert kda.lib.kda_prefill_workspace_size(1, 10, 4, 10, 0) == 0  # fp32 path needs none


def _prefill(cu, H=4, dt=1, act=0, q=Q, o=O, final=FS, tail=CT, ws=WS, wsb=1 << 40, beta=B,
             recurrent=False, odt=0, sdt=0):
    cu = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
    args = [q, K, V, G, beta, W, None, None, CU, cu.ctypes.data, len(cu) - 1, H, dt, act, odt, sdt, o, final,
            tail]
    if recurrent:
        return kda.lib.kda_prefill_recurrent(*args, None)
    return kda.lib.kda_prefill(*args, ws, wsb, None)


@pytest.mark.parametrize("recurrent", [False, True])
def test_prefill_argument_validation(recurrent):
    p = lambda *a, **kw: _prefill(*a, recurrent=recurrent, **kw)  # noqa: E731
    assert p([0, 5], H=0) == 1
    assert p([0, 5], dt=7) == 1
    assert p([0, 5], act=5) == 1
    assert p([0, 5], odt=3) == 1
    assert p([0, 5], sdt=2) == 1   # state element type
    assert p([1, 5]) == 1          # cu[0] != 0
    assert p([0, 5, 3]) == 1       # decreasing offsets
    assert p([0, 5], q=Q + 2) == 3  # misaligned
    assert p([0, 5], beta=B + 1) == 3
    assert p([0, 5], final=None) == 1
    assert p([0, 5], tail=None) == 1
    assert p([0, 5], q=None) == 1
    assert p([0, 5], o=Q) == 1     # output aliases an input
    assert p([0] * 70001) == 2     # more segments than the grid allows
    assert p([0]) == 0             # no segments: nothing to do, no launch


def test_prefill_workspace_check():
    need = kda.lib.kda_prefill_workspace_size(2, 10, 4, 5, 1)
    if need == 0:
        pytest.skip("the bf16 path needs no workspace")
    assert _prefill([0, 5, 10], ws=None, wsb=0) == 4
    assert _prefill([0, 5, 10], wsb=need - 1) == 4
    assert _prefill([0, 5, 10], ws=WS + 8) == 3


ZG, NW = 12 << 20, 13 << 20  # gate and norm weight


def _gated(cu, dt=1, odt=1, gate=ZG, nw=NW, eps=1e-6, o=O, **kw):
    cu = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
    args = [Q, K, V, G, B, W, None, None, CU, cu.ctypes.data, len(cu) - 1, 4, dt, 0, odt, 0, o, FS, CT]
    return kda.lib.kda_prefill_gated(*args, WS, 1 << 40, gate, nw, eps, None)


def test_prefill_gated_argument_validation():
    """The fused epilogue writes bf16 and needs a gate and a weight; fp32
    inputs have no fused epilogue.  Every case returns before any launch."""
    assert _gated([0, 5], odt=0) == 1           # fp32 output
    assert _gated([0, 5], gate=None) == 1
    assert _gated([0, 5], nw=None) == 1
    assert _gated([0, 5], eps=-1.0) == 1
    assert _gated([0, 5], eps=float("nan")) == 1
    assert _gated([0, 5], eps=float("inf")) == 1
    assert _gated([0, 5], gate=O) == 1          # gate aliases the output
    assert _gated([0, 5], gate=ZG + 8) == 3     # misaligned
    assert _gated([0, 5], nw=NW + 4) == 3
    assert _gated([0, 5], dt=0) == 2            # fp32 inputs: recurrent path, no fused epilogue
    assert _gated([1, 5]) == 1                  # the prefill checks still apply
    assert _gated([0]) == 0                     # no segments: nothing to do


def test_output_norm_argument_validation():
    f = kda.lib.kda_output_norm
    assert f(O, 1, ZG, NW, 1e-6, O, 0, 4, None) == 0        # no rows: nothing enqueued
    assert f(O, 1, ZG, NW, 1e-6, O, -1, 4, None) == 1
    assert f(O, 1, ZG, NW, 1e-6, O, 5, 0, None) == 1
    assert f(O, 5, ZG, NW, 1e-6, O, 5, 4, None) == 1        # bad dtype
    assert f(O, 1, ZG, None, 1e-6, O, 5, 4, None) == 1
    assert f(O, 1, ZG, NW, -1.0, O, 5, 4, None) == 1
    assert f(None, 1, ZG, NW, 1e-6, O, 5, 4, None) == 1
    assert f(O, 1, ZG, NW, 1e-6, ZG, 5, 4, None) == 1       # y aliases the gate
    assert f(O, 0, ZG, NW, 1e-6, O, 5, 4, None) == 1        # in place needs a bf16 o
    assert f(O + 8, 1, ZG, NW, 1e-6, Q, 5, 4, None) == 3


def test_decode_argument_validation():
    d = kda.lib.kda_decode_step
    assert d(FS, CT, Q, K, V, G, B, W, 4, 0, 1, 0, 0, 0, O, None) == 1
    assert d(FS, CT, Q, K, V, G, B, W, 4, 2, 3, 0, 0, 0, O, None) == 1
    assert d(FS, CT, Q, K, V, G, B, W, 4, 2, 1, 9, 0, 0, O, None) == 1
    assert d(FS, CT, Q, K, V, G, B, W, 4, 2, 1, 0, 5, 0, O, None) == 1
    assert d(FS + 4, CT, Q, K, V, G, B, W, 4, 2, 1, 0, 0, 0, O, None) == 3
    assert d(FS, CT, Q, K, V, G, B + 1, W, 4, 2, 1, 0, 0, 0, O, None) == 3
    assert d(None, CT, Q, K, V, G, B, W, 4, 2, 1, 0, 0, 0, O, None) == 1
    assert d(FS, CT, Q, K, V, G, B, W, 4, 2, 1, 0, 0, 0, Q, None) == 1
    assert d(FS, CT, Q, K, V, G, B, W, 70000, 2, 1, 0, 0, 0, O, None) == 2
    assert d(FS, CT, Q, K, V, G, B, W, 0, 2, 1, 0, 0, 0, O, None) == 0
    assert d(FS, CT, Q, K, V, G, B, W, 4, 2, 1, 0, 0, 2, O, None) == 1  # state element type


DL, NA = 12 << 20, 13 << 20  # fake deltas and n_accept addresses


def test_decode_rows_argument_validation():
    assert kda.lib.kda_decode_deltas_size(4, 6, 2) == 4 * 2 * 6 * 3 * 128 * 4
    assert kda.lib.kda_decode_deltas_size(4, 0, 2) == 0
    assert kda.lib.kda_decode_deltas_size(4, kda.MAX_VERIFY_ROWS + 1, 2) == 0
    vf = kda.lib.kda_decode_verify
    #      state CT Q K V G B W  N  R  H dt act odt sdt o  deltas
    assert vf(None, CT, Q, K, V, G, B, W, 4, 6, 2, 1, 0, 0, 0, O, DL, None) == 1
    assert vf(FS, CT, Q, K, V, G, B, W, 4, 0, 2, 1, 0, 0, 0, O, DL, None) == 1
    assert vf(FS, CT, Q, K, V, G, B, W, 4, 9, 2, 1, 0, 0, 0, O, DL, None) == 1
    assert vf(FS, CT, Q, K, V, G, B, W, 4, 6, 0, 1, 0, 0, 0, O, DL, None) == 1
    assert vf(FS, CT, Q, K, V, G, B, W, 4, 6, 2, 3, 0, 0, 0, O, DL, None) == 1
    assert vf(FS, CT, Q, K, V, G, B, W, 4, 6, 2, 1, 0, 0, 0, O, None, None) == 1
    assert vf(FS, CT, Q, K, V, G, B, W, 4, 6, 2, 1, 0, 0, 0, O, DL + 8, None) == 3
    assert vf(FS, CT, Q, K, V, G, B + 1, W, 4, 6, 2, 1, 0, 0, 0, O, DL, None) == 3
    assert vf(FS, CT, Q, K, V, G, B, W, 4, 6, 2, 1, 0, 0, 0, Q, DL, None) == 1
    assert vf(FS, CT, Q, K, V, G, B, W, 70000, 6, 2, 1, 0, 0, 0, O, DL, None) == 2
    assert vf(FS, CT, Q, K, V, G, B, W, 0, 6, 2, 1, 0, 0, 0, O, DL, None) == 0
    assert vf(FS, CT, Q, K, V, G, B, W, 4, 6, 2, 1, 0, 0, 5, O, DL, None) == 1
    cm = kda.lib.kda_decode_commit
    #      state CT Q K V deltas n_acc N R H dt sdt
    assert cm(FS, CT, Q, K, V, DL, NA, 4, 0, 2, 1, 0, None) == 1
    assert cm(FS, CT, Q, K, V, DL, NA, 4, 6, 2, 7, 0, None) == 1
    assert cm(FS, CT, Q, K, V, None, NA, 4, 6, 2, 1, 0, None) == 1
    assert cm(FS, CT, Q, K, V, DL, None, 4, 6, 2, 1, 0, None) == 1
    assert cm(FS, CT, Q, K, V, DL, NA + 2, 4, 6, 2, 1, 0, None) == 3
    assert cm(FS + 4, CT, Q, K, V, DL, NA, 4, 6, 2, 1, 0, None) == 3
    assert cm(FS, CT, Q, K, V, DL, NA, 70000, 6, 2, 1, 0, None) == 2
    assert cm(FS, CT, Q, K, V, DL, NA, 0, 6, 2, 1, 0, None) == 0
    assert cm(FS, CT, Q, K, V, DL, NA, 4, 6, 2, 1, 3, None) == 1


def test_commit_verify_argument_validation():
    cv = kda.lib.kda_decode_commit_verify
    PQ, PK, PV, PD = 14 << 20, 15 << 20, 16 << 20, 17 << 20
    size = kda.lib.kda_decode_deltas_size(4, 6, 2)

    def call(state=FS, pq=PQ, pdl=PD, na=NA, prows=6, rows=6, deltas=DL, sdt=0, n=4):
        #         state CT  prev q k v  deltas  n_acc prows  Q K V G B W  N rows H dt act odt sdt o deltas
        return cv(state, CT, pq, PK, PV, pdl, na, prows, Q, K, V, G, B, W, n, rows, 2, 1, 0, 0, sdt, O, deltas, None)

    assert call(n=0) == 0
    assert call(prows=0) == 1 and call(prows=kda.MAX_VERIFY_ROWS + 1) == 1
    assert call(rows=0) == 1
    assert call(pq=None) == 1 and call(pdl=None) == 1 and call(na=None) == 1
    assert call(na=NA + 2) == 3 and call(pq=PQ + 4) == 3
    assert call(sdt=4) == 1
    assert call(deltas=PD) == 1                        # the same buffer
    assert call(deltas=PD + size - 16) == 1            # overlapping ranges
    assert call(deltas=PD - size + 16) == 1
    assert call(n=70000) == 2


def test_state_affine_argument_validation():
    af = kda.lib.kda_state_affine
    Aa, Ss, Bb, So = 20 << 20, 21 << 20, 22 << 20, 23 << 20
    assert af(Aa, Ss, Bb, So, 0, 0, None) == 0          # nothing to do
    assert af(Aa, Ss, Bb, So, -1, 0, None) == 1
    assert af(None, Ss, Bb, So, 4, 0, None) == 1
    assert af(Aa, Ss, Bb, So, 4, 3, None) == 1          # state element type
    assert af(Aa, Ss, Bb, Aa, 4, 0, None) == 1          # output aliases A
    assert af(Aa + 4, Ss, Bb, So, 4, 0, None) == 3


def test_binding_constants_match_the_header():
    """The binding's copies of the header's constants and enum values."""
    txt = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    defines = dict(re.findall(r"#define\s+(KDA_[A-Z_]+)\s+(\d+)\s*$", txt, flags=re.M))
    assert int(defines["KDA_HEAD_DIM"]) == kda.HEAD_DIM
    assert int(defines["KDA_CHUNK"]) == kda.CHUNK
    assert int(defines["KDA_MAX_VERIFY_ROWS"]) == kda.MAX_VERIFY_ROWS
    m = re.search(r"#define\s+KDA_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", txt)
    assert m and int(m.group(1)) << int(m.group(2)) == kda.NOALLOC_SCRATCH_BYTES
    enums = {name: int(v) for name, v in re.findall(r"\b(KDA_[A-Z0-9_]+)\s*=\s*(\d+)", txt)}
    statuses = {k: v for k, v in enums.items() if k == "KDA_OK" or k.startswith("KDA_ERR_")}
    assert {name: code for code, name in kda.STATUS.items()} == statuses
    assert (enums["KDA_F32"], enums["KDA_BF16"]) == (kda.KDA_F32, kda.KDA_BF16)
    assert (enums["KDA_CONV_NONE"], enums["KDA_CONV_SILU"]) == (kda.KDA_CONV_NONE, kda.KDA_CONV_SILU)
    assert (enums["KDA_FAULT_NONE"], enums["KDA_FAULT_DROP_READY"]) == \
        (kda.KDA_FAULT_NONE, kda.KDA_FAULT_DROP_READY)
