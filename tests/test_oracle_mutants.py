"""The oracle's pins catch plausible mistakes.  Each case plants one mistake in
a copy of the oracle's C source (a dropped term, a wrong sign, a wrong operand,
a transposed index, a reversed order, a wrong rounding), builds it into a
library of its own, lets the oracle run on that library, and requires at least
one pin of test_oracle_pins.py to fail.  The oracle itself is not modified;
every planted change keeps all memory accesses in bounds."""
import ctypes
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

# name -> (text in the oracle's C source, its replacement); each text occurs once
MUTANTS = {
    "delta with the wrong sign": ("(vv[j] - r[j])", "(vv[j] + r[j])"),
    "beta dropped from the write": ("+= b * kh[i] * (vv[j] - r[j])", "+= kh[i] * (vv[j] - r[j])"),
    "decay not applied": ("S[i * dv + j] *= al[i];", "S[i * dv + j] *= 1.0;"),
    "readout of the transposed state": ("ot[j] += S[i * dv + j] * qh[i];",
                                        "ot[j] += S[(dk == dv ? j * dv + i : i * dv + j)] * qh[i];"),
    "readout with k instead of q": ("ot[j] += S[i * dv + j] * qh[i];", "ot[j] += S[i * dv + j] * kh[i];"),
    "removal with q instead of k": ("r[j] += S[i * dv + j] * kh[i];", "r[j] += S[i * dv + j] * qh[i];"),
    "conv taps reversed": ("y += w[c * 4 + j] * xs;", "y += w[c * 4 + (3 - j)] * xs;"),
    "conv history reversed": ("xs = hist ? hist[(3 + s) * d + c] : 0.0;",
                              "xs = hist ? hist[(-1 - s) * d + c] : 0.0;"),
    "log-decay floor dropped": ("if (gc < KDA_ORACLE_LOG_DECAY_FLOOR) gc = KDA_ORACLE_LOG_DECAY_FLOOR;", ";"),
    "q not normalised": ("qh[c] *= nq;", "qh[c] *= 1.0;"),
    "norm without the square root": ("nk = 1.0 / sqrt(nk + KDA_ORACLE_NORM_EPS);",
                                     "nk = 1.0 / (nk + KDA_ORACLE_NORM_EPS);"),
    "SiLU with the sigmoid of -y": ("y = y / (1.0 + exp(-y));", "y = y / (1.0 + exp(y));"),
    "SiLU without the factor y": ("y = y / (1.0 + exp(-y));", "y = 1.0 / (1.0 + exp(-y));"),
    "bf16 storage truncates": ("ldexp(nearbyint(ldexp(x, shift)), -shift)", "ldexp(floor(ldexp(x, shift)), -shift)"),
}

# every pin, with arguments for the parametrised ones
PINS = [(f, ()) for name, f in sorted(vars(pins).items())
        if name.startswith("test_") and callable(f)
        and name not in ("test_literal_matrix_form_equals_recurrence", "test_chunked_form_equals_recurrence")]
PINS += [(pins.test_literal_matrix_form_equals_recurrence, a) for a in [(2, 4), (4, 3), (128, 9)]]
PINS += [(pins.test_chunked_form_equals_recurrence, (c,)) for c in (7, 64)]


def _build_mutant(tmp_path, old, new):
    with open(oracle._SRC) as f:
        src = f.read()
    assert src.count(old) == 1, old
    c_path, so_path = tmp_path / "mutant.c", tmp_path / "mutant.so"
    c_path.write_text(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(so_path), str(c_path),
                           "-lm", "-lpthread"])
    lib = ctypes.CDLL(str(so_path))
    lib.kda_oracle_run_jobs.argtypes = [ctypes.POINTER(oracle._Job), ctypes.c_int, ctypes.c_int]
    lib.kda_oracle_run_jobs.restype = ctypes.c_int
    lib.kda_oracle_job_size.restype = ctypes.c_int
    lib.kda_oracle_round_bf16.argtypes = [oracle._dp, oracle._dp, ctypes.c_int64]
    assert lib.kda_oracle_job_size() == ctypes.sizeof(oracle._Job)
    return lib


def _failing_pins():
    failed = []
    for f, args in PINS:
        try:
            f(*args)
        except AssertionError:
            failed.append(f.__name__)
    return failed


def test_unmodified_oracle_passes_every_pin():
    assert _failing_pins() == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    monkeypatch.setattr(oracle, "_lib", _build_mutant(tmp_path, *MUTANTS[name]))
    failed = _failing_pins()
    assert failed, f"no pin catches: {name}"
