"""Planted mistakes: each mutant of the C oracle (a dropped term, a wrong sign,
index or operand) must fail at least one of the pins the real oracle passes.
The mutants are built on the CPU from a text edit of the oracle source."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

MUTANTS = {
    "decay_dropped": ("S[(size_t)i * dv + j] *= a;", "S[(size_t)i * dv + j] *= 1.0;"),
    "decay_wrong_channel": ("const double a = exp(gt[i]);", "const double a = exp(gt[0]);"),
    "erase_sign": ("S[(size_t)i * dv + j] -= bt * kt[i] * p[j];", "S[(size_t)i * dv + j] += bt * kt[i] * p[j];"),
    "erase_no_beta": ("S[(size_t)i * dv + j] -= bt * kt[i] * p[j];", "S[(size_t)i * dv + j] -= kt[i] * p[j];"),
    "readout_uses_k": ("p[j] += qt[i] * S[(size_t)i * dv + j];", "p[j] += kt[i] * S[(size_t)i * dv + j];"),
    "scale_dropped": ("o[(size_t)t * dv + j] = scale * p[j];", "o[(size_t)t * dv + j] = p[j];"),
    "write_no_beta": ("S[(size_t)i * dv + j] += bt * kt[i] * vt[j];", "S[(size_t)i * dv + j] += kt[i] * vt[j];"),
}


def _build(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    p = tmp_path / (name + ".c")
    p.write_text(src.replace(old, new))
    so = tmp_path / (name + ".so")
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", str(so), str(p), "-lm", "-lpthread"])
    lib = ctypes.CDLL(str(so))
    dp = ctypes.POINTER(ctypes.c_double)
    lib.kda_oracle_recurrent.argtypes = [dp] * 8 + [ctypes.c_int] * 5 + [ctypes.c_double] + [ctypes.c_int] * 2
    return lib


def _run(lib, q, k, v, g, beta, h0, scale, erase=1):
    T, dk = q.shape
    dv = v.shape[1]
    o = np.empty((T, dv))
    hT = np.empty((dk, dv))
    arrs = [np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v, g, beta, h0)]
    assert lib.kda_oracle_recurrent(*[a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) for a in arrs],
                                    o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                    hT.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                    1, 1, T, dk, dv, scale, erase, 1) == 0
    return o, hT


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    lib = _build(tmp_path, name, *MUTANTS[name])
    rs = np.random.default_rng(4)
    T, dk, dv = 6, 3, 4
    q = rs.standard_normal((T, dk))
    k = rs.standard_normal((T, dk))
    v = rs.standard_normal((T, dv))
    g = -rs.uniform(0.1, 3, (T, dk))
    beta = rs.uniform(0.1, 0.9, T)
    h0 = rs.standard_normal((dk, dv))
    o_ref, h_ref = oracle.recurrent(q, k, v, g, beta, h0, scale=0.6)
    o_mut, h_mut = _run(lib, q, k, v, g, beta, h0, 0.6)
    # the real oracle passes the brute-force pin (test_oracle.py); the mutant must differ
    assert not (np.allclose(o_mut, o_ref, atol=1e-9) and np.allclose(h_mut, h_ref, atol=1e-9))
