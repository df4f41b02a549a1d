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


# ---- planted mistakes in the fp64 restatements of Eq. 5 and Eq. 6 ----------

def _gate_pins(gate):
    """The checks test_oracle's gate pin makes, against a candidate gate(z, A, g_min)."""
    A = np.array([[0.0, np.log(2.0)], [-1.0, 0.5]])
    z = np.array([[[[1.0, 1.0]], [[-2.0, 3.0]]]])
    ref = -5.0 / (1.0 + np.exp(-np.array([[[1.0, 2.0]], [[-2.0 * np.exp(-1.0), 3.0 * np.exp(0.5)]]])))
    ok = np.allclose(gate(np.zeros((1, 2, 1, 2)), A, -5.0), -2.5, rtol=0, atol=1e-15)
    ok &= np.allclose(gate(z, A, -5.0)[0], ref, rtol=1e-15)
    zz = np.random.default_rng(5).standard_normal((2, 2, 50, 2)) * 3
    gg = gate(zz, A, -5.0)
    ok &= bool(np.all(gg > -5.0) and np.all(gg < 0.0))
    ok &= np.allclose(gate(zz, A, -2.0), gg * 0.4, rtol=1e-14)
    return bool(ok)


GATE_MUTANTS = {
    "no_scale": lambda z, A, gm: gm / (1.0 + np.exp(-np.asarray(z))),
    "scale_not_exponentiated": lambda z, A, gm: gm / (1.0 + np.exp(-np.asarray(A)[:, None, :] * z)),
    "wrong_sigmoid_side": lambda z, A, gm: gm / (1.0 + np.exp(np.exp(np.asarray(A))[:, None, :] * z)),
    "scale_of_channel_0_only": lambda z, A, gm: gm / (1.0 + np.exp(-np.exp(np.asarray(A)[:, None, :1]) * z)),
}


def test_gate_pins_hold_for_the_oracle():
    assert _gate_pins(oracle.gate)


@pytest.mark.parametrize("name", sorted(GATE_MUTANTS))
def test_gate_mutant_is_caught(name):
    assert not _gate_pins(GATE_MUTANTS[name])


def _output_gate_pins(fn):
    o = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    y = fn(o, np.zeros_like(o), np.array([[1.0, 2.0]]), 0.0)
    ok = np.allclose(y.ravel(), [0.5 * 3.0 / np.sqrt(12.5), 0.5 * 2.0 * 4.0 / np.sqrt(12.5)], rtol=1e-15)
    rs = np.random.default_rng(6)
    o = rs.standard_normal((2, 3, 5, 16))
    gate = rs.standard_normal((2, 3, 5, 16))
    w = rs.standard_normal((3, 16))
    y = fn(o, gate, w, 0.0)
    ok &= np.allclose(fn(7.5 * o, gate, w, 0.0), y, rtol=1e-13)
    yy = fn(o, np.full_like(o, 60.0), np.ones((3, 16)), 0.0)
    ok &= np.allclose(np.sqrt(np.mean(yy * yy, axis=-1)), 1.0, rtol=1e-12)
    w2 = w.copy()
    w2[0] *= 3.0
    ok &= np.array_equal(fn(o, gate, w2, 0.0)[:, 1:], y[:, 1:])
    return bool(ok)


def _og(norm, gate_act, weight_index):
    def fn(o, gate, w, eps):
        o = np.asarray(o, dtype=np.float64)
        wv = np.asarray(w, dtype=np.float64)
        wv = wv[:, None, :] if weight_index == "head" else wv[None, :1, None, :].reshape(1, 1, 1, -1)
        return gate_act(np.asarray(gate)) * wv * o / norm(o, eps)
    return fn


_sig = lambda x: 1.0 / (1.0 + np.exp(-x))
OUT_GATE_MUTANTS = {
    "l2_norm_not_rms": _og(lambda o, e: np.sqrt(np.sum(o * o, axis=-1, keepdims=True) + e), _sig, "head"),
    "mean_abs_norm": _og(lambda o, e: np.mean(np.abs(o), axis=-1, keepdims=True) + e, _sig, "head"),
    "gate_not_sigmoid": _og(lambda o, e: np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + e), np.tanh, "head"),
    "weight_of_head_0_everywhere": _og(lambda o, e: np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + e), _sig,
                                       "first"),
}


def test_output_gate_pins_hold_for_the_oracle():
    assert _output_gate_pins(oracle.output_gate)


@pytest.mark.parametrize("name", sorted(OUT_GATE_MUTANTS))
def test_output_gate_mutant_is_caught(name):
    assert not _output_gate_pins(OUT_GATE_MUTANTS[name])
