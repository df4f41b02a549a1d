"""KDA forward oracle -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct CPU restatements of what the CUDA library
computes, in fp64:

* ``recurrent``   -- the token-by-token recurrence of the Kimi K3 report,
  section 2.1.1, Eq. 1 (C code in ``kda_oracle.c``, threaded over chains);
* ``chunked``     -- the chunkwise-parallel form of the same report (Eq. 3
  cumulative decay, Eq. 4 outputs, UT transform) with the inter-chunk state
  update derived from Eq. 1 (numpy, one chain at a time);
* ``transition``  -- the per-segment pair (cumulative transition M, state from
  zero S~) of KDA Context Parallelism (section 5.1.2, Eq. 17), used to pin the
  oracle and to check in-device context parallelism;
* ``gate``        -- the lower-bounded decay gate of Eq. 5, g = g_min Sigmoid(e^A z);
* ``output_gate`` -- the output edge of Eq. 6, Sigmoid(gate) * RMSNorm(o);
* ``checkpoints`` -- the recurrent state at every multiple of a block size,
  the snapshots section 5.4.1 persists for prefix caching (by definition the
  final state of each prefix).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library
(``gated_delta_rule_117_b200``), which never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .chunked import chunked, chunked_chain, transition  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "kda_oracle.c")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no GPU needed)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.kda_oracle_recurrent.argtypes = [dp] * 8 + [ctypes.c_int] * 5 + [ctypes.c_double] + [ctypes.c_int] * 2
        lib.kda_oracle_recurrent.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def recurrent(q, k, v, g, beta, h0=None, scale=None, erase=True, nthreads=None):
    """Token recurrence (Eq. 1) over independent chains, fp64.

    Shapes: q, k, g [..., T, dk]; v [..., T, dv]; beta [..., T]; h0 [..., dk, dv]
    or None (zeros).  Leading dims are flattened into chains.  ``scale`` None
    means dk**-0.5.  Returns (o [..., T, dv], h_T [..., dk, dv]) as fp64.
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    lead = q.shape[:-2]
    T, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    n = int(np.prod(lead)) if lead else 1
    assert k.shape == q.shape and g.shape == q.shape and v.shape == lead + (T, dv)
    assert beta.shape == lead + (T,)
    if h0 is not None:
        h0 = _f64(h0)
        assert h0.shape == lead + (dk, dv)
    o = np.empty(lead + (T, dv))
    hT = np.empty(lead + (dk, dv))
    if scale is None:
        scale = dk ** -0.5
    if nthreads is None:
        nthreads = min(os.cpu_count() or 1, max(n, 1))
    rc = _load().kda_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o), _ptr(hT),
                                      1, n, T, dk, dv, float(scale), 1 if erase else 0, int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle failed (%d)" % rc)
    return o, hT


def checkpoints(q, k, v, g, beta, h0=None, interval=512, scale=None):
    """States a prefix cache would persist (Kimi K3 report, section 5.4.1): entry
    j is the state after token (j + 1) * interval - 1, i.e. h_T of the prefix of
    (j + 1) * interval tokens, computed here by running the recurrence on that
    prefix.  Shapes as for ``recurrent``; returns [..., T // interval, dk, dv]."""
    T = np.shape(q)[-2]
    out = []
    for j in range(T // interval):
        p = (j + 1) * interval
        _, hT = recurrent(np.asarray(q)[..., :p, :], np.asarray(k)[..., :p, :], np.asarray(v)[..., :p, :],
                          np.asarray(g)[..., :p, :], np.asarray(beta)[..., :p], h0, scale=scale)
        out.append(hT)
    lead = np.shape(q)[:-2]
    dk, dv = np.shape(q)[-1], np.shape(v)[-1]
    if not out:
        return np.zeros(lead + (0, dk, dv))
    return np.stack(out, axis=-3)


def gate(z, A_log, g_min=-5.0):
    """Eq. 5 of the Kimi K3 report: the per-channel log-decay
    g = g_min * Sigmoid(exp(A) * z), in fp64.  z [..., H, T, dk], A_log [H, dk]
    (broadcast over the leading and token dimensions)."""
    z = np.asarray(z, dtype=np.float64)
    eA = np.exp(np.asarray(A_log, dtype=np.float64))[:, None, :]
    return g_min / (1.0 + np.exp(-eA * z))


def output_gate(o, gate, w, eps=1e-6):
    """Eq. 6 of the Kimi K3 report without its projections: per-head RMSNorm of
    the recurrent output (over dv, weights w [H, dv]) times Sigmoid(gate), in
    fp64.  o, gate [B, H, T, dv]."""
    o = np.asarray(o, dtype=np.float64)
    gate = np.asarray(gate, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)[:, None, :]
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return (1.0 / (1.0 + np.exp(-gate))) * w * o / rms
