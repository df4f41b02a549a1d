"""Pins for the fp64 oracle, against facts fixed by the Kimi K3 report and by
the mathematics (no GPU needed).

Each pin is chosen so that a plausible mistake in the oracle fails it:
  * brute-force products        -- decay/erase order, transposed read-out,
                                   scale applied to the state, dropped write;
  * beta = 0, g = 0              -- spurious state changes;
  * delta-write property         -- the erase uses the decayed state and k k^T;
  * reduction to gated linear    -- the decay channel (rows of S = key dim),
    attention (closed form)         the inclusive cumulative product, the scale;
  * scalar closed form           -- textbook first-order linear recurrence;
  * chunk-size independence      -- the UT transform / chunked restatement;
  * state split                  -- h0 handling and the carried state;
  * KCP linearity (Eq. 17)       -- S_T(h0) = S~_T + M h0;
  * Eq. 5 gate                   -- midpoint, bounds, limits, per-channel scale;
  * Eq. 6 output edge            -- hand-worked row, scale invariance, unit RMS;
  * prefix-cache checkpoints     -- each snapshot is the brute-force state at
    (section 5.4.1)                 its position, and prefill resumed from a
                                    snapshot reproduces the rest of the run.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inputs(rs, T, dk, dv, decay_scale=1.0, unit_k=True):
    q = rs.standard_normal((T, dk))
    k = rs.standard_normal((T, dk))
    if unit_k:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rs.standard_normal((T, dv))
    # Eq. 5 shape of the log-decay: g in (-5, 0)
    g = -5.0 / (1.0 + np.exp(-decay_scale * rs.standard_normal((T, dk))))
    beta = 1.0 / (1.0 + np.exp(-rs.standard_normal(T)))
    return q, k, v, g, beta


def _brute(q, k, v, g, beta, h0, scale):
    """S_t = (M_t ... M_1) h0 + sum_{j<=t} (M_t ... M_{j+1}) beta_j k_j v_j^T with
    M_t = (I - beta_t k_t k_t^T) Diag(exp g_t), built as explicit matrices."""
    T, dk = q.shape
    Ms = [(np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) for t in range(T)]
    outs, S_t = [], None
    for t in range(T):
        P = np.eye(dk)
        for r in range(t, -1, -1):
            P = P @ Ms[r]
        S_t = P @ h0
        for j in range(t + 1):
            Pj = np.eye(dk)
            for r in range(t, j, -1):
                Pj = Pj @ Ms[r]
            S_t = S_t + Pj @ (beta[j] * np.outer(k[j], v[j]))
        outs.append(scale * S_t.T @ q[t])
    return np.array(outs), S_t


@pytest.mark.parametrize("T,dk,dv", [(1, 1, 1), (3, 3, 4), (6, 4, 2), (5, 2, 3)])
def test_brute_force_products(T, dk, dv):
    rs = np.random.default_rng(7 + T * 10 + dk)
    q, k, v, g, beta = _rand_inputs(rs, T, dk, dv, unit_k=False)
    h0 = rs.standard_normal((dk, dv))
    o, hT = oracle.recurrent(q, k, v, g, beta, h0, scale=0.7)
    ob, hb = _brute(q, k, v, g, beta, h0, 0.7)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hT, hb, rtol=0, atol=1e-12)


def test_default_scale_is_inverse_sqrt_dk():
    rs = np.random.default_rng(3)
    q, k, v, g, beta = _rand_inputs(rs, 5, 9, 4)
    o1, _ = oracle.recurrent(q, k, v, g, beta)
    o2, _ = oracle.recurrent(q, k, v, g, beta, scale=1.0)
    np.testing.assert_allclose(o1, o2 / 3.0, rtol=1e-14, atol=0)


def test_zero_beta_zero_decay_keeps_state():
    rs = np.random.default_rng(11)
    T, dk, dv = 9, 5, 6
    q, k, v, _, _ = _rand_inputs(rs, T, dk, dv)
    h0 = rs.standard_normal((dk, dv))
    o, hT = oracle.recurrent(q, k, v, np.zeros((T, dk)), np.zeros(T), h0)
    assert np.array_equal(hT, h0)
    np.testing.assert_allclose(o, dk ** -0.5 * q @ h0, rtol=0, atol=1e-14)


def test_delta_write_property():
    # g = 0, beta = 1, |k| = 1: after token t the state maps k_t exactly onto v_t.
    rs = np.random.default_rng(5)
    T, dk, dv = 7, 6, 5
    q, k, v, _, _ = _rand_inputs(rs, T, dk, dv)
    h0 = rs.standard_normal((dk, dv))
    for t in range(1, T + 1):
        _, S = oracle.recurrent(q[:t], k[:t], v[:t], np.zeros((t, dk)), np.ones(t), h0)
        np.testing.assert_allclose(S.T @ k[t - 1], v[t - 1], rtol=0, atol=1e-12)
    # general beta, g = 0: k_t^T S_t = (1 - beta_t) k_t^T S_{t-1} + beta_t v_t^T
    beta = rs.uniform(0.05, 0.95, T)
    g0 = np.zeros((T, dk))
    for t in range(1, T):
        _, Sp = oracle.recurrent(q[:t], k[:t], v[:t], g0[:t], beta[:t], h0)
        _, St = oracle.recurrent(q[:t + 1], k[:t + 1], v[:t + 1], g0[:t + 1], beta[:t + 1], h0)
        np.testing.assert_allclose(k[t] @ St, (1 - beta[t]) * (k[t] @ Sp) + beta[t] * v[t], rtol=0, atol=1e-12)


def test_reduces_to_gated_linear_attention():
    # Without the erase term the recurrence is gated linear attention whose
    # closed form uses the global inclusive cumulative log-decay along keys.
    rs = np.random.default_rng(9)
    T, dk, dv = 23, 7, 5
    q, k, v, g, beta = _rand_inputs(rs, T, dk, dv)
    h0 = rs.standard_normal((dk, dv))
    o, hT = oracle.recurrent(q, k, v, g, beta, h0, erase=False)
    Gh = np.cumsum(g, axis=0)
    ref = np.zeros((T, dv))
    for t in range(T):
        acc = (q[t] * np.exp(Gh[t])) @ h0
        for j in range(t + 1):
            acc = acc + np.dot(q[t] * np.exp(Gh[t] - Gh[j]), k[j]) * beta[j] * v[j]
        ref[t] = dk ** -0.5 * acc
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    S_ref = np.exp(Gh[-1])[:, None] * h0 + sum(
        np.outer(k[j] * np.exp(Gh[-1] - Gh[j]), beta[j] * v[j]) for j in range(T))
    np.testing.assert_allclose(hT, S_ref, rtol=0, atol=1e-12)


def test_scalar_closed_form():
    # dk = dv = 1: s_t = a_t s_{t-1} + b_t with a_t = (1 - beta k^2) alpha,
    # b_t = beta k v, whose solution is s_T = (prod a) s_0 + sum_j (prod_{r>j} a_r) b_j.
    rs = np.random.default_rng(21)
    T = 40
    k = rs.uniform(-1, 1, (T, 1))
    q = rs.standard_normal((T, 1))
    v = rs.standard_normal((T, 1))
    g = rs.uniform(-5, 0, (T, 1))
    beta = rs.uniform(0, 1, T)
    s0 = np.array([[0.3]])
    o, hT = oracle.recurrent(q, k, v, g, beta, s0)
    a = (1 - beta * k[:, 0] ** 2) * np.exp(g[:, 0])
    b = beta * k[:, 0] * v[:, 0]
    s = np.empty(T)
    for t in range(T):
        s[t] = np.prod(a[:t + 1]) * 0.3 + sum(np.prod(a[j + 1:t + 1]) * b[j] for j in range(t + 1))
    np.testing.assert_allclose(hT[0, 0], s[-1], rtol=1e-13)
    np.testing.assert_allclose(o[:, 0], q[:, 0] * s, rtol=1e-12, atol=1e-14)


def test_hand_worked_golden():
    # Hand-derived values (exact decimal arithmetic), see the fixture for the derivation.
    rows = [l.split() for l in open(os.path.join(GOLDEN, "hand_worked_d1.txt")) if l.strip() and not l.startswith("#")]
    rec = {r[0]: [float(x) for x in r[1:]] for r in rows}
    q, k, v = np.array(rec["q"])[:, None], np.array(rec["k"])[:, None], np.array(rec["v"])[:, None]
    g, beta = np.log(np.array(rec["alpha"]))[:, None], np.array(rec["beta"])
    o, hT = oracle.recurrent(q, k, v, g, beta, np.array([rec["h0"]]), scale=1.0)
    np.testing.assert_allclose(o[:, 0], rec["o"], rtol=1e-14)
    np.testing.assert_allclose(hT[0, 0], rec["hT"][0], rtol=1e-14)


@pytest.mark.parametrize("C", [1, 2, 4, 8, 16, 32, 64])
def test_chunk_size_independence(C):
    rs = np.random.default_rng(100 + C)
    T, dk, dv = 75, 8, 6      # 75: ragged last chunk for every C > 1
    q, k, v, g, beta = _rand_inputs(rs, T, dk, dv)
    h0 = 0.1 * rs.standard_normal((dk, dv))
    o, hT = oracle.recurrent(q, k, v, g, beta, h0)
    oc, hc = oracle.chunked_chain(q, k, v, g, beta, h0, C=C)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hc, hT, rtol=0, atol=1e-12)


def test_chunked_strong_decay_16_token_tiles():
    # g pinned at the -5 bound: 16-token cumulative log-decay reaches -80 and a
    # 64-token chunk -320; the log-space form must stay exact.
    rs = np.random.default_rng(8)
    T, dk, dv = 130, 4, 3
    q, k, v, _, beta = _rand_inputs(rs, T, dk, dv)
    g = np.full((T, dk), -5.0)
    g[:, 0] = -0.01
    o, hT = oracle.recurrent(q, k, v, g, beta)
    oc, hc = oracle.chunked_chain(q, k, v, g, beta, None, C=64)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hc, hT, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T1", [1, 13, 16, 40, 63])
def test_state_split_identity(T1):
    rs = np.random.default_rng(40 + T1)
    T, dk, dv = 64, 6, 7
    q, k, v, g, beta = _rand_inputs(rs, T, dk, dv)
    h0 = rs.standard_normal((dk, dv))
    o, hT = oracle.recurrent(q, k, v, g, beta, h0)
    o1, h1 = oracle.recurrent(q[:T1], k[:T1], v[:T1], g[:T1], beta[:T1], h0)
    o2, h2 = oracle.recurrent(q[T1:], k[T1:], v[T1:], g[T1:], beta[T1:], h1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(h2, hT, rtol=0, atol=1e-13)


def test_kcp_linearity_eq17():
    rs = np.random.default_rng(17)
    T, dk, dv = 37, 6, 5
    q, k, v, g, beta = _rand_inputs(rs, T, dk, dv)
    h0 = rs.standard_normal((dk, dv))
    h1 = rs.standard_normal((dk, dv))
    _, S0 = oracle.recurrent(q, k, v, g, beta, None)
    _, Sh = oracle.recurrent(q, k, v, g, beta, h0)
    M = oracle.transition(k, g, beta)
    np.testing.assert_allclose(Sh, S0 + M @ h0, rtol=0, atol=1e-12)
    _, Sa = oracle.recurrent(q, k, v, g, beta, h0 + h1)
    _, Sb = oracle.recurrent(q, k, v, g, beta, h1)
    np.testing.assert_allclose(Sa - Sb, Sh - S0, rtol=0, atol=1e-12)
    # Three segments recombined by the prefix scan S <- M_j S + S~_j
    cuts = [0, 10, 26, T]
    S = h0.copy()
    for a, b in zip(cuts[:-1], cuts[1:]):
        Mj = oracle.transition(k[a:b], g[a:b], beta[a:b])
        _, St = oracle.recurrent(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], None)
        S = Mj @ S + St
    np.testing.assert_allclose(S, Sh, rtol=0, atol=1e-12)


def test_chunk_transitions_compose_to_token_transition():
    rs = np.random.default_rng(23)
    T, dk, dv = 48, 5, 4
    q, k, v, g, beta = _rand_inputs(rs, T, dk, dv)
    _, _, trans = oracle.chunked_chain(q, k, v, g, beta, None, C=16, return_transitions=True)
    M = np.eye(dk)
    for Mc, _ in trans:
        M = Mc @ M
    np.testing.assert_allclose(M, oracle.transition(k, g, beta), rtol=0, atol=1e-12)


def test_batched_chains_match_single_chains():
    rs = np.random.default_rng(31)
    B, H, T, dk, dv = 2, 3, 11, 4, 5
    q = rs.standard_normal((B, H, T, dk))
    k = rs.standard_normal((B, H, T, dk))
    v = rs.standard_normal((B, H, T, dv))
    g = -rs.uniform(0, 5, (B, H, T, dk))
    beta = rs.uniform(0, 1, (B, H, T))
    h0 = rs.standard_normal((B, H, dk, dv))
    o, hT = oracle.recurrent(q, k, v, g, beta, h0, nthreads=4)
    for b in range(B):
        for h in range(H):
            o1, h1 = oracle.recurrent(q[b, h], k[b, h], v[b, h], g[b, h], beta[b, h], h0[b, h], nthreads=1)
            assert np.array_equal(o1, o[b, h]) and np.array_equal(h1, hT[b, h])


def test_empty_sequence_returns_h0():
    h0 = np.arange(12.0).reshape(3, 4)
    e = np.zeros((0, 3))
    o, hT = oracle.recurrent(e, e, np.zeros((0, 4)), e, np.zeros(0), h0)
    assert o.shape == (0, 4) and np.array_equal(hT, h0)


def test_checkpoints_are_brute_force_prefix_states():
    # section 5.4.1: the snapshot at a block boundary p is the state after token p - 1
    rs = np.random.default_rng(515)
    T, dk, dv, interval = 7, 3, 2, 3
    q, k, v, g, beta = _rand_inputs(rs, T, dk, dv, unit_k=False)
    h0 = rs.standard_normal((dk, dv))
    ck = oracle.checkpoints(q, k, v, g, beta, h0, interval=interval, scale=0.5)
    assert ck.shape == (T // interval, dk, dv)
    for j in range(T // interval):
        p = (j + 1) * interval
        _, S_p = _brute(q[:p], k[:p], v[:p], g[:p], beta[:p], h0, 0.5)
        np.testing.assert_allclose(ck[j], S_p, rtol=0, atol=1e-12)


def test_resume_from_checkpoint_reproduces_the_run():
    rs = np.random.default_rng(516)
    T, dk, dv, interval = 200, 8, 6, 64
    q, k, v, g, beta = _rand_inputs(rs, T, dk, dv)
    h0 = 0.02 * rs.standard_normal((dk, dv))
    o, hT = oracle.recurrent(q, k, v, g, beta, h0)
    ck = oracle.checkpoints(q, k, v, g, beta, h0, interval=interval)
    assert ck.shape == (3, dk, dv)
    for j in range(3):
        p = (j + 1) * interval
        o2, h2 = oracle.recurrent(q[p:], k[p:], v[p:], g[p:], beta[p:], ck[j])
        np.testing.assert_allclose(o2, o[p:], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(h2, hT, rtol=1e-12, atol=1e-13)
    # no block boundary inside a short sequence: no snapshot
    assert oracle.checkpoints(q[:50], k[:50], v[:50], g[:50], beta[:50], h0, interval=interval).shape == (0, dk, dv)


def test_gate_eq5_closed_forms():
    # Eq. 5: g = g_min Sigmoid(e^A z), in (g_min, 0); A is a per-head, per-channel log-scale
    A = np.array([[0.0, math.log(2.0)], [-1.0, 0.5]])
    z = np.zeros((1, 2, 1, 2))
    np.testing.assert_allclose(oracle.gate(z, A), -2.5, rtol=0, atol=1e-15)  # Sigmoid(0) = 1/2
    z = np.array([[[[1.0, 1.0]], [[-2.0, 3.0]]]])
    ref = -5.0 / (1.0 + np.exp(-np.array([[[1.0, 2.0]], [[-2.0 * math.exp(-1.0), 3.0 * math.exp(0.5)]]])))
    np.testing.assert_allclose(oracle.gate(z, A)[0], ref, rtol=1e-15)
    big = oracle.gate(np.full((1, 2, 1, 2), 200.0), A)
    small = oracle.gate(np.full((1, 2, 1, 2), -200.0), A)
    assert np.all(big >= -5.0) and np.all(big < -4.999999) and np.all(small < 0) and np.all(small > -1e-9)
    zz = np.random.default_rng(5).standard_normal((2, 2, 50, 2)) * 3
    gg = oracle.gate(zz, A)
    assert np.all(gg > -5.0) and np.all(gg < 0.0)
    # retention alpha = e^g stays above e^{g_min} (the bound the report prints)
    assert np.exp(gg).min() > math.exp(-5.0)
    # a different g_min scales the gate
    np.testing.assert_allclose(oracle.gate(zz, A, g_min=-2.0), gg * 0.4, rtol=1e-14)


def test_output_gate_eq6():
    # hand-worked row: o = (3, 4), mean square 12.5, gate 0 -> Sigmoid = 1/2, w = (1, 2)
    o = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    y = oracle.output_gate(o, np.zeros_like(o), np.array([[1.0, 2.0]]), eps=0.0)
    np.testing.assert_allclose(y.ravel(), [0.5 * 3.0 / math.sqrt(12.5), 0.5 * 2.0 * 4.0 / math.sqrt(12.5)], rtol=1e-15)
    rs = np.random.default_rng(6)
    o = rs.standard_normal((2, 3, 5, 16))
    gate = rs.standard_normal((2, 3, 5, 16))
    w = rs.standard_normal((3, 16))
    y = oracle.output_gate(o, gate, w, eps=0.0)
    # RMSNorm is invariant to a positive rescaling of the row
    np.testing.assert_allclose(oracle.output_gate(7.5 * o, gate, w, eps=0.0), y, rtol=1e-13)
    # with unit weights and an open gate (large logits) the rows have unit RMS
    yy = oracle.output_gate(o, np.full_like(o, 60.0), np.ones((3, 16)), eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(yy * yy, axis=-1)), 1.0, rtol=1e-12)
    # the weight is per head: head 1 only sees w[1]
    w2 = w.copy()
    w2[0] *= 3.0
    np.testing.assert_allclose(oracle.output_gate(o, gate, w2, eps=0.0)[:, 1:], y[:, 1:], rtol=0, atol=0)
