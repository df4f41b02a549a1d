"""Chunkwise-parallel KDA forward in fp64 numpy -- TEST INFRASTRUCTURE ONLY.

Restates the Kimi K3 report's chunked form (section 2.1.1): inside a chunk of
C tokens everything is parallel, across chunks the state is carried.

For one chunk with entering state S (dk x dv), per-token log-decay g, and the
chunk-local inclusive cumulative log-decay G_r = sum_{s<=r} g_s (Eq. 3, kept in
log space; gamma^r = exp(G_r)):

  A_rj = sum_c q_rc k_jc exp(G_rc - G_jc)          for j <= r   (Eq. 4, Tril
                                                   keeps the diagonal)
  L_rj = beta_r sum_c k_rc k_jc exp(G_rc - G_jc)   for j <  r
  T    = (I + L)^-1 Diag(beta)                     (UT transform)
  U    = T V,   W = T (K * exp(G))
  V~   = U - W S                                   (pseudo-values)
  O    = scale * [ (Q * exp(G)) S + A V~ ]          (Eq. 4)
  S'   = Diag(exp(G_C)) S + (K * exp(G_C - G))^T V~

The report defers the UT derivation and does not print the state update; both
follow from Eq. 1: with u_r = beta_r (v_r - S_{r-1}^T (alpha_r * k_r)) the
recurrence reads S_r = Diag(alpha_r) S_{r-1} + k_r u_r^T; unrolling inside the
chunk gives (I + L) U~ = Diag(beta)(V - (K * exp(G)) S), i.e. U~ = V~ above.
The chunk's action on its entering state is S' = M S + K'^T U with
M = Diag(exp(G_C)) - (K * exp(G_C - G))^T W, which is the per-chunk factor of
KDA Context Parallelism (section 5.1.2, Eq. 17).
"""
from __future__ import annotations

import numpy as np


def chunked_chain(q, k, v, g, beta, h0=None, C=64, scale=None, return_transitions=False):
    """One (b, h) chain.  q, k, g [T, dk]; v [T, dv]; beta [T]; h0 [dk, dv].

    The last chunk may be shorter than C.  Returns (o [T, dv], h_T [dk, dv]) and,
    with ``return_transitions``, the list of per-chunk (M, K'^T U) pairs.
    """
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, dk = q.shape
    dv = v.shape[1]
    if scale is None:
        scale = dk ** -0.5
    S = np.zeros((dk, dv)) if h0 is None else np.array(h0, dtype=np.float64)
    o = np.empty((T, dv))
    trans = []
    for t0 in range(0, T, C):
        t1 = min(t0 + C, T)
        n = t1 - t0
        Q, K, V, b = q[t0:t1], k[t0:t1], v[t0:t1], beta[t0:t1]
        G = np.cumsum(g[t0:t1], axis=0)                    # inclusive, [n, dk]
        A = np.zeros((n, n))
        L = np.zeros((n, n))
        for r in range(n):
            for j in range(r + 1):
                w = np.exp(G[r] - G[j])                    # gamma^{j+1 -> r}
                A[r, j] = np.sum(Q[r] * K[j] * w)
                if j < r:
                    L[r, j] = b[r] * np.sum(K[r] * K[j] * w)
        Tm = np.linalg.solve(np.eye(n) + L, np.diag(b))    # (I + L)^-1 Diag(beta)
        U = Tm @ V
        W = Tm @ (K * np.exp(G))
        Vt = U - W @ S
        o[t0:t1] = scale * ((Q * np.exp(G)) @ S + A @ Vt)
        Kp = K * np.exp(G[-1] - G)                         # K * exp(G_C - G)
        if return_transitions:
            trans.append((np.diag(np.exp(G[-1])) - Kp.T @ W, Kp.T @ U))
        S = np.exp(G[-1])[:, None] * S + Kp.T @ Vt
    if return_transitions:
        return o, S, trans
    return o, S


def chunked(q, k, v, g, beta, h0=None, C=64, scale=None):
    """Chunked form over leading (batch, head) dims; same shapes as oracle.recurrent."""
    q = np.asarray(q, dtype=np.float64)
    lead = q.shape[:-2]
    n = int(np.prod(lead)) if lead else 1
    T, dk = q.shape[-2:]
    dv = np.shape(v)[-1]
    qf = q.reshape(n, T, dk)
    kf = np.asarray(k, dtype=np.float64).reshape(n, T, dk)
    vf = np.asarray(v, dtype=np.float64).reshape(n, T, dv)
    gf = np.asarray(g, dtype=np.float64).reshape(n, T, dk)
    bf = np.asarray(beta, dtype=np.float64).reshape(n, T)
    hf = None if h0 is None else np.asarray(h0, dtype=np.float64).reshape(n, dk, dv)
    o = np.empty((n, T, dv))
    hT = np.empty((n, dk, dv))
    for i in range(n):
        o[i], hT[i] = chunked_chain(qf[i], kf[i], vf[i], gf[i], bf[i], None if hf is None else hf[i], C, scale)
    return o.reshape(lead + (T, dv)), hT.reshape(lead + (dk, dv))


def transition(k, g, beta):
    """Cumulative transition of a token segment, M = M_T ... M_1 with
    M_t = (I - beta_t k_t k_t^T) Diag(alpha_t)  (Kimi K3 report, Eq. 17).

    k, g [T, dk]; beta [T].  Returns M [dk, dk] such that the segment maps an
    entering state S to S~ + M S, where S~ is the segment run from S = 0.
    """
    k, g, beta = (np.asarray(x, dtype=np.float64) for x in (k, g, beta))
    dk = k.shape[1]
    M = np.eye(dk)
    for t in range(k.shape[0]):
        Mt = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) * np.exp(g[t])[None, :]
        M = Mt @ M
    return M
