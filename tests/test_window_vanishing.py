"""Why a 128-token window settles a context-parallel segment transition.

The tensor-core plan first computes each segment's transition over the last
128 tokens only; where that window's M = prod_t (I - beta_t k_t k_t^T) Diag(alpha_t)
underflows to an exactly zero fp32 state, the segment's M is zero and its S~ is
the window's (Kimi K3 report, section 5.1.2, Eq. 17, split at the window's
start).  Here the same product is run token by token in fp32 numpy on the
synthetic workloads' inputs: at their decay it reaches exact zero well inside
128 tokens, and at decays 20x slower it does not (those segments run again in
full on the device, which the GPU tests exercise)."""
import numpy as np
import pytest

from gated_delta_rule_117_b200 import synth

WINDOW = 128


def _window_transition(x, start, scale=1.0):
    k = x["k"].astype(np.float32)
    g = (x["g"] * scale).astype(np.float32)
    beta = x["beta"].astype(np.float32)
    M = np.eye(k.shape[1], dtype=np.float32)
    for t in range(start, start + WINDOW):
        M = np.exp(g[t])[:, None] * M
        M = M - beta[t] * np.outer(k[t], k[t] @ M)
        if not np.any(M):
            return M, t - start + 1
    return M, None


@pytest.mark.parametrize("name,h", [("prefill_h16_t4k", 0), ("prefill_h16_t4k", 9), ("long_h16_t1m", 5),
                                    ("batched_b8_h32_t8k", 0)])
def test_window_transition_vanishes_at_the_workloads_decay(name, h):
    w = synth.WORKLOADS[name]
    x = synth.head_inputs(w, 0, h, T=3 * WINDOW)
    for start in (0, WINDOW, 2 * WINDOW - 40):
        M, tokens = _window_transition(x, start)
        assert tokens is not None and tokens <= 96, (name, h, start, tokens)  # a chunk of margin at least


def test_fast_decay_heads_vanish_within_the_window():
    # A ~ N(2, 0.5) makes the gate bimodal (g near -5 or near 0 per token and channel), so the
    # product takes longer to underflow: 108-115 tokens, inside the window without a chunk to
    # spare (a window that does not vanish only sends its segment through the full pass)
    w = synth.WORKLOADS["batched_b8_h32_t8k"]
    for h in synth.fast_decay_heads(w):
        M, tokens = _window_transition(synth.head_inputs(w, 0, int(h), T=WINDOW), 0)
        assert tokens is not None and tokens <= WINDOW, (h, tokens)


def test_slow_decay_window_does_not_vanish():
    w = synth.WORKLOADS["prefill_h16_t4k"]
    M, tokens = _window_transition(synth.head_inputs(w, 0, 0, T=WINDOW), 0, scale=0.05)
    assert tokens is None and np.abs(M).max() > 1e-12
