"""Host-side logic of bench.py (no GPU): rank-count checks, the chains the
oracle leg samples, and the plan's segment bookkeeping it relies on."""
import os
import subprocess
import sys

import pytest

import bench
from gated_delta_rule_117_b200 import kda, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_gpus_must_match_world_size():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE=1" in (r.stderr + r.stdout)


def test_sampled_chains_cover_ends_and_fast_decay_heads():
    w = synth.WORKLOADS["batched_b8_h32_t8k"]
    c = bench.sample_chains(w)
    assert (0, 0) in c and (w.B - 1, w.H - 1) in c
    fast = set(synth.fast_decay_heads(w).tolist())
    assert any(h in fast for _, h in c)
    assert len(set(c)) == len(c)
    assert all(0 <= b < w.B and 0 <= h < w.H for b, h in c)


@pytest.mark.parametrize("B,H,T", [(1, 16, 1 << 20), (1, 16, 4096), (2, 3, 1100), (8, 32, 8192), (1, 1, 0)])
def test_plan_segment_tokens(B, H, T):
    p = kda.kda_chunk_fwd_plan(B, H, T, 128, 128, kda.KDA_DTYPE_BF16, 0)
    L, P = p["segment_tokens"], p["segments"]
    if P == 1:
        assert L == T
    else:
        assert L % p["chunk_size"] == 0 and (P - 1) * L < T <= P * L


def test_oracle_leg_rel_l2_helper():
    import numpy as np
    a = np.ones((4, 3))
    assert bench.rel_l2_np(a, a) == 0.0
    assert bench.rel_l2_np(2 * a, a) == pytest.approx(1.0)
