"""GPU parity of kda_recurrent_step (one token per sequence, state updated in
place) against the fp64 oracle run over the same steps."""
import numpy as np
import pytest
import torch

from gated_delta_rule_117_b200 import kda, synth
from parity_util import TOL, f64, rel_l2

import oracle

pytestmark = pytest.mark.gpu


def _decode(w, steps, heads=None):
    x = synth.decode_inputs(w, steps=steps)
    d = {k: v.cuda() for k, v in x.items()}
    S = d["S0"].clone()
    outs = []
    for t in range(steps):
        outs.append(kda.recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S))
    o = torch.stack(outs, 2)  # [B, H, steps, dv]
    # oracle: the decode steps are the recurrence over `steps` tokens from S0
    def pick(a):
        return a[[b for b, _ in heads], [h for _, h in heads]] if heads else a

    seq = lambda n: pick(f64(x[n].movedim(0, 2)))  # [steps, B, H, ...] -> [B, H, steps, ...]
    o_ref, S_ref = oracle.recurrent(seq("q"), seq("k"), seq("v"), seq("g"), seq("beta"), pick(f64(x["S0"])))
    if heads:
        o = torch.stack([o[b, h] for b, h in heads])
        S = torch.stack([S[b, h] for b, h in heads])
    return o, S, o_ref, S_ref


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 128), (128, 32), (64, 64), (128, 128)])
def test_small_shapes(dtype, dk, dv):
    w = synth.WORKLOADS["decode_b256_h32"].with_(B=3, H=5, dk=dk, dv=dv, dtype=dtype, seed=55)
    o, S, o_ref, S_ref = _decode(w, 9)
    assert rel_l2(o, o_ref) <= TOL[dtype]
    assert rel_l2(S, S_ref) <= TOL[dtype]


def test_decode_workload_full_size_sampled_heads():
    w = synth.WORKLOADS["decode_b256_h32"]
    heads = [(0, 0), (17, 5), (128, 31), (255, 16), (200, 3), (64, 30)]
    o, S, o_ref, S_ref = _decode(w, w.T, heads)
    assert rel_l2(o, o_ref) <= TOL["bf16"]
    assert rel_l2(S, S_ref) <= TOL["bf16"]


def test_decode_matches_prefill_of_same_tokens():
    # one decode step per token == prefill over those tokens (same recurrence)
    w = synth.WORKLOADS["decode_b256_h32"].with_(B=2, H=4, dtype="f32", seed=9)
    x = synth.decode_inputs(w, steps=20)
    d = {k: v.cuda() for k, v in x.items()}
    S = d["S0"].clone()
    outs = [kda.recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S) for t in range(20)]
    mv = lambda t: t.movedim(0, 2).contiguous()
    o_p, h_p = kda.chunk_fwd(mv(d["q"]), mv(d["k"]), mv(d["v"]), mv(d["g"]), d["beta"].movedim(0, 2).contiguous(),
                             d["S0"])
    assert rel_l2(torch.stack(outs, 2), o_p) <= 1e-5 and rel_l2(S, h_p) <= 1e-5
