"""Speculative-decode replay and verify (Kimi K3 report, section 5.4.2):
kda_spec_replay_verify over a W-token window against the oracle recurrence.
The committed state must equal the state after the replayed (accepted)
tokens, and the outputs of the remaining tokens must equal the recurrence's
outputs when the window is run from the committed state onward."""
import numpy as np
import pytest
import torch

from gated_delta_rule_117_b200 import kda, synth
from parity_util import TOL, f64, rel_l2

import oracle

pytestmark = pytest.mark.gpu


def _check(w, n_replay, key):
    x = synth.prefill_inputs(w)  # [B, H, W, d] window inputs, h0 = the committed state
    d = {n: t.cuda() for n, t in x.items()}
    S = d["h0"].clone()
    nr = torch.tensor(n_replay, dtype=torch.int32, device="cuda")
    o = kda.spec_replay_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], S, nr)
    torch.cuda.synchronize()
    a = [f64(x[n]) for n in ("q", "k", "v", "g", "beta")]
    o_ref, _ = oracle.recurrent(*a, f64(x["h0"]))
    for b, n in enumerate(n_replay):
        n = min(max(n, 0), w.T)
        if n > 0:
            _, s_ref = oracle.recurrent(*[t[b:b + 1, :, :n] for t in a], f64(x["h0"])[b:b + 1])
        else:
            s_ref = f64(x["h0"])[b:b + 1]
        assert rel_l2(S[b:b + 1], s_ref) <= TOL["f32"], (b, n)
        if n < w.T:
            assert rel_l2(o[b:b + 1, :, n:], o_ref[b:b + 1, :, n:]) <= TOL[key], (b, n)


def test_bf16_d128_window():
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=5, H=3, T=6, seed=81)
    _check(w, [0, 1, 3, 6, 9], "bf16")  # 9 is clamped to the window


def test_fp32_shapes():
    for dk, dv in ((32, 64), (64, 16), (128, 128)):
        w = synth.WORKLOADS["tiny_f32"].with_(B=3, H=2, T=5, dk=dk, dv=dv, h0_std=0.05, seed=82 + dk)
        _check(w, [2, -1, 5], "f32")  # -1 is clamped to 0


def test_replay_then_verify_equals_stepwise_decode():
    # the window is the same recurrence as W single decode steps from the same state
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=2, H=2, T=4, seed=83)
    x = synth.prefill_inputs(w)
    d = {n: t.cuda() for n, t in x.items()}
    S_a = d["h0"].clone()
    nr = torch.tensor([4, 4], dtype=torch.int32, device="cuda")
    kda.spec_replay_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], S_a, nr)
    S_b = d["h0"].clone()
    for t in range(4):
        sl = {n: d[n][:, :, t].contiguous() for n in ("q", "k", "v", "g", "beta")}
        kda.recurrent_step(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], S_b)
    torch.cuda.synchronize()
    assert rel_l2(S_a, S_b) <= 1e-6


@pytest.mark.parametrize("dtype,key", [("bf16", "bf16"), ("f32", "f32")])
def test_fused_gate_edges_in_the_replay_loop(dtype, key):
    # the replay loop with the Eq. 5 gate on the inputs and the Eq. 6 edge on the
    # verified outputs: against oracle.gate -> oracle.recurrent -> oracle.output_gate
    W = 6
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=3, H=2, T=W, dtype=dtype, seed=84)
    x = synth.prefill_inputs(w)
    gi = synth.gate_inputs(w)
    g = torch.Generator().manual_seed(85)
    gate = (2 * torch.randn(w.B, w.H, W, 128, generator=g)).to(w.torch_dtype)
    rw = (1 + 0.3 * torch.randn(w.H, 128, generator=g)).float()
    n_replay = [0, 2, 6]
    d = {n: t.cuda() for n, t in x.items()}
    S = d["h0"].clone()
    nr = torch.tensor(n_replay, dtype=torch.int32, device="cuda")
    y = kda.spec_replay_verify_fused(d["q"], d["k"], d["v"], gi["z"].cuda(), gi["A_log"].cuda(), d["beta"], S,
                                     gate.cuda(), rw.cuda(), nr, eps=1e-6)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    g_ref = oracle.gate(f64(gi["z"]), gi["A_log"].double().numpy())
    a = [f64(x["q"]), f64(x["k"]), f64(x["v"]), g_ref, f64(x["beta"])]
    o_ref, _ = oracle.recurrent(*a, f64(x["h0"]))
    y_ref = oracle.output_gate(o_ref, f64(gate), rw.double().numpy(), 1e-6)
    for b, n in enumerate(n_replay):
        if n > 0:
            _, s_ref = oracle.recurrent(*[t[b:b + 1, :, :n] for t in a], f64(x["h0"])[b:b + 1])
        else:
            s_ref = f64(x["h0"])[b:b + 1]
        assert rel_l2(S[b:b + 1], s_ref) <= 1e-5, (b, n)
        if n < W:
            assert rel_l2(y[b:b + 1, :, n:], y_ref[b:b + 1, :, n:]) <= TOL[key], (b, n)


def test_many_chains_per_cta_and_two_staged_blocks():
    # more chains than the SMs hold at once (several waves of CTAs); W = 11 spans two
    # staged blocks of 8 tokens
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=24, H=16, T=11, seed=86)
    assert w.B * w.H > 2 * torch.cuda.get_device_properties(0).multi_processor_count
    _check(w, [(5 * b) % 13 for b in range(w.B)], "bf16")  # 0 .. 12: none, some, all, clamped


def test_fused_many_chains():
    W = 3
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=20, H=16, T=W, seed=87)
    x = synth.prefill_inputs(w)
    gi = synth.gate_inputs(w)
    g = torch.Generator().manual_seed(88)
    gate = (2 * torch.randn(w.B, w.H, W, 128, generator=g)).to(w.torch_dtype)
    rw = (1 + 0.3 * torch.randn(w.H, 128, generator=g)).float()
    n_replay = [b % 4 for b in range(w.B)]
    d = {n: t.cuda() for n, t in x.items()}
    S = d["h0"].clone()
    nr = torch.tensor(n_replay, dtype=torch.int32, device="cuda")
    y = kda.spec_replay_verify_fused(d["q"], d["k"], d["v"], gi["z"].cuda(), gi["A_log"].cuda(), d["beta"], S,
                                     gate.cuda(), rw.cuda(), nr, eps=1e-6)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    g_ref = oracle.gate(f64(gi["z"]), gi["A_log"].double().numpy())
    a = [f64(x["q"]), f64(x["k"]), f64(x["v"]), g_ref, f64(x["beta"])]
    o_ref, _ = oracle.recurrent(*a, f64(x["h0"]))
    y_ref = oracle.output_gate(o_ref, f64(gate), rw.double().numpy(), 1e-6)
    for b, n in enumerate(n_replay):
        s_ref = (oracle.recurrent(*[t[b:b + 1, :, :n] for t in a], f64(x["h0"])[b:b + 1])[1] if n > 0
                 else f64(x["h0"])[b:b + 1])
        assert rel_l2(S[b:b + 1], s_ref) <= 1e-5, (b, n)
        if n < W:
            assert rel_l2(y[b:b + 1, :, n:], y_ref[b:b + 1, :, n:]) <= TOL["bf16"], (b, n)


def test_inputs_off_16_byte_boundaries():
    # window inputs that start 2 bytes past a 16-byte boundary (element-aligned only)
    # must give bitwise the same result as aligned ones
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=3, H=4, T=5, seed=89)
    x = synth.prefill_inputs(w)
    d = {n: t.cuda() for n, t in x.items()}
    nr = torch.tensor([0, 2, 5], dtype=torch.int32, device="cuda")
    S_a = d["h0"].clone()
    o_a = kda.spec_replay_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], S_a, nr)
    shifted = {}
    for n in ("q", "k", "v", "g"):
        buf = torch.empty(d[n].numel() + 1, dtype=d[n].dtype, device="cuda")
        view = buf[1:].view(d[n].shape)
        view.copy_(d[n])
        assert view.data_ptr() % 16 != 0
        shifted[n] = view
    S_b = d["h0"].clone()
    o_b = kda.spec_replay_verify(shifted["q"], shifted["k"], shifted["v"], shifted["g"], d["beta"], S_b, nr)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    assert torch.equal(S_a, S_b) and torch.equal(o_a, o_b)
