"""The Eq. 5 decay gate fused into the prefill loads (Kimi K3 report, section
2.1.1): kda_chunk_fwd_gated takes the logits z and log-scales A instead of g;
checked against the oracle recurrence run on the oracle's own gate
g = g_min Sigmoid(e^A z), on both prefill paths and the segmented path."""
import pytest
import torch

from gated_delta_rule_117_b200 import kda, synth
from parity_util import TOL, f64, rel_l2, to_dev

import oracle

pytestmark = pytest.mark.gpu


def _check(w, chunk_size=0, tol_key="bf16", g_min=-5.0):
    x = synth.prefill_inputs(w)
    gi = synth.gate_inputs(w)
    d = to_dev(x)
    z, A = gi["z"].cuda(), gi["A_log"].cuda()
    o, hT = kda.chunk_fwd_gated(d["q"], d["k"], d["v"], z, A, d["beta"], d["h0"], g_min=g_min,
                                chunk_size=chunk_size)
    assert kda.kda_get_device_status() == 0
    g = oracle.gate(f64(gi["z"]), gi["A_log"].double().numpy(), g_min)
    o_ref, h_ref = oracle.recurrent(f64(x["q"]), f64(x["k"]), f64(x["v"]), g, f64(x["beta"]), f64(x["h0"]))
    assert rel_l2(o, o_ref) <= TOL[tol_key] and rel_l2(hT, h_ref) <= TOL[tol_key]


def test_tensor_core_path_single_pass():
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=2, H=3, T=333, seed=61)
    assert kda.kda_chunk_fwd_plan(w.B, w.H, w.T, 128, 128, kda.KDA_DTYPE_BF16, 0)["path"] == kda.KDA_PATH_TC32
    _check(w)


def test_tensor_core_path_segmented_fast_heads():
    # few chains (segmented call), heads whose decay sits near the bound
    w = synth.WORKLOADS["batched_b8_h32_t8k"].with_(B=1, H=16, T=1500, seed=62)
    assert kda.kda_chunk_fwd_plan(w.B, w.H, w.T, 128, 128, kda.KDA_DTYPE_BF16, 0)["segments"] > 1
    _check(w)


def test_cuda_core_path_fp32():
    w = synth.WORKLOADS["tiny_f32"].with_(T=130, h0_std=0.02, seed=63)
    _check(w, chunk_size=16, tol_key="f32")


def test_other_bound():
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=2, T=200, seed=64)
    _check(w, g_min=-2.0)
