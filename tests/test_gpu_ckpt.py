"""State checkpoints for prefix caching (Kimi K3 report, section 5.4.1):
kda_chunk_fwd_ckpt against the oracle's prefix states, on both prefill paths
and through the segmented (context-parallel) path, plus the use the report
makes of them: prefill resumed from a snapshot reproduces the rest of the run."""
import pytest
import torch

from gated_delta_rule_117_b200 import kda, synth
from parity_util import TOL, f64, oracle_prefill, rel_l2, to_dev

import oracle

pytestmark = pytest.mark.gpu


def _oracle_ckpt(x, interval, h0=True):
    return oracle.checkpoints(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]),
                              f64(x["h0"]) if h0 else None, interval=interval)


def _check(w, interval, chunk_size=0, tol_key="bf16"):
    x = synth.prefill_inputs(w)
    d = to_dev(x)
    o, hT, ck = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], chunk_size=chunk_size,
                              ckpt_interval=interval)
    assert kda.kda_get_device_status() == 0
    assert ck.shape == (w.B, w.H, w.T // interval, w.dk, w.dv)
    ref = _oracle_ckpt(x, interval)
    for j in range(w.T // interval):
        assert rel_l2(ck[:, :, j], ref[:, :, j]) <= TOL[tol_key], j
    # emitting checkpoints leaves o and h_T bit for bit unchanged
    o2, h2 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], chunk_size=chunk_size)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(hT, h2)
    return x, d, ck


def test_tensor_core_path_single_pass():
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=2, H=3, T=700, seed=41)
    plan = kda.kda_chunk_fwd_plan(w.B, w.H, w.T, 128, 128, kda.KDA_DTYPE_BF16, 0)
    assert plan["path"] == kda.KDA_PATH_TC32
    _check(w, 128)


def test_tensor_core_path_segmented():
    # few chains: the call splits each chain into segments; checkpoints fall on
    # and between segment boundaries
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=2, T=2304, seed=42)
    plan = kda.kda_chunk_fwd_plan(w.B, w.H, w.T, 128, 128, kda.KDA_DTYPE_BF16, 0)
    assert plan["segments"] > 1
    _check(w, 256)


def test_cuda_core_path_fp32():
    w = synth.WORKLOADS["tiny_f32"].with_(T=200, h0_std=0.02, seed=43)
    _check(w, 64, chunk_size=16, tol_key="f32")


def test_resume_from_checkpoint():
    # section 5.4.1: a request sharing the first p tokens copies the snapshot at p
    # and resumes prefill from token p
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=4, T=640, seed=44)
    x, d, ck = _check(w, 256)
    o_ref, h_ref = oracle_prefill(x)
    for j in range(ck.shape[2]):
        p = (j + 1) * 256
        tail = {n: d[n][:, :, p:].contiguous() for n in ("q", "k", "v", "g", "beta")}
        o2, h2 = kda.chunk_fwd(tail["q"], tail["k"], tail["v"], tail["g"], tail["beta"],
                               ck[:, :, j].contiguous())
        assert rel_l2(o2, o_ref[:, :, p:]) <= TOL["bf16"] and rel_l2(h2, h_ref) <= TOL["bf16"], j


def test_short_sequence_has_no_snapshot():
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=2, T=100, seed=45)
    x = synth.prefill_inputs(w)
    d = to_dev(x)
    o, hT, ck = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], ckpt_interval=128)
    assert ck.shape[2] == 0
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]
