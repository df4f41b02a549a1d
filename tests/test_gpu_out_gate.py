"""The output edge of a KDA layer (Kimi K3 report, section 2.1.1, Eq. 6):
kda_output_gate against the oracle's Sigmoid(gate) * RMSNorm(o), on the
vectorised bf16 d = 128 kernel, the generic kernel (other dv, fp32) and in place."""
import numpy as np
import pytest
import torch

from gated_delta_rule_117_b200 import kda
from parity_util import TOL, rel_l2

import oracle

pytestmark = pytest.mark.gpu


def _inputs(B, H, T, dv, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    o = torch.randn(B, H, T, dv, generator=g).to(dtype)
    gate = (2 * torch.randn(B, H, T, dv, generator=g)).to(dtype)
    w = (1 + 0.3 * torch.randn(H, dv, generator=g)).float()
    return o, gate, w


@pytest.mark.parametrize("B,H,T,dv,dtype,key", [
    (2, 16, 300, 128, torch.bfloat16, "bf16"),
    (1, 3, 29, 128, torch.bfloat16, "bf16"),  # 87 rows: a partial CTA, warps with rows past the end
    (1, 3, 77, 64, torch.bfloat16, "bf16"),
    (2, 2, 50, 16, torch.float32, "f32"),
    (1, 4, 33, 128, torch.float32, "f32"),
])
def test_matches_oracle(B, H, T, dv, dtype, key):
    o, gate, w = _inputs(B, H, T, dv, dtype, 11 + dv + T)
    y = kda.output_gate(o.cuda(), gate.cuda(), w.cuda(), 1e-6)
    torch.cuda.synchronize()
    ref = oracle.output_gate(o.double().numpy(), gate.double().numpy(), w.double().numpy(), 1e-6)
    assert rel_l2(y, ref) <= TOL[key]


def test_in_place():
    o, gate, w = _inputs(1, 2, 40, 128, torch.bfloat16, 5)
    ref = oracle.output_gate(o.double().numpy(), gate.double().numpy(), w.double().numpy(), 1e-5)
    od = o.cuda()
    y = kda.output_gate(od, gate.cuda(), w.cuda(), 1e-5, y=od)
    torch.cuda.synchronize()
    assert y.data_ptr() == od.data_ptr() and rel_l2(od, ref) <= TOL["bf16"]


def _edge_inputs(w, seed):
    g = torch.Generator().manual_seed(seed)
    gate = (2 * torch.randn(w.B, w.H, w.T, w.dv, generator=g)).to(w.torch_dtype)
    rw = (1 + 0.3 * torch.randn(w.H, w.dv, generator=g)).float()
    return gate, rw


@pytest.mark.parametrize("dtype,d,T,H", [
    ("bf16", 128, 100, 3),    # tensor-core path, one CTA per chain, ragged tail
    ("bf16", 128, 1100, 2),   # tensor-core path, context-parallel segments (final pass fused)
    ("bf16", 64, 70, 2),      # CUDA-core path (prefill into y, edge in place)
    ("f32", 16, 64, 2),       # CUDA-core path, fp32
])
def test_fused_output_edge_matches_oracle(dtype, d, T, H):
    # y = Sigmoid(gate) * RMSNorm_w(o), o the recurrence's output: oracle.output_gate of oracle.recurrent
    from gated_delta_rule_117_b200 import synth
    from parity_util import oracle_prefill
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(dtype=dtype, dk=d, dv=d, T=T, H=H, B=1, seed=202 + T)
    x = synth.prefill_inputs(w)
    gate, rw = _edge_inputs(w, 9 + T)
    dv_ = {k: v.cuda() for k, v in x.items()}
    y, hT = kda.chunk_fwd_outgate(dv_["q"], dv_["k"], dv_["v"], dv_["g"], dv_["beta"], gate.cuda(), rw.cuda(),
                                  dv_["h0"], eps=1e-6)
    assert kda.kda_get_device_status() == 0
    o_ref, h_ref = oracle_prefill(x)
    y_ref = oracle.output_gate(o_ref, gate.double().numpy(), rw.double().numpy(), 1e-6)
    key = "bf16" if dtype == "bf16" else "f32"
    assert rel_l2(y, y_ref) <= TOL[key] and rel_l2(hT, h_ref) <= TOL[key]
    if dtype == "bf16" and d == 128:
        plan = kda.kda_chunk_fwd_plan(1, H, T, 128, 128, kda.KDA_DTYPE_BF16, 0)
        assert plan["path"] == kda.KDA_PATH_TC32 and (plan["segments"] > 1) == (T > 1000)
        # the fused edge gives what the unfused pair of calls gives, up to the rounding of o to bf16
        o, _ = kda.chunk_fwd(dv_["q"], dv_["k"], dv_["v"], dv_["g"], dv_["beta"], dv_["h0"])
        y2 = kda.output_gate(o, gate.cuda(), rw.cuda(), 1e-6)
        torch.cuda.synchronize()
        assert rel_l2(y, y2.double().cpu().numpy()) <= TOL["bf16"]


def test_fused_output_edge_rejects_aliasing():
    from gated_delta_rule_117_b200 import synth
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(T=64, H=2, B=1)
    x = {k: v.cuda() for k, v in synth.prefill_inputs(w).items()}
    gate, rw = _edge_inputs(w, 3)
    gate = gate.cuda()
    with pytest.raises(kda.KdaError) as e:  # y written over its own gate input
        kda.chunk_fwd_outgate(x["q"], x["k"], x["v"], x["g"], x["beta"], gate, rw.cuda(), x["h0"], y=gate)
    assert e.value.status == 5
