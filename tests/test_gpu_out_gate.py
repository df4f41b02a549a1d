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
