"""kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot
allocate device memory (no workspace argument; libkda's fixed device scratch
array stands in for it).  Checked through the C ABI against kda_chunk_fwd with
a caller-allocated workspace, on two calls in a row.  Kept in its own file,
collected last, so a failure here does not hide the other tests' results."""
import pytest
import torch

from gated_delta_rule_117_b200 import kda, synth
from parity_util import TOL, oracle_prefill, rel_l2

pytestmark = pytest.mark.gpu


def _inputs(seed):
    # few chains, enough tokens: the planner splits chains into segments, so
    # the call needs scratch memory
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=8, T=1100, seed=seed)
    x = synth.prefill_inputs(w)
    return w, {k: v.cuda() for k, v in x.items()}


def _noalloc(w, d):
    o = torch.empty(w.B, w.H, w.T, w.dv, dtype=torch.bfloat16, device="cuda")
    hT = torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32, device="cuda")
    st = kda.kda_chunk_fwd_noalloc(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["g"].data_ptr(),
                                   d["beta"].data_ptr(), d["h0"].data_ptr(), o.data_ptr(), hT.data_ptr(), w.B, w.H,
                                   w.T, w.dk, w.dv, kda.KDA_DTYPE_BF16, 0, 0.0,
                                   torch.cuda.current_stream().cuda_stream)
    assert st == 0, kda.kda_status_string(st)
    assert kda.kda_get_device_status() == 0
    return o, hT


def test_noalloc_matches_workspace_entry_point_twice():
    w, _ = _inputs(301)
    plan = kda.kda_chunk_fwd_plan(w.B, w.H, w.T, w.dk, w.dv, kda.KDA_DTYPE_BF16, 0)
    assert plan["segments"] > 1 and 0 < plan["workspace"] <= kda.kda_noalloc_scratch_bytes()
    for seed in (301, 302):  # two calls in a row share (and reuse) the scratch array
        w, d = _inputs(seed)
        o_n, h_n = _noalloc(w, d)
        o_w, h_w = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
        torch.cuda.synchronize()
        # both calls run the same plan and kernels, which are deterministic: the
        # results must agree bit for bit (stale scratch from the previous call
        # would show up here)
        assert torch.equal(o_n, o_w) and torch.equal(h_n, h_w)
    # the second call, whose scratch the first one had filled, against the oracle
    x = {k: v.cpu() for k, v in d.items()}
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o_n, o_ref) <= TOL["bf16"] and rel_l2(h_n, h_ref) <= TOL["bf16"]


def test_noalloc_rejects_bad_sizes_before_device_work():
    # invalid sizes are reported like kda_chunk_fwd reports them
    assert kda.kda_chunk_fwd_noalloc(None, None, None, None, None, None, None, None, 1, 1, 64, 24, 128,
                                     kda.KDA_DTYPE_BF16, 0, 0.0, None) == 2
