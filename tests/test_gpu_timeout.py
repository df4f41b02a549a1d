"""Failure detection without a GPU fault: a bounded wait of the tensor-core
prefill kernel is made to run out.  The injection is host-side: with a 20 ms
wait limit, the kernel's chain role first waits on a barrier that nothing ever
arrives on, so the wait gives up, the CTA aborts (drains its copies and MMAs,
releases its tensor memory, returns) and the timeout is recorded in the device
status word.  Nothing traps, faults or hangs; afterwards the same context must
run a normal call correctly."""
import pytest
import torch

from gated_delta_rule_117_b200 import kda, synth
from parity_util import TOL, oracle_prefill, rel_l2

pytestmark = pytest.mark.gpu

KDA_ERR_TIMEOUT = 8


@pytest.mark.parametrize("T", [200, 1100])  # one chain per CTA; segmented (context-parallel) plan
def test_wait_that_runs_out_reports_timeout_and_context_survives(T):
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=2, T=T, seed=41)
    plan = kda.kda_chunk_fwd_plan(w.B, w.H, w.T, 128, 128, kda.KDA_DTYPE_BF16, 0)
    assert plan["path"] == kda.KDA_PATH_TC32 and (plan["segments"] > 1) == (T > 1000)
    x = synth.prefill_inputs(w)
    d = {k: v.cuda() for k, v in x.items()}
    assert kda.kda_get_device_status() == 0
    kda.kda_debug_set_wait_limit(20_000_000)  # 20 ms
    kda.kda_debug_inject_stall(True)
    try:
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])  # enqueues fine
        st = kda.kda_get_device_status()  # synchronises; the kernel has returned
    finally:
        kda.kda_debug_inject_stall(False)
        kda.kda_debug_set_wait_limit(0)
    assert st == KDA_ERR_TIMEOUT, kda.kda_status_string(st)
    assert kda.kda_get_device_status() == 0  # reading the word cleared it
    # the context is intact: a normal call now gives correct results
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    assert kda.kda_get_device_status() == 0
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]
    torch.cuda.synchronize()
