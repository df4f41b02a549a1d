"""GPU parity of kda_chunk_fwd against the fp64 oracle on the same seeded
inputs: relative L2 error <= 1e-5 for fp32 inputs and <= 3e-3 (o and h_T) for
bf16 inputs, at small sizes spanning several chunks plus ragged tails, at the
full workload sizes (oracle on sampled heads), and on the edge cases."""
import numpy as np
import pytest
import torch

from gated_delta_rule_117_b200 import kda, synth
from parity_util import TOL, f64, oracle_prefill, rel_l2, to_dev

import oracle

pytestmark = pytest.mark.gpu


def _run(x, chunk_size=0, use_h0=True, scale=0.0, **kw):
    d = to_dev(x)
    out = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"] if use_h0 else None,
                        chunk_size=chunk_size, scale=scale, **kw)
    assert kda.kda_get_device_status() == 0  # no bounded wait gave up
    return out


def test_tiny_f32_workload():
    w = synth.WORKLOADS["tiny_f32"]
    x = synth.prefill_inputs(w)
    o, hT = _run(x, chunk_size=w.chunk, use_h0=False)
    o_ref, h_ref = oracle_prefill(x, h0=False)
    assert rel_l2(o, o_ref) <= TOL["f32"]
    assert rel_l2(hT, h_ref) <= TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 16), (16, 128), (128, 128)])
@pytest.mark.parametrize("T", [1, 15, 16, 47, 130])
def test_shapes_and_ragged_tails(dtype, dk, dv, T):
    w = synth.WORKLOADS["tiny_f32"].with_(dtype=dtype, B=2, H=3, T=T, dk=dk, dv=dv, h0_std=0.02, seed=77)
    x = synth.prefill_inputs(w)
    o, hT = _run(x)
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL[dtype]
    assert rel_l2(hT, h_ref) <= TOL[dtype]


@pytest.mark.parametrize("chunk", [16, 32])
@pytest.mark.parametrize("T", [1, 15, 16, 31, 32, 33, 64, 100, 257])
def test_bf16_d128_both_paths(chunk, T):
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=2, H=2, T=T, seed=91)
    x = synth.prefill_inputs(w)
    o, hT = _run(x, chunk_size=chunk)
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL["bf16"]
    assert rel_l2(hT, h_ref) <= TOL["bf16"]


def test_fast_decay_heads_both_paths():
    # heads whose g sits at the -5 bound: 16-token windows reach -80
    w = synth.WORKLOADS["batched_b8_h32_t8k"].with_(B=1, T=512)
    fast = synth.fast_decay_heads(w).tolist()
    x = synth.prefill_inputs(w)
    x = {k: v[:, fast].contiguous() for k, v in x.items()}
    o_ref, h_ref = oracle_prefill(x, h0=False)
    for chunk in (16, 32):
        o, hT = _run(x, chunk_size=chunk, use_h0=False)
        assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"], chunk


@pytest.mark.parametrize("T", [300, 1100])
def test_decay_at_the_bound(T):
    # g = g_min = -5 on every token of half the key channels: each 16-token
    # window there sums to exactly -80, the widest range one reference point
    # per 32-token chunk has to carry (T = 1100 also runs the segmented path)
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=4, T=T, seed=5)
    x = synth.prefill_inputs(w)
    g = x["g"].clone()
    g[..., :64] = -5.0
    x["g"] = g
    o, hT = _run(x)
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]


@pytest.mark.parametrize("B,H,T", [(1, 16, 2305), (1, 2, 2304), (2, 3, 1100), (1, 74, 600)])
def test_in_device_context_parallel(B, H, T):
    # few chains and enough tokens: the call splits every chain into segments
    # (transition pass, scan, final pass); results must match the recurrence
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=B, H=H, T=T, seed=123)
    plan = kda.kda_chunk_fwd_plan(B, H, T, 128, 128, kda.KDA_DTYPE_BF16, 0)
    assert plan["segments"] > 1 and plan["launches"] == 4 and plan["workspace"] > 0
    x = synth.prefill_inputs(w)
    o, hT = _run(x)
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]


@pytest.mark.parametrize("g_scale", [1.0, 0.05])
def test_in_device_context_parallel_vanishing_and_persistent_transitions(g_scale):
    # at the workloads' decay every segment's transition M underflows to exactly zero
    # (the M runs stop early and the scan skips them); with decays 20x slower M stays
    # nonzero over a 256-token segment (~e^-32) and the scan multiplies by it
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=8, T=2304, seed=141)
    x = synth.prefill_inputs(w)
    x["g"] = (x["g"].float() * g_scale).to(x["g"].dtype)
    plan = kda.kda_chunk_fwd_plan(1, 8, 2304, 128, 128, kda.KDA_DTYPE_BF16, 0)
    assert plan["segments"] > 1
    o, hT = _run(x)
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]


def test_in_device_context_parallel_transition_windows():
    # The first transition pass covers only the last 128 tokens of each 256-token
    # segment; a segment whose window transition vanished keeps the window's (S~, M),
    # the others run again in full.  Per head: both halves fast (window final);
    # both slow (full run, M persists); fast head, slow window (full run, whose M
    # vanishes); slow head, fast window (window final).  Each head must match the
    # oracle on its own.
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=4, T=2304, seed=143)
    plan = kda.kda_chunk_fwd_plan(1, 4, 2304, 128, 128, kda.KDA_DTYPE_BF16, 0)
    assert plan["segments"] == 9 and plan["segment_tokens"] == 256
    x = synth.prefill_inputs(w)
    in_window = (torch.arange(w.T) % 256) >= 128
    scale = torch.ones(w.H, w.T)
    scale[1] = 0.05
    scale[2, in_window] = 0.05
    scale[3, ~in_window] = 0.05
    x["g"] = (x["g"].float() * scale[None, :, :, None]).to(x["g"].dtype)
    o, hT = _run(x)
    o_ref, h_ref = oracle_prefill(x)
    for h in range(w.H):
        assert rel_l2(o[:, h], o_ref[:, h]) <= TOL["bf16"], h
        assert rel_l2(hT[:, h], h_ref[:, h]) <= TOL["bf16"], h


def test_context_parallel_inplace_state_and_missing_workspace():
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=1, H=8, T=1024, seed=5)
    x = synth.prefill_inputs(w)
    d = to_dev(x)
    assert kda.kda_chunk_fwd_plan(1, 8, 1024, 128, 128, kda.KDA_DTYPE_BF16, 0)["segments"] > 1
    o_ref, h_ref = oracle_prefill(x)
    h = d["h0"].clone()
    o, _ = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h, h_T=h)
    assert kda.kda_get_device_status() == 0
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(h, h_ref) <= TOL["bf16"]
    ws = kda.kda_chunk_fwd_workspace_size(1, 8, 1024, 128, 128, kda.KDA_DTYPE_BF16, 0)
    st = kda.kda_chunk_fwd(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["g"].data_ptr(),
                           d["beta"].data_ptr(), None, o.data_ptr(), None, 1, 8, 1024, 128, 128,
                           kda.KDA_DTYPE_BF16, 0, 0.0, None, 0, None)
    assert st == 6  # KDA_ERR_WORKSPACE
    small = torch.empty(ws - 16, dtype=torch.uint8, device="cuda")
    st = kda.kda_chunk_fwd(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["g"].data_ptr(),
                           d["beta"].data_ptr(), None, o.data_ptr(), None, 1, 8, 1024, 128, 128,
                           kda.KDA_DTYPE_BF16, 0, 0.0, small.data_ptr(), small.numel(), None)
    assert st == 6


def test_prefill_workload_reduced_T():
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(T=700)
    x = synth.prefill_inputs(w)
    o, hT = _run(x)
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]


def test_prefill_workload_full():
    w = synth.WORKLOADS["prefill_h16_t4k"]
    x = synth.prefill_inputs(w)
    o, hT = _run(x)
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]


def _chain_errors(o, hT, o_ref, h_ref, chains, seg_len=None):
    """Per-chain relative L2 of o and h_T (and the worst per-segment value of o
    when seg_len is given) for the sampled chains; printed with the margin."""
    rows = []
    for i, (b, h) in enumerate(chains):
        ob, hb = o[b, h].cpu(), hT[b, h].cpu()
        eo, eh = rel_l2(ob, o_ref[i]), rel_l2(hb, h_ref[i])
        seg = 0.0
        if seg_len:
            T = ob.shape[0]
            seg = max(rel_l2(ob[s:s + seg_len], o_ref[i][s:s + seg_len]) for s in range(0, T, seg_len))
        rows.append((b, h, eo, eh, seg))
        print("chain (%d, %d): o %.3e  h_T %.3e  worst segment %.3e  (tol %.0e)" % (b, h, eo, eh, seg, TOL["bf16"]))
    return rows


def test_batched_workload_full_sampled_heads():
    # 16 of the 256 chains, every fast-decay head among them, each checked on its own
    import os
    w = synth.WORKLOADS["batched_b8_h32_t8k"]
    x = synth.prefill_inputs_parallel(w, workers=min(os.cpu_count() or 1, 16))
    o, hT = _run(x, use_h0=False)
    fast = synth.fast_decay_heads(w).tolist()
    assert len(fast) == 3
    rng = np.random.default_rng(2024)
    heads = [(b, h) for b, h in zip([0, 3, 7], fast)]
    while len(heads) < 16:
        c = (int(rng.integers(w.B)), int(rng.integers(w.H)))
        if c not in heads:
            heads.append(c)
    o_ref, h_ref = oracle_prefill(x, heads=heads, h0=False)
    rows = _chain_errors(o, hT, o_ref, h_ref, heads)
    assert max(max(r[2], r[3]) for r in rows) <= TOL["bf16"]
    assert torch.isfinite(o).all() and torch.isfinite(hT).all()


def test_long_workload_reduced_T():
    w = synth.WORKLOADS["long_h16_t1m"].with_(T=1 << 15, H=4)
    x = synth.prefill_inputs(w)
    o, hT = _run(x, use_h0=False)
    o_ref, h_ref = oracle_prefill(x, h0=False)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]


def test_long_workload_full_sampled_heads():
    # the 1M-token workload at full size (16 chains, the context-parallel plan
    # the benchmark times); the oracle recomputes three whole chains (every
    # chain's last segment writes its h_T), each checked on its own and per
    # segment, so one wrong segment boundary cannot hide in the average
    import os
    w = synth.WORKLOADS["long_h16_t1m"]
    x = synth.prefill_inputs_parallel(w, workers=min(os.cpu_count() or 1, 16))
    o, hT = _run(x, use_h0=False)
    plan = kda.kda_chunk_fwd_plan(w.B, w.H, w.T, 128, 128, kda.KDA_DTYPE_BF16, 0)
    assert plan["segments"] > 1
    heads = [(0, 0), (0, 7), (0, 15)]
    o_ref, h_ref = oracle_prefill(x, heads=heads, h0=False)
    rows = _chain_errors(o, hT, o_ref, h_ref, heads, seg_len=plan["segment_tokens"])
    assert max(max(r[2], r[3], r[4]) for r in rows) <= TOL["bf16"]
    assert torch.isfinite(o).all() and torch.isfinite(hT).all()


@pytest.mark.parametrize("dtype,d", [("f32", 16), ("bf16", 128)])
def test_zero_length_copies_state(dtype, d):
    # bf16 with d = 128 is the tensor-core plan: T = 0 must still copy h0 to h_T
    w = synth.WORKLOADS["tiny_f32"].with_(T=0, h0_std=0.02, dtype=dtype, dk=d, dv=d, B=2, H=3)
    x = synth.prefill_inputs(w)
    if dtype == "bf16":
        assert kda.kda_chunk_fwd_plan(2, 3, 0, d, d, kda.KDA_DTYPE_BF16, 0)["path"] == kda.KDA_PATH_TC32
    o, hT = _run(x)
    assert o.numel() == 0 and torch.equal(hT.cpu(), x["h0"])
    o, hT = _run(x, use_h0=False)
    assert torch.count_nonzero(hT) == 0


def test_inplace_state_and_no_final_state():
    w = synth.WORKLOADS["tiny_f32"].with_(T=40, h0_std=0.02, dtype="bf16", dk=32, dv=32)
    x = synth.prefill_inputs(w)
    d = to_dev(x)
    o_ref, h_ref = oracle_prefill(x)
    h = d["h0"].clone()
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h, h_T=h)
    assert hT.data_ptr() == h.data_ptr()
    assert rel_l2(h, h_ref) <= TOL["bf16"] and rel_l2(o, o_ref) <= TOL["bf16"]
    o2, none = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], output_final_state=False)
    assert none is None and torch.equal(o2, o)


def test_explicit_scale():
    w = synth.WORKLOADS["tiny_f32"].with_(T=33, h0_std=0.02)
    x = synth.prefill_inputs(w)
    o, _ = _run(x, scale=0.5)
    o_ref, _ = oracle_prefill(x, scale=0.5)
    assert rel_l2(o, o_ref) <= TOL["f32"]


def test_state_split_resume_on_gpu():
    # run(T) == run(T1) then run(T - T1) from h_T1, on the device path itself
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(T=256, H=2)
    x = synth.prefill_inputs(w)
    d = to_dev(x)
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    T1 = 100
    sl = lambda t, a, b: t[:, :, a:b].contiguous()
    o1, h1 = kda.chunk_fwd(*(sl(d[n], 0, T1) for n in ("q", "k", "v", "g", "beta")), d["h0"])
    o2, h2 = kda.chunk_fwd(*(sl(d[n], T1, 256) for n in ("q", "k", "v", "g", "beta")), h1)
    o_ref, h_ref = oracle_prefill(x)
    assert rel_l2(torch.cat([o1, o2], 2), o_ref) <= TOL["bf16"] and rel_l2(o, o_ref) <= TOL["bf16"]
    assert rel_l2(h2, h_ref) <= TOL["bf16"] and rel_l2(hT, h_ref) <= TOL["bf16"]


@pytest.mark.parametrize("T", [300, 1100])  # one CTA per chain; segmented plan
def test_deterministic(T):
    # the roles hand data over through shared and tensor memory; a missing wait or
    # barrier usually shows up as run-to-run differences, so results must be bitwise stable
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(T=T, H=4)
    x = synth.prefill_inputs(w)
    o1, h1 = _run(x)
    for _ in range(3):
        o2, h2 = _run(x)
        assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_misaligned_pointer_is_rejected():
    w = synth.WORKLOADS["tiny_f32"].with_(T=16)
    d = to_dev(synth.prefill_inputs(w))
    buf = torch.empty(d["q"].numel() + 4, device="cuda")
    qm = buf[1:1 + d["q"].numel()].view_as(d["q"])
    with pytest.raises(kda.KdaError) as e:
        kda.chunk_fwd(qm, d["k"], d["v"], d["g"], d["beta"], None)
    assert e.value.status == 4
    assert kda.kda_get_device_status() == 0


@pytest.mark.parametrize("B,H,T", [(1, 16, 4096), (4, 37, 700)])
def test_back_to_back_calls_record_no_timeout(B, H, T):
    # the roles of the tensor-core kernel hand chunks over through mbarrier phases;
    # a wait on a phase that can alias (complete twice before it is observed) stalls
    # until its bounded wait gives up.  Such a race is timing-dependent, so run many
    # calls back to back and require that none recorded a timeout, and that the
    # calls take normal time (a stall costs the 2 s wait limit)
    import time
    w = synth.WORKLOADS["prefill_h16_t4k"].with_(B=B, H=H, T=T, seed=131)
    d = to_dev(synth.prefill_inputs(w))
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    assert kda.kda_get_device_status() == 0
    t0 = time.perf_counter()
    for _ in range(40):
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], o=o, h_T=hT)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    assert time.perf_counter() - t0 < 1.0
