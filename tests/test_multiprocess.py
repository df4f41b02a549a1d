"""The multi-rank bench logic on CPU (gloo, world size 2): every rank runs an
independent replica on its own inputs, the job time is the max over ranks, and
the throughput counts all ranks' tokens."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from gated_delta_rule_117_b200 import synth
        w = bench.rank_workload(synth.WORKLOADS["prefill_h16_t4k"], rank)
        x = synth.head_inputs(w, 0, 0, T=8)
        local_ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(local_ms, dist)
        out[rank] = (w.seed, float(x["q"][0, 0]), mx, bench.job_throughput(1000, world, mx))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    (s0, q0, m0, v0), (s1, q1, m1, v1) = out[0], out[1]
    assert s0 != s1 and q0 != q1          # independent replicas, different inputs
    assert m0 == m1 == 15.0               # slowest rank's time on every rank
    assert v0 == v1 == pytest.approx(2 * 1000 / 0.015)


def test_single_process_helpers():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(4096, 1, 2.0) == pytest.approx(4096 / 0.002)


# ---- cross-device KCP orchestration (gloo, 2 ranks, CPU stand-ins) ----------

class _OracleOps:
    """The KCP steps on the CPU with the fp64 oracle (test stand-ins for the
    device kernels): the orchestration, not the arithmetic, is under test."""

    @staticmethod
    def transition_packed(q, k, v, g, beta, scale=0.0):
        import numpy as np
        import oracle
        from gated_delta_rule_117_b200 import kcp
        a = [t.double().numpy() for t in (q, k, v, g, beta)]
        _, st = oracle.recurrent(*a)
        B, H = q.shape[:2]
        m = np.stack([np.stack([oracle.transition(a[1][b, h], a[3][b, h], a[4][b, h]) for h in range(H)])
                      for b in range(B)])
        return kcp.pack(torch.from_numpy(m), torch.from_numpy(st))

    @staticmethod
    def compose(ms, sts, h0, like):
        s = torch.zeros_like(like, dtype=torch.float64) if h0 is None else h0.double().clone()
        for m, st in zip(ms, sts):
            s = m @ s + st
        return s

    @staticmethod
    def prefill(q, k, v, g, beta, h0, scale=0.0):
        import oracle
        a = [t.double().numpy() for t in (q, k, v, g, beta)]
        o, hT = oracle.recurrent(*a, h0.double().numpy())
        return torch.from_numpy(o), torch.from_numpy(hT)


def _kcp_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from gated_delta_rule_117_b200 import kcp, synth
        w = synth.WORKLOADS["tiny_f32"].with_(H=2, T=90, h0_std=0.05, seed=21)
        x = synth.prefill_inputs(w)
        n = w.T // world
        sl = {k2: (x[k2][:, :, rank * n:(rank + 1) * n] if k2 != "h0" else x[k2]) for k2 in x}
        calls = []
        real = dist.all_gather
        dist.all_gather = lambda *a, **kw: (calls.append(1), real(*a, **kw))[1]
        try:
            o, hT = kcp.kcp_prefill(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], x["h0"], ops=_OracleOps)
        finally:
            dist.all_gather = real
        assert len(calls) == 1  # one exchange of the packed (M, S~) pairs
        out[rank] = (o.numpy(), hT.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_cross_device_kcp_orchestration(world):
    import numpy as np
    import oracle
    from gated_delta_rule_117_b200 import synth
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_kcp_worker, args=(world, port, out), nprocs=world, join=True)
    w = synth.WORKLOADS["tiny_f32"].with_(H=2, T=90, h0_std=0.05, seed=21)
    x = synth.prefill_inputs(w)
    o_ref, h_ref = oracle.recurrent(*[x[n].double().numpy() for n in ("q", "k", "v", "g", "beta", "h0")])
    o = np.concatenate([out[r][0] for r in range(world)], axis=2)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)               # rank r's tokens, in rank order
    np.testing.assert_allclose(out[world - 1][1], h_ref, rtol=1e-10, atol=1e-12)  # last rank: the final state
