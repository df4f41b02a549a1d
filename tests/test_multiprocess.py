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
