#!/usr/bin/env python
"""Throughput of libkda's KDA forward on B200.

Default line: chunked prefill (kda_chunk_fwd) on the long-context workload
(B=1, H=16, T=2^20, dk=dv=128, bf16 inputs, fp32 state, h0 = 0; in-device
context parallelism over the 148 SMs), reported as tokens/s with algorithmic
TFLOP/s and the HBM roofline fraction of the prefill step.  The same line
carries:
  * `configs`: the other prefill workloads (B1 H16 T4096 with h0, B8 H32 T8192
    with fast-decay heads), each timed the same way with its own roofline and
    an oracle check of sampled whole chains;
  * `decode`: the decode step (kda_recurrent_step, B=256, H=32, 64 steps,
    state updated in place) as GB/s against the HBM peak;
  * `parity` and `cpu_baseline`: the fp64 oracle over whole sampled chains of
    the main workload (run on host cores while the GPU legs run), compared
    with the timed run's own output, and its throughput;
  * `e2e`: the same metric through the C ABI from pinned host buffers, every
    step's uploads and downloads inside the timed region, consecutive steps
    pipelined over two copy streams and two device buffer sets;
  * secondary legs (checkpoints, output gate, fused gate, replay).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl libkda|reference]

With --gpus N > 1 the script starts N ranks itself (torch.distributed.run)
unless a launcher already set WORLD_SIZE, which must then equal N.  Each rank
runs an independent replica of the workload (the (batch, head) chains are
independent: no collective on the data path), time is the max over ranks, and
value is the whole-job throughput.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s + TFLOP/s (% tensor peak); decode GB/s (% HBM) on 1 B200"
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_record(kernel: str, src_files):
    """ncu DRAM bytes per launch recorded under profiles/ for `kernel`, or None
    when the kernel's sources changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec:
        return None
    h = hashlib.sha256()
    for f in src_files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if rec.get("source_sha256") != h.hexdigest():
        return None
    return rec


class ClockSampler:
    """nvidia-smi SM clock / throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.dev = device_id  # nvidia-smi -i accepts the GPU UUID (robust to CUDA_VISIBLE_DEVICES)
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), "kda_bench_clocks_%d.csv" % os.getpid())

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def count(self):
        try:
            with open(self.path) as f:
                return sum(1 for line in f if line.count(",") >= 8)
        except OSError:
            return 0

    def soak(self, fn, torch, min_samples=3, max_s=4.0):
        """Run `fn` (the step, untimed) until nvidia-smi has logged a few
        samples: a timed region of a few milliseconds is far shorter than its
        sampling period, so the clock record spans this soak of the same work
        running right before the timed region, plus the timed region itself."""
        if self.proc is None:
            return
        t0 = time.time()
        while self.count() < min_samples and time.time() - t0 < max_s:
            for _ in range(10):
                fn()
            torch.cuda.synchronize()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "window": "soak of the same step just before the timed region, then the timed region"}


def rank_workload(w, rank):
    """Weak scaling: every rank runs its own replica of the workload on its own
    seeded inputs (the (b, h) chains are independent; nothing is exchanged)."""
    return w if rank == 0 else w.with_(seed=w.seed + 7919 * rank)


def max_over_ranks(value, dist=None, device=None):
    """Max of a per-rank scalar over all ranks (the job's time is the slowest rank's)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, max_ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


def gpu_uuid(torch, dev):
    u = str(torch.cuda.get_device_properties(dev).uuid)
    return u if u.startswith("GPU-") else "GPU-" + u


def cpu_oracle_prefill(w, x, threads):
    import oracle
    f = lambda t: t.double().numpy()
    h0 = f(x["h0"]) if w.h0_std > 0 else None
    args = [f(x[n]) for n in ("q", "k", "v", "g", "beta")]
    t0 = time.perf_counter()
    oracle.recurrent(*args, h0, nthreads=threads)
    return time.perf_counter() - t0


ORACLE_BLOCK = 1 << 16  # tokens per oracle call; the state is carried between calls


def _oracle_chain(job):
    """CPU-baseline leg, in a spawned worker: the fp64 oracle over one whole
    (b, h) chain of the host inputs, token block by token block with the state
    carried, into shared-memory o_ref / h_ref.  Returns the compute seconds."""
    import torch
    import oracle
    x, b, h, o_ref, h_ref, use_h0 = job
    T = x["q"].shape[2]
    S = x["h0"][b, h].double().numpy() if use_h0 else None
    secs = 0.0
    for s in range(0, T, ORACLE_BLOCK):
        e = min(T, s + ORACLE_BLOCK)
        f = lambda n: x[n][b, h, s:e].double().numpy()
        args = (f("q"), f("k"), f("v"), f("g"), f("beta"))
        t0 = time.perf_counter()
        o, S = oracle.recurrent(*args, S, nthreads=1)
        secs += time.perf_counter() - t0
        o_ref[s:e] = torch.from_numpy(o)
    if S is None:  # T == 0
        S = x["h0"][b, h].double().numpy() if use_h0 else 0.0 * x["h0"][b, h].double().numpy()
    h_ref.copy_(torch.from_numpy(S))
    return secs


class OracleLeg:
    """The oracle on whole sampled chains of a workload's host inputs.  It is
    the CPU baseline (the oracle as it stands, one core per chain, compute time
    only) and, compared with the GPU output of the timed run, the parity check
    of that run.  Started in spawned processes before the GPU work so the CPU
    time overlaps it."""

    def __init__(self, w, x, chains, workers):
        import torch
        self.w, self.chains = w, chains
        self.o_ref = [torch.empty(w.T, w.dv, dtype=torch.float64).share_memory_() for _ in chains]
        self.h_ref = [torch.empty(w.dk, w.dv, dtype=torch.float64).share_memory_() for _ in chains]
        ctx = torch.multiprocessing.get_context("spawn")
        self.pool = ctx.Pool(max(1, min(workers, len(chains))))
        self.t0 = time.perf_counter()
        self.res = [self.pool.apply_async(_oracle_chain, ((x, b, h, o, hr, w.h0_std > 0),))
                    for (b, h), o, hr in zip(chains, self.o_ref, self.h_ref)]

    def finish(self, o_gpu, h_gpu, seg_len):
        """o_gpu [n, T, dv], h_gpu [n, dk, dv]: the timed run's output on the sampled chains (host)."""
        import numpy as np
        secs = [r.get() for r in self.res]
        wall = time.perf_counter() - self.t0
        self.pool.close()
        self.pool.join()
        eo, eh, seg_worst = [], [], 0.0
        for i in range(len(self.chains)):
            ref = self.o_ref[i].numpy()
            got = o_gpu[i].double().numpy()
            eo.append(rel_l2_np(got, ref))
            eh.append(rel_l2_np(h_gpu[i].double().numpy(), self.h_ref[i].numpy()))
            for s in range(0, self.w.T, seg_len):
                seg_worst = max(seg_worst, rel_l2_np(got[s:s + seg_len], ref[s:s + seg_len]))
        tol = 3e-3 if self.w.dtype == "bf16" else 1e-5
        parity = {"chains": [list(c) for c in self.chains], "o_rel_l2": eo, "hT_rel_l2": eh,
                  "o_rel_l2_worst_segment": seg_worst, "segment_tokens": seg_len, "tol": tol,
                  "pass": bool(max(eo + eh + [seg_worst]) <= tol),
                  "reference": "fp64 C token recurrence (oracle) over each whole chain"}
        n = len(self.chains)
        cpu = {"value": n * self.w.T / max(secs) / self.w.H, "unit": "tokens/s", "cores": n, "kind": "oracle",
               "sample": "%d whole chains (b, h) = %s of %d tokens, one core each, compute time of the slowest; "
                         "tokens/s of the workload = chain-tokens/s / H; ran while the GPU legs ran (wall %.1f s)"
                         % (n, [list(c) for c in self.chains], self.w.T, wall)}
        return parity, cpu


def rel_l2_np(x, ref):
    import numpy as np
    den = float(np.linalg.norm(ref))
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def sample_chains(w):
    """Chains whose whole output the oracle recomputes: first, last and a middle
    one; in a workload with fast-decay heads, those heads as well."""
    from gated_delta_rule_117_b200 import synth
    c = [(0, 0), (w.B - 1, w.H - 1)]
    if w.B * w.H > 2:
        c.insert(1, (w.B // 2, w.H // 3))
    for h in synth.fast_decay_heads(w).tolist()[:2]:
        c.append((min(1, w.B - 1), h))
    out = []
    for x in c:
        if x not in out:
            out.append(x)
    return out


def host_inputs(synth, w, world):
    """Seeded host inputs of a prefill workload; large ones are generated by a
    pool of spawned processes into shared memory (same values bit for bit)."""
    if w.B * w.H * w.T <= (1 << 20):
        return synth.prefill_inputs(w)
    workers = max(1, min(16, (os.cpu_count() or 1) // max(1, world)))
    return synth.prefill_inputs_parallel(w, workers=workers)


def time_prefill(args, w, d, plan, kda, torch, flush, dev, clk=None, dist=None):
    """CUDA-event time of each of args.steps kda_chunk_fwd calls on device-resident
    inputs, L2 flushed (outside the events) before each; W untimed warm-ups.
    Returns (per-step ms, o, h_T)."""
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    h0 = d["h0"] if w.h0_std > 0 else None
    o = torch.empty(B, H, T, dv, dtype=w.torch_dtype, device=dev)
    hT = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    ws = torch.empty(max(plan["workspace"], 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    ptr = lambda t: None if t is None else t.data_ptr()

    def step():
        st = kda.kda_chunk_fwd(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["g"]), ptr(d["beta"]), ptr(h0),
                               ptr(o), ptr(hT), B, H, T, dk, dv, dt, args.chunk_size, 0.0, ws.data_ptr(),
                               ws.numel(), sp)
        if st != 0:
            raise kda.KdaError(st, "kda_chunk_fwd")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if clk is not None:
        clk.soak(lambda: (flush.zero_(), step()), torch)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()  # L2 flush between timed iterations (outside the events)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    check_device_status(kda, "kda_chunk_fwd")
    return [a.elapsed_time(b) for a, b in ev], o, hT


def check_device_status(kda, what):
    """A timed run whose kernels recorded an error (a bounded wait that gave up)
    is not a measurement: raise instead of reporting its time."""
    st = kda.kda_get_device_status(None)
    if st != 0:
        raise kda.KdaError(st, what + " (device status after the timed steps)")


def prefill_figures(w, plan, ms, pk, pk_kind, synth):
    """Throughput, algorithmic TFLOP/s and the HBM roofline of one prefill step."""
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    nbytes = synth.prefill_bytes(w)
    achieved = nbytes / (ms / 1e3) / 1e9
    flop_tok = synth.flops_per_token_head(dk, dv, 64)
    tflops = flop_tok * B * H * T / (ms / 1e3) / 1e12
    kernel = "chunk16_kernel" if plan["path"] == 1 else "chunk_tc_kernel"
    # With in-device context parallelism one step is four launches (the two
    # segment-transition passes, the prefix scan, the final pass); the roofline
    # then uses the whole step's time, which is the conservative reading.
    scope = "kernel" if plan["launches"] == 1 else "step (%d launches)" % plan["launches"]
    src = (["gated_delta_rule_117_b200/csrc/kda_chunk_simt.cu"] if plan["path"] == 1
           else ["gated_delta_rule_117_b200/csrc/kda_chunk_tc.cu"])
    trec = traffic_record("%s:%s" % (kernel, w.name), src)
    traffic = None
    if trec:
        # a segmented step records the DRAM bytes of all its launches, like `achieved`
        traffic = trec.get("dram_bytes_per_step", trec.get("dram_bytes_per_launch"))
    return {
        "tokens_per_s": B * T / (ms / 1e3),
        "tflops": {"value": tflops, "flop_per_token_head": flop_tok, "frac_of_bf16_peak": tflops / pk["bf16_tflops"],
                   "peak_kind": pk_kind},
        "roofline": {"kernel": kernel, "scope": scope, "bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                     "algorithmic_bytes_per_launch": nbytes, "peak_kind": pk_kind, "kernel_ms": ms},
    }


def measure_subconfig(args, name, synth, kda, torch, dev, flush, pk, pk_kind, world):
    """Another prefill workload, timed like the main line, with the oracle on
    sampled whole chains (in process: these chains are short)."""
    import oracle
    w = synth.WORKLOADS[name]
    x = host_inputs(synth, w, world)
    d = {k: v.to(dev) for k, v in x.items()}
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    plan = kda.kda_chunk_fwd_plan(w.B, w.H, w.T, w.dk, w.dv, dt, args.chunk_size)
    times, o, hT = time_prefill(args, w, d, plan, kda, torch, flush, dev)
    ms = statistics.mean(times)
    res = {"workload": name, "B": w.B, "H": w.H, "T": w.T, "segments": plan["segments"],
           "launches_per_step": plan["launches"], "ms_per_step": ms, "steps": args.steps}
    res.update(prefill_figures(w, plan, ms, pk, pk_kind, synth))
    chains = sample_chains(w)
    f = lambda t: t.double().numpy()
    eo, eh = [], []
    for b, h in chains:
        o_ref, h_ref = oracle.recurrent(f(x["q"][b, h]), f(x["k"][b, h]), f(x["v"][b, h]), f(x["g"][b, h]),
                                        f(x["beta"][b, h]), f(x["h0"][b, h]) if w.h0_std > 0 else None)
        eo.append(rel_l2_np(f(o[b, h].cpu()), o_ref))
        eh.append(rel_l2_np(f(hT[b, h].cpu()), h_ref))
    res["parity"] = {"chains": [list(c) for c in chains], "o_rel_l2": eo, "hT_rel_l2": eh, "tol": 3e-3,
                     "pass": bool(max(eo + eh) <= 3e-3)}
    del d, o, hT
    return res


def relaunch_under_torchrun(n):
    """`--gpus N` without a launcher: start N ranks of this same command."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


SUBCONFIGS = ("prefill_h16_t4k", "batched_b8_h32_t8k")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_h16_t1m")
    ap.add_argument("--impl", default="libkda", choices=["libkda", "reference"])
    ap.add_argument("--chunk-size", type=int, default=0)
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the workload's T (smaller slices for profiling; 0 = the workload's own)")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle leg (baseline and parity)")
    ap.add_argument("--no-subconfigs", action="store_true", help="skip the other prefill workloads")
    ap.add_argument("--no-legs", action="store_true", help="skip the secondary legs (ckpt, gates, replay)")
    ap.add_argument("--decode-only", action="store_true", help="only the decode measurement (for profiling)")
    ap.add_argument("--spec-only", action="store_true", help="only the replay-window measurement (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_under_torchrun(args.gpus))

    from gated_delta_rule_117_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.seq_len > 0:
        w = w.with_(T=args.seq_len, name="%s_T%d" % (w.name, args.seq_len))

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        raise SystemExit("bench.py: --gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    import torch
    import torch.distributed as dist
    from gated_delta_rule_117_b200 import kda
    from gated_delta_rule_117_b200 import build as kbuild

    assert not w.decode, "main line is a prefill workload"
    w = rank_workload(w, rank)
    # host inputs and the oracle processes come before the first CUDA call
    x = host_inputs(synth, w, world)
    leg = None
    if rank == 0 and world == 1 and not args.no_cpu:
        chains = sample_chains(w) if w.T < (1 << 18) else [(0, 5), (w.B - 1, w.H - 1)]
        leg = OracleLeg(w, x, chains, workers=len(chains))

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    kbuild.build()
    kda.load_library()
    dev = torch.device("cuda", local)
    pk, pk_kind = peaks()

    if args.decode_only:
        print(json.dumps(measure_decode(args, synth, kda, torch, dev, pk, pk_kind)))
        return
    if args.spec_only:
        print(json.dumps(measure_spec(args, synth, kda, torch, dev, pk)))
        return
    d = {k: v.to(dev) for k, v in x.items()}
    h0 = d["h0"] if w.h0_std > 0 else None
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    plan = kda.kda_chunk_fwd_plan(B, H, T, dk, dv, dt, args.chunk_size)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    with ClockSampler(gpu_uuid(torch, dev)) as clk:
        times_ms, o, hT = time_prefill(args, w, d, plan, kda, torch, flush, dev, clk=clk,
                                       dist=dist if world > 1 else None)
    total_ms = max_over_ranks(sum(times_ms), dist if world > 1 else None, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(B * T, world, ms_per_step)
    kern_ms = statistics.mean(times_ms)
    fig = prefill_figures(w, plan, kern_ms, pk, pk_kind, synth)
    # the timed run's own output on the chains the oracle recomputes
    if leg is not None:
        o_s = torch.stack([o[b, h] for b, h in leg.chains]).cpu()
        h_s = torch.stack([hT[b, h] for b, h in leg.chains]).cpu()

    e2e = measure_e2e(args, w, x, d, kda, torch, dev, plan, dist=dist if world > 1 else None)

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded; report's KDA input distributions)",
        "config": {"workload": w.name, "B": B, "H": H, "T": T, "dk": dk, "dv": dv,
                   "chunk_size": plan["chunk_size"], "path": plan["path"], "segments": plan["segments"],
                   "h0": "N(0,0.02)" if w.h0_std > 0 else "zeros",
                   "l2": "flushed (256 MB write) between steps; inputs %.1f GB" % (synth.prefill_bytes(w) / 1e9),
                   "parallelism": "replicas" if world > 1 else "single"},
        "tflops": fig["tflops"],
        "roofline": fig["roofline"],
        "e2e": e2e,
        "gpu_launches": plan["launches"] * args.steps,
    }
    if world == 1 and not args.no_legs:
        ws = torch.empty(max(plan["workspace"], 16), dtype=torch.uint8, device=dev)
        if T >= CKPT_INTERVAL:
            result["ckpt"] = optional_leg(lambda: measure_ckpt(args, w, d, h0, o, hT, ws, flush, kda, torch,
                                                               kern_ms))
        result["out_gate"] = optional_leg(lambda: measure_out_gate(args, w, o, flush, kda, torch, pk))
        sep = result["out_gate"].get("ms") if isinstance(result.get("out_gate"), dict) else None
        result["out_gate_fused"] = optional_leg(lambda: measure_outgate_fused(args, w, d, h0, hT, ws, flush, kda, torch,
                                                                              kern_ms, sep))
        if B * H * T <= (1 << 17):  # z is regenerated on the host: small workloads only
            result["gate"] = optional_leg(lambda: measure_gate(args, w, d, h0, o, hT, ws, flush, synth, kda, torch,
                                                               kern_ms))
        del ws
    del d, o, hT
    if world == 1 and not args.no_subconfigs:
        result["configs"] = [optional_leg(lambda n=n: measure_subconfig(args, n, synth, kda, torch, dev, flush, pk,
                                                                        pk_kind, world))
                             for n in SUBCONFIGS if n != w.name]
    if not args.no_decode and world == 1:
        result["decode"] = measure_decode(args, synth, kda, torch, dev, pk, pk_kind)
        if not args.no_legs:
            result["spec"] = optional_leg(lambda: measure_spec(args, synth, kda, torch, dev, pk))
    result["clocks"] = clk.summary()
    if leg is not None:
        parity, cpu = leg.finish(o_s, h_s, max(plan["segment_tokens"], 1))
        result["parity"] = parity
        result["cpu_baseline"] = cpu
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def optional_leg(fn):
    """A secondary measurement (checkpoints, fused gate, output edge, replay):
    a failure there is recorded in its own object and never costs the main line."""
    try:
        return fn()
    except Exception as ex:  # noqa: BLE001
        return {"error": "%s: %s" % (type(ex).__name__, ex)}


CKPT_INTERVAL = 512  # hash-block size of the prefix cache (tokens)


def measure_ckpt(args, w, d, h0, o, hT, ws, flush, kda, torch, plain_ms):
    """The same step through kda_chunk_fwd_ckpt, persisting the state every
    CKPT_INTERVAL tokens for a prefix cache: time per step and its overhead."""
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    dev, sp = o.device, torch.cuda.current_stream().cuda_stream
    n = T // CKPT_INTERVAL
    ck = torch.empty(B, H, n, dk, dv, dtype=torch.float32, device=dev)
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    ptr = lambda t: None if t is None else t.data_ptr()

    def step():
        st = kda.kda_chunk_fwd_ckpt(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["g"]), ptr(d["beta"]), ptr(h0),
                                    ptr(o), ptr(hT), ck.data_ptr(), CKPT_INTERVAL, B, H, T, dk, dv, dt,
                                    args.chunk_size, 0.0, ws.data_ptr(), ws.numel(), sp)
        if st != 0:
            raise kda.KdaError(st, "kda_chunk_fwd_ckpt")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        flush.zero_()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    check_device_status(kda, "kda_chunk_fwd_ckpt")
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    launches = kda.kda_chunk_fwd_plan(B, H, T, dk, dv, dt, args.chunk_size)["launches"]
    return {"interval": CKPT_INTERVAL, "checkpoints_per_chain": n, "ms_per_step": ms,
            "overhead": ms / plain_ms - 1.0, "extra_bytes_per_step": B * H * n * dk * dv * 4,
            "gpu_launches": len(ev) * launches}


def measure_gate(args, w, d, h0, o, hT, ws, flush, synth, kda, torch, plain_ms):
    """The same step through kda_chunk_fwd_gated (Eq. 5 gate fused into the
    loads: z and A in, g never in memory): time per step against the plain call,
    and the bytes a separate gate pass would move (read z, write g)."""
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    gi = synth.gate_inputs(w)
    z, A = gi["z"].to(o.device), gi["A_log"].to(o.device)
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    sp = torch.cuda.current_stream().cuda_stream
    ptr = lambda t: None if t is None else t.data_ptr()

    def step():
        st = kda.kda_chunk_fwd_gated(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), z.data_ptr(), A.data_ptr(), -5.0,
                                     ptr(d["beta"]), ptr(h0), ptr(o), ptr(hT), B, H, T, dk, dv, dt, args.chunk_size,
                                     0.0, ws.data_ptr(), ws.numel(), sp)
        if st != 0:
            raise kda.KdaError(st, "kda_chunk_fwd_gated")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        flush.zero_()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    check_device_status(kda, "kda_chunk_fwd_gated")
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    launches = kda.kda_chunk_fwd_plan(B, H, T, dk, dv, dt, args.chunk_size)["launches"]
    e = 2 if w.dtype == "bf16" else 4
    return {"ms_per_step": ms, "overhead": ms / plain_ms - 1.0,
            "separate_gate_bytes_per_step": 2 * B * H * T * dk * e, "gpu_launches": len(ev) * launches}


def measure_outgate_fused(args, w, d, h0, hT, ws, flush, kda, torch, plain_ms, sep_ms):
    """The same step through kda_chunk_fwd_outgate (Eq. 6 output edge fused into
    the output epilogue: y written instead of o, o never in memory) against the
    plain step followed by the separate edge pass."""
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    dev, sp = hT.device, torch.cuda.current_stream().cuda_stream
    gen = torch.Generator(device=dev).manual_seed(7)
    gate = torch.randn(B, H, T, dv, generator=gen, device=dev).to(w.torch_dtype)
    wt = torch.ones(H, dv, dtype=torch.float32, device=dev)
    y = torch.empty(B, H, T, dv, dtype=w.torch_dtype, device=dev)
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    ptr = lambda t: None if t is None else t.data_ptr()

    def step():
        st = kda.kda_chunk_fwd_outgate(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["g"]), ptr(d["beta"]), ptr(h0),
                                       gate.data_ptr(), wt.data_ptr(), 1e-6, y.data_ptr(), ptr(hT), B, H, T, dk, dv, dt,
                                       args.chunk_size, 0.0, ws.data_ptr(), ws.numel(), sp)
        if st != 0:
            raise kda.KdaError(st, "kda_chunk_fwd_outgate")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        flush.zero_()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    check_device_status(kda, "kda_chunk_fwd_outgate")
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    e = 2 if w.dtype == "bf16" else 4
    launches = kda.kda_chunk_fwd_plan(B, H, T, dk, dv, dt, args.chunk_size)["launches"]
    out = {"ms_per_step": ms, "vs_plain_step": ms / plain_ms - 1.0,
           "round_trip_bytes_removed": 2 * B * H * T * dv * e, "gpu_launches": len(ev) * launches}
    if sep_ms is not None:
        out["unfused_ms_per_step"] = plain_ms + sep_ms
        out["speedup_vs_unfused"] = (plain_ms + sep_ms) / ms
    del gate, wt, y
    return out


def measure_out_gate(args, w, o, flush, kda, torch, pk):
    """Eq. 6 output edge (per-head RMSNorm and sigmoid gate) on the prefill's
    output: an HBM-bound pass, reported against the copy bandwidth."""
    B, H, T, dv = o.shape
    gen = torch.Generator(device=o.device).manual_seed(7)
    gate = torch.randn(o.shape, generator=gen, device=o.device).to(o.dtype)
    wt = torch.ones(H, dv, dtype=torch.float32, device=o.device)
    y = torch.empty_like(o)
    dt = kda.KDA_DTYPE_BF16 if o.dtype == torch.bfloat16 else kda.KDA_DTYPE_F32
    sp = torch.cuda.current_stream().cuda_stream

    def step():
        st = kda.kda_output_gate(o.data_ptr(), gate.data_ptr(), wt.data_ptr(), 1e-6, y.data_ptr(), B, H, T, dv, dt, sp)
        if st != 0:
            raise kda.KdaError(st, "kda_output_gate")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        flush.zero_()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    nbytes = 3 * o.numel() * o.element_size() + wt.numel() * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"ms": ms, "bytes": nbytes, "GB/s": gbs, "frac_of_hbm_peak": gbs / pk["hbm_gbs"], "gpu_launches": len(ev)}


def pin_host(torch, t):
    """Page-lock a host tensor in place (cudaHostRegister) so copies from it
    are true async DMA; returns (tensor, registered).  Falls back to a pinned
    copy when registration is refused."""
    nbytes = t.numel() * t.element_size()
    if nbytes and t.is_contiguous():
        try:
            if int(torch.cuda.cudart().cudaHostRegister(t.data_ptr(), nbytes, 0)) == 0:
                return t, True
        except Exception:  # noqa: BLE001
            pass
    return t.pin_memory(), False


def measure_e2e(args, w, x, d, kda, torch, dev, plan, dist=None):
    """Same metric through the C ABI from pinned host buffers, for a stream of
    steps: every step copies its inputs host->device, runs kda_chunk_fwd and
    copies o and h_T back to pinned host memory, all inside the timed region.
    Consecutive steps are pipelined as a serving loop would run them: two sets
    of device buffers, uploads on one copy stream and downloads on another, so
    step i+1's upload overlaps step i's compute and download (the host link is
    full duplex); a step's compute waits for its own upload, and a buffer is
    refilled only after the step two back has finished with it."""
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    use_h0 = w.h0_std > 0
    names = ["q", "k", "v", "g", "beta"] + (["h0"] if use_h0 else [])
    pinned = {n: pin_host(torch, x[n]) for n in names}
    hx = {n: p[0] for n, p in pinned.items()}
    ho = torch.empty(B, H, T, dv, dtype=w.torch_dtype).pin_memory()
    hh = torch.empty(B, H, dk, dv, dtype=torch.float32).pin_memory()
    ins = [d, {n: torch.empty_like(d[n]) for n in names}]
    outs = [(torch.empty(B, H, T, dv, dtype=w.torch_dtype, device=dev),
             torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)) for _ in range(2)]
    ws = torch.empty(max(plan["workspace"], 16), dtype=torch.uint8, device=dev)
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    h2d = sum(hx[n].numel() * hx[n].element_size() for n in names)
    d2h = ho.numel() * ho.element_size() + hh.numel() * hh.element_size()
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]
    count = [0]

    def step():
        i = count[0]
        count[0] += 1
        b = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(computed[b])  # step i - 2 has read these inputs
            for n in names:
                ins[b][n].copy_(hx[n], non_blocking=True)
            uploaded[b].record(up)
        comp.wait_event(uploaded[b])
        if i >= 2:
            comp.wait_event(downloaded[b])  # step i - 2's outputs have left
        di, (do, dh) = ins[b], outs[b]
        st = kda.kda_chunk_fwd(di["q"].data_ptr(), di["k"].data_ptr(), di["v"].data_ptr(), di["g"].data_ptr(),
                               di["beta"].data_ptr(), di["h0"].data_ptr() if use_h0 else None, do.data_ptr(),
                               dh.data_ptr(), B, H, T, dk, dv, dt, args.chunk_size, 0.0, ws.data_ptr(), ws.numel(),
                               comp.cuda_stream)
        if st != 0:
            raise kda.KdaError(st)
        computed[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(computed[b])
            ho.copy_(do, non_blocking=True)
            hh.copy_(dh, non_blocking=True)
            downloaded[b].record(down)

    try:
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(comp)
        up.wait_event(a)  # the first timed upload starts inside the region
        for _ in range(args.steps):
            step()
        for ev in downloaded:  # every step's download (hence its compute and upload) is done
            comp.wait_event(ev)
        e.record(comp)
        torch.cuda.synchronize()
        check_device_status(kda, "kda_chunk_fwd (e2e)")
        ms = max_over_ranks(a.elapsed_time(e) / args.steps, dist, dev)
    finally:
        for n, (t, reg) in pinned.items():
            if reg:
                torch.cuda.cudart().cudaHostUnregister(t.data_ptr())
    world = dist.get_world_size() if dist is not None else 1
    return {"value": job_throughput(B * T, world, ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "warmup": 3,
            "host_buffers": "pinned (page-locked in place where possible)",
            "pipelining": "steps overlap: upload of step i+1 with compute and download of step i (two buffer sets)"}


SPEC_WINDOW, SPEC_REPLAY = 4, 2  # window of 4 tokens: 2 accepted drafts replayed, bonus + 1 draft verified


def measure_spec(args, synth, kda, torch, dev, pk):
    """Speculative-decode replay and verify on the decode workload's state
    (B256 H32, 512 MiB fp32): one kda_spec_replay_verify per window of
    SPEC_WINDOW tokens, SPEC_REPLAY of them replayed and committed.  The state
    is read once and written once per window."""
    w = synth.WORKLOADS["decode_b256_h32"]
    x = synth.decode_inputs(w, steps=SPEC_WINDOW)
    S = x["S0"].to(dev)
    # window inputs [B, H, W, d] from the first SPEC_WINDOW pre-generated steps
    win = {n: x[n][:SPEC_WINDOW].movedim(0, 2).contiguous().to(dev) for n in ("q", "k", "v", "g", "beta")}
    o = torch.empty(w.B, w.H, SPEC_WINDOW, w.dv, dtype=w.torch_dtype, device=dev)
    nr = torch.full((w.B,), SPEC_REPLAY, dtype=torch.int32, device=dev)
    sp = torch.cuda.current_stream().cuda_stream

    def one():
        st = kda.kda_spec_replay_verify(win["q"].data_ptr(), win["k"].data_ptr(), win["v"].data_ptr(),
                                        win["g"].data_ptr(), win["beta"].data_ptr(), S.data_ptr(), o.data_ptr(),
                                        nr.data_ptr(), w.B, w.H, SPEC_WINDOW, w.dk, w.dv, kda.KDA_DTYPE_BF16, 0.0, sp)
        if st != 0:
            raise kda.KdaError(st, "kda_spec_replay_verify")

    for _ in range(max(args.warmup, 3)):
        one()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(16)]
    for a, b in ev:
        a.record()
        one()
        b.record()
    torch.cuda.synchronize()
    med = statistics.median(a.elapsed_time(b) for a, b in ev)
    e = 2
    nbytes = (2 * S.numel() * 4 + w.B * w.H * SPEC_WINDOW * (3 * w.dk + w.dv + 1) * e
              + w.B * w.H * (SPEC_WINDOW - SPEC_REPLAY) * w.dv * e)
    gbs = nbytes / (med / 1e3) / 1e9
    return {"window": SPEC_WINDOW, "replayed": SPEC_REPLAY, "ms_per_window_median": med, "bytes_per_window": nbytes,
            "GB/s": gbs, "frac_of_hbm_peak": gbs / pk["hbm_gbs"], "gpu_launches": len(ev)}


def measure_decode(args, synth, kda, torch, dev, pk, pk_kind):
    """kda_recurrent_step on the decode workload: 64 separate step launches
    over pre-generated tokens, state (512 MiB fp32, > L2) updated in place."""
    w = synth.WORKLOADS["decode_b256_h32"]
    x = synth.decode_inputs(w)
    d = {k: v.to(dev) for k, v in x.items()}
    S = d["S0"].clone()
    o = torch.empty(w.T, w.B, w.H, w.dv, dtype=w.torch_dtype, device=dev)
    stream = torch.cuda.current_stream()
    dt = kda.KDA_DTYPE_BF16
    ptr = lambda t: t.data_ptr()

    def one(t):
        st = kda.kda_recurrent_step(ptr(d["q"][t]), ptr(d["k"][t]), ptr(d["v"][t]), ptr(d["g"][t]),
                                    ptr(d["beta"][t]), ptr(S), ptr(o[t]), w.B, w.H, w.dk, w.dv, dt, 0.0,
                                    stream.cuda_stream)
        if st != 0:
            raise kda.KdaError(st)

    for t in range(max(args.warmup, 3)):
        one(t)
    S.copy_(d["S0"])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(w.T)]
    for t in range(w.T):
        ev[t][0].record(stream)
        one(t)
        ev[t][1].record(stream)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    med = statistics.median(ms)
    byts = synth.decode_bytes_per_step(w)
    gbs = byts / (med / 1e3) / 1e9
    return {"workload": w.name, "steps": w.T, "ms_per_step_median": med, "ms_per_step_mean": statistics.mean(ms),
            "GB/s": gbs, "bytes_per_step": byts, "gpu_launches": w.T,
            "roofline": {"kernel": "recurrent_step_kernel", "bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / pk["hbm_gbs"], "peak_kind": pk_kind,
                         "traffic": (traffic_record("recurrent_step_kernel:" + w.name,
                                                    ["gated_delta_rule_117_b200/csrc/kda_decode.cu"]) or {}
                                     ).get("dram_bytes_per_launch")}}


def run_reference(args, w, rank, world):
    """The reference arm is the fp64 CPU oracle timed on the host cores."""
    if rank != 0:
        return
    import oracle
    from gated_delta_rule_117_b200 import synth
    threads = min(os.cpu_count() or 1, w.B * w.H)
    # bounded sample of the workload: the first Ts tokens of every chain
    Ts = min(w.T, 512)
    x = synth.prefill_inputs(w, T=Ts)
    for _ in range(args.warmup):
        cpu_oracle_prefill(w, x, threads)
    secs = [cpu_oracle_prefill(w, x, threads) for _ in range(args.steps)]
    tot = sum(secs)
    value = w.B * Ts * args.steps / tot
    res = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded; report's KDA input distributions)",
           "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                            "sample": "first %d tokens of each of the %d chains per step" % (Ts, w.B * w.H)},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res))


if __name__ == "__main__":
    main()
