#!/usr/bin/env python
"""Throughput of libkda's KDA forward on B200.

Default line: chunked prefill (kda_chunk_fwd) on the prefill workload
(B=1, H=16, T=4096, dk=dv=128, bf16 inputs, fp32 state, h0 ~ N(0, 0.02)),
reported as tokens/s with algorithmic TFLOP/s and the HBM roofline fraction of
the prefill kernel.  The same line carries the decode step (kda_recurrent_step,
B=256, H=32, 64 steps, state updated in place) as GB/s against the HBM peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl libkda|reference]

Under torchrun each rank runs an independent replica of the workload (the
(batch, head) chains are independent: no collective on the data path), time is
the max over ranks, and value is the whole-job throughput.
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill_h16_t4k")
    ap.add_argument("--impl", default="libkda", choices=["libkda", "reference"])
    ap.add_argument("--chunk-size", type=int, default=0)
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--decode-only", action="store_true", help="only the decode measurement (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from gated_delta_rule_117_b200 import synth
    w = synth.WORKLOADS[args.workload]

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    import torch
    import torch.distributed as dist
    from gated_delta_rule_117_b200 import kda
    from gated_delta_rule_117_b200 import build as kbuild

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    kbuild.build()
    kda.load_library()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    pk, pk_kind = peaks()

    if args.decode_only:
        print(json.dumps(measure_decode(args, synth, kda, torch, dev, pk, pk_kind)))
        return
    assert not w.decode, "main line is a prefill workload"
    w = rank_workload(w, rank)
    x = synth.prefill_inputs(w)
    d = {k: v.to(dev) for k, v in x.items()}
    h0 = d["h0"] if w.h0_std > 0 else None
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    plan = kda.kda_chunk_fwd_plan(B, H, T, dk, dv, dt, args.chunk_size)
    o = torch.empty(B, H, T, dv, dtype=w.torch_dtype, device=dev)
    hT = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    ws = torch.empty(max(plan["workspace"], 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    ptr = lambda t: None if t is None else t.data_ptr()
    sp = stream.cuda_stream

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
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_uuid(torch, dev)) as clk:
        clk.soak(lambda: (flush.zero_(), step()), torch)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()  # L2 flush between timed iterations (outside the events)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
    times_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(times_ms), dist if world > 1 else None, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(B * T, world, ms_per_step)
    kern_ms = statistics.mean(times_ms)  # one launch per step: the step is the kernel
    bytes_per_launch = synth.prefill_bytes(w)
    achieved = bytes_per_launch / (kern_ms / 1e3) / 1e9
    flops = synth.flops_per_token_head(dk, dv, 64) * B * H * T
    tflops = flops / (kern_ms / 1e3) / 1e12
    kernel_name = "chunk16_kernel" if plan["path"] == kda.KDA_PATH_SIMT16 else "chunk_tc_kernel"
    # With in-device context parallelism one step is three launches (segment
    # transitions, the prefix scan, the final pass); the roofline then uses the
    # whole step's time, which is the conservative reading.
    roofline_scope = "kernel" if plan["launches"] == 1 else "step (%d launches)" % plan["launches"]
    src = (["gated_delta_rule_117_b200/csrc/kda_chunk_simt.cu"] if plan["path"] == kda.KDA_PATH_SIMT16
           else ["gated_delta_rule_117_b200/csrc/kda_chunk_tc.cu"])
    trec = traffic_record("%s:%s" % (kernel_name, w.name), src)
    traffic = None
    if trec:
        # a segmented step records the DRAM bytes of all its launches, like `achieved`
        traffic = trec.get("dram_bytes_per_step", trec.get("dram_bytes_per_launch"))

    e2e = measure_e2e(args, w, x, kda, torch, dev, plan)

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded; report's KDA input distributions)",
        "config": {"workload": w.name, "B": B, "H": H, "T": T, "dk": dk, "dv": dv,
                   "chunk_size": plan["chunk_size"], "path": plan["path"], "segments": plan["segments"],
                   "h0": "N(0,0.02)" if w.h0_std > 0 else "zeros", "l2": "flushed (256 MB write) between steps",
                   "parallelism": "replicas" if world > 1 else "single"},
        "tflops": {"value": tflops, "flop_per_token_head": synth.flops_per_token_head(dk, dv, 64),
                   "frac_of_bf16_peak": tflops / pk["bf16_tflops"], "peak_kind": pk_kind},
        "roofline": {"kernel": kernel_name, "scope": roofline_scope, "bound": "hbm", "achieved": achieved,
                     "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                     "algorithmic_bytes_per_launch": bytes_per_launch, "peak_kind": pk_kind,
                     "kernel_ms": kern_ms},
        "e2e": e2e,
        "gpu_launches": plan["launches"] * args.steps,
    }
    if world == 1 and T >= CKPT_INTERVAL:
        result["ckpt"] = optional_leg(lambda: measure_ckpt(args, w, d, h0, o, hT, ws, flush, kda, torch, ms_per_step))
    if world == 1:
        result["out_gate"] = optional_leg(lambda: measure_out_gate(args, w, o, flush, kda, torch, pk))
    if world == 1 and B * H * T <= (1 << 17):  # z is regenerated on the host: small workloads only
        result["gate"] = optional_leg(lambda: measure_gate(args, w, d, h0, o, hT, ws, flush, synth, kda, torch,
                                                           ms_per_step))
    if not args.no_decode and world == 1:
        result["decode"] = measure_decode(args, synth, kda, torch, dev, pk, pk_kind)
        result["spec"] = optional_leg(lambda: measure_spec(args, synth, kda, torch, dev, pk))
    clocks = clk.summary()
    result["clocks"] = clocks
    if rank == 0 and world == 1 and not args.no_cpu:
        threads = min(os.cpu_count() or 1, B * H)
        secs = cpu_oracle_prefill(w, x, threads)
        result["cpu_baseline"] = {"value": B * T / secs, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                  "sample": "whole workload (%d chains x %d tokens), fp64 C recurrence, 1 pass"
                                            % (B * H, T)}
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
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    launches = kda.kda_chunk_fwd_plan(B, H, T, dk, dv, dt, args.chunk_size)["launches"]
    e = 2 if w.dtype == "bf16" else 4
    return {"ms_per_step": ms, "overhead": ms / plain_ms - 1.0,
            "separate_gate_bytes_per_step": 2 * B * H * T * dk * e, "gpu_launches": len(ev) * launches}


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


def measure_e2e(args, w, x, kda, torch, dev, plan):
    """Same metric through the C ABI from pinned host buffers: each step copies
    the inputs host->device, runs kda_chunk_fwd and copies o and h_T back."""
    stream = torch.cuda.current_stream()
    hx = {k: v.pin_memory() for k, v in x.items()}
    dx = {k: torch.empty_like(v, device=dev) for k, v in x.items()}
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    use_h0 = w.h0_std > 0
    ho = torch.empty(B, H, T, dv, dtype=w.torch_dtype).pin_memory()
    hh = torch.empty(B, H, dk, dv, dtype=torch.float32).pin_memory()
    do = torch.empty(B, H, T, dv, dtype=w.torch_dtype, device=dev)
    dh = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    ws = torch.empty(max(plan["workspace"], 16), dtype=torch.uint8, device=dev)
    dt = kda.KDA_DTYPE_BF16 if w.dtype == "bf16" else kda.KDA_DTYPE_F32
    names = ["q", "k", "v", "g", "beta"] + (["h0"] if use_h0 else [])
    h2d = sum(hx[n].numel() * hx[n].element_size() for n in names)
    d2h = ho.numel() * ho.element_size() + hh.numel() * hh.element_size()

    def step():
        for n in names:
            dx[n].copy_(hx[n], non_blocking=True)
        st = kda.kda_chunk_fwd(dx["q"].data_ptr(), dx["k"].data_ptr(), dx["v"].data_ptr(), dx["g"].data_ptr(),
                               dx["beta"].data_ptr(), dx["h0"].data_ptr() if use_h0 else None, do.data_ptr(),
                               dh.data_ptr(), B, H, T, dk, dv, dt, args.chunk_size, 0.0, ws.data_ptr(), ws.numel(),
                               stream.cuda_stream)
        if st != 0:
            raise kda.KdaError(st)
        ho.copy_(do, non_blocking=True)
        hh.copy_(dh, non_blocking=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    return {"value": B * T / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms}


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
