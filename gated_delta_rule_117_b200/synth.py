"""Seeded synthetic KDA inputs (shared by the CUDA tests/bench and the CPU oracle).

This module holds no KDA arithmetic: it only draws random tensors with the
value distributions of the Kimi K3 report's KDA layer and rounds them to the
stored dtype.  Both the GPU path and the oracle read the bits it returns.

Distributions (Kimi K3 technical report, section 2.1.1):
  * q, k ~ N(0, 1), then L2-normalised over the key dimension per token and
    head (the report normalises q and k after the short convolution, Eq. 2);
  * v ~ N(0, 1);
  * beta = Sigmoid(N(0, 1)) per token and head (Eq. 2 gives beta in (0, 1));
  * per-channel log-decay g = g_min * Sigmoid(e^A * z), g_min = -5 (Eq. 5),
    with A ~ N(0, 0.5) per (head, key channel) and z ~ N(0, 1) per (token,
    channel).  In the batched workload 10 % of the heads draw A ~ N(2, 0.5),
    which pushes g toward the -5 bound (near-zero retention);
  * h0 ~ N(0, 0.02) in fp32 where a workload asks for it, else zeros.

Every (tensor, batch, head) owns an independent PCG64 stream seeded from
``SeedSequence([seed, tensor_id, b, h])`` so one head can be regenerated on its
own (the oracle samples single heads of the large workloads).  Values are
computed in fp64 and rounded round-to-nearest-even to the workload dtype
(via fp32 for bf16, i.e. torch's own conversion).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np
import torch

G_MIN = -5.0  # lower bound of the per-token log-decay (Kimi K3 report, Eq. 5)

# stream ids
_Q, _K, _V, _Z, _BETA, _A, _H0, _FASTHEADS = range(8)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str          # "f32" or "bf16": dtype of q, k, v, g, beta (and o)
    B: int
    H: int
    T: int              # tokens per sequence (decode: number of steps)
    dk: int
    dv: int
    chunk: int          # chunk size the workload names (0 = library default)
    h0_std: float       # 0 -> h0 = zeros
    fast_decay_frac: float
    seed: int
    decode: bool = False

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads: tiny fp32 check, prefill, batched prefill, 1M-token
# prefill and the recurrent decode step (64 steps, state updated in place).
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", "f32", 1, 2, 64, 16, 16, 16, 0.0, 0.0, 1000),
    "prefill_h16_t4k": Workload("prefill_h16_t4k", "bf16", 1, 16, 4096, 128, 128, 64, 0.02, 0.0, 1001),
    "batched_b8_h32_t8k": Workload("batched_b8_h32_t8k", "bf16", 8, 32, 8192, 128, 128, 64, 0.0, 0.1, 1002),
    "long_h16_t1m": Workload("long_h16_t1m", "bf16", 1, 16, 1 << 20, 128, 128, 64, 0.0, 0.0, 1003),
    "decode_b256_h32": Workload("decode_b256_h32", "bf16", 256, 32, 64, 128, 128, 0, 0.02, 0.0, 1004, decode=True),
}


def _rng(w: Workload, tensor: int, b: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, tensor, b, h])))


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def fast_decay_heads(w: Workload) -> np.ndarray:
    """Head indices whose A is drawn from N(2, 0.5) (shared across the batch)."""
    n = int(round(w.fast_decay_frac * w.H))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    perm = _rng(w, _FASTHEADS, 0, 0).permutation(w.H)
    return np.sort(perm[:n])


def decay_log_scale(w: Workload, h: int) -> np.ndarray:
    """A for head h: one value per key channel (fp64)."""
    mean = 2.0 if h in set(fast_decay_heads(w).tolist()) else 0.0
    return mean + 0.5 * _rng(w, _A, 0, h).standard_normal(w.dk)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the stored dtype (RNE) and return them as fp64."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    if dtype == "f32":
        return t.to(torch.float32).to(torch.float64).numpy()
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def head_inputs(w: Workload, b: int, h: int, T: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Stored (already rounded) inputs of one (b, h) chain, as fp64 arrays.

    Returns q, k, g: [T, dk]; v: [T, dv]; beta: [T]; h0: [dk, dv] (fp32 values).
    For a decode workload T counts steps.
    """
    T = w.T if T is None else T
    q = _rng(w, _Q, b, h).standard_normal((T, w.dk))
    k = _rng(w, _K, b, h).standard_normal((T, w.dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = _rng(w, _V, b, h).standard_normal((T, w.dv))
    z = _rng(w, _Z, b, h).standard_normal((T, w.dk))
    A = decay_log_scale(w, h)
    g = G_MIN * _sigmoid(np.exp(A)[None, :] * z)
    beta = _sigmoid(_rng(w, _BETA, b, h).standard_normal(T))
    if w.h0_std > 0:
        h0 = round_to(w.h0_std * _rng(w, _H0, b, h).standard_normal((w.dk, w.dv)), "f32")
    else:
        h0 = np.zeros((w.dk, w.dv))
    return dict(q=round_to(q, w.dtype), k=round_to(k, w.dtype), v=round_to(v, w.dtype),
                g=round_to(g, w.dtype), beta=round_to(beta, w.dtype), h0=h0)


def gate_inputs(w: Workload, T: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """The decay logits z [B, H, T, dk] (rounded to the workload dtype) and the
    log-scales A [H, dk] (fp32) behind every workload's g: the raw draws, before
    any gate arithmetic, for calls that take z and A instead of g."""
    T = w.T if T is None else T
    z = np.stack([np.stack([round_to(_rng(w, _Z, b, h).standard_normal((T, w.dk)), w.dtype) for h in range(w.H)])
                  for b in range(w.B)])
    A = np.stack([round_to(decay_log_scale(w, h), "f32") for h in range(w.H)])
    return dict(z=_to_torch(z, w.torch_dtype), A_log=torch.from_numpy(A).float())


def head_input_blocks(w: Workload, b: int, h: int, T: Optional[int] = None, block: int = 65536):
    """The stored inputs of one (b, h) chain in token blocks (same values as
    head_inputs: every stream is drawn sequentially).  Yields (t0, dict) with
    q, k, g [n, dk], v [n, dv], beta [n]; h0 is not included."""
    T = w.T if T is None else T
    rq, rk, rv, rz, rb = (_rng(w, i, b, h) for i in (_Q, _K, _V, _Z, _BETA))
    eA = np.exp(decay_log_scale(w, h))[None, :]
    for t0 in range(0, T, block):
        n = min(block, T - t0)
        q = rq.standard_normal((n, w.dk))
        k = rk.standard_normal((n, w.dk))
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        v = rv.standard_normal((n, w.dv))
        g = G_MIN * _sigmoid(eA * rz.standard_normal((n, w.dk)))
        beta = _sigmoid(rb.standard_normal(n))
        yield t0, dict(q=round_to(q, w.dtype), k=round_to(k, w.dtype), v=round_to(v, w.dtype),
                       g=round_to(g, w.dtype), beta=round_to(beta, w.dtype))


def _to_torch(x: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(x).to(dtype)


def prefill_inputs(w: Workload, T: Optional[int] = None, heads=None) -> Dict[str, torch.Tensor]:
    """Whole-workload prefill inputs as CPU torch tensors in the stored dtype.

    q, k, g: [B, H, T, dk]; v: [B, H, T, dv]; beta: [B, H, T]; h0: [B, H, dk, dv]
    fp32 (zeros when the workload has no h0).
    """
    assert not w.decode
    T = w.T if T is None else T
    dt = w.torch_dtype
    out = dict(q=torch.empty(w.B, w.H, T, w.dk, dtype=dt), k=torch.empty(w.B, w.H, T, w.dk, dtype=dt),
               v=torch.empty(w.B, w.H, T, w.dv, dtype=dt), g=torch.empty(w.B, w.H, T, w.dk, dtype=dt),
               beta=torch.empty(w.B, w.H, T, dtype=dt), h0=torch.zeros(w.B, w.H, w.dk, w.dv, dtype=torch.float32))
    for b in range(w.B):
        for h in range(w.H):
            x = head_inputs(w, b, h, T)
            for name in ("q", "k", "v", "g", "beta"):
                out[name][b, h] = _to_torch(x[name], dt)
            out["h0"][b, h] = _to_torch(x["h0"], torch.float32)
    return out


def _fill_heads(args):
    w, T, heads, tensors = args
    for b, h in heads:
        for t0, x in head_input_blocks(w, b, h, T):
            n = x["beta"].shape[0]
            for name in ("q", "k", "v", "g", "beta"):
                tensors[name][b, h, t0:t0 + n] = _to_torch(x[name], w.torch_dtype)
        if w.h0_std > 0:
            h0 = round_to(w.h0_std * _rng(w, _H0, b, h).standard_normal((w.dk, w.dv)), "f32")
            tensors["h0"][b, h] = _to_torch(h0, torch.float32)
    return len(heads)


def prefill_inputs_parallel(w: Workload, workers: int, T: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """prefill_inputs computed by a pool of `workers` spawned processes writing
    into shared-memory tensors in token blocks (same values, bit for bit)."""
    assert not w.decode
    T = w.T if T is None else T
    dt = w.torch_dtype
    out = dict(q=torch.empty(w.B, w.H, T, w.dk, dtype=dt), k=torch.empty(w.B, w.H, T, w.dk, dtype=dt),
               v=torch.empty(w.B, w.H, T, w.dv, dtype=dt), g=torch.empty(w.B, w.H, T, w.dk, dtype=dt),
               beta=torch.empty(w.B, w.H, T, dtype=dt), h0=torch.zeros(w.B, w.H, w.dk, w.dv, dtype=torch.float32))
    for t in out.values():
        t.share_memory_()
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    workers = max(1, min(workers, len(heads)))
    parts = [heads[i::workers] for i in range(workers)]
    ctx = torch.multiprocessing.get_context("spawn")
    with ctx.Pool(workers) as pool:
        pool.map(_fill_heads, [(w, T, part, out) for part in parts])
    return out


def decode_inputs(w: Workload, steps: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Decode workload: S0 [B, H, dk, dv] fp32 and per-step q, k, g: [steps, B, H, dk],
    v: [steps, B, H, dv], beta: [steps, B, H] in the stored dtype."""
    assert w.decode
    n = w.T if steps is None else steps
    dt = w.torch_dtype
    out = dict(q=torch.empty(n, w.B, w.H, w.dk, dtype=dt), k=torch.empty(n, w.B, w.H, w.dk, dtype=dt),
               v=torch.empty(n, w.B, w.H, w.dv, dtype=dt), g=torch.empty(n, w.B, w.H, w.dk, dtype=dt),
               beta=torch.empty(n, w.B, w.H, dtype=dt), S0=torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32))
    for b in range(w.B):
        for h in range(w.H):
            x = head_inputs(w, b, h, n)
            for name in ("q", "k", "v", "g", "beta"):
                out[name][:, b, h] = _to_torch(x[name], dt)
            out["S0"][b, h] = _to_torch(x["h0"], torch.float32)
    return out


def flops_per_token_head(dk: int, dv: int, C: int) -> float:
    """Algorithmic prefill FLOPs per token-head of the chunked form (triangles as
    triangles; exp and elementwise work not counted)."""
    return 2.0 * (3 * dk * dv + (C / 2.0) * (3 * dk + 2 * dv) + C * C / 6.0)


def prefill_bytes(w: Workload, T: Optional[int] = None) -> float:
    """Algorithmic HBM bytes of one prefill: each input read once, o written once,
    h0 read (when present) and h_T written once."""
    T = w.T if T is None else T
    e = 4 if w.dtype == "f32" else 2
    per_tok = e * (2 * w.dk + w.dk + w.dv + 1 + w.dv)  # q, k, g, v, beta in; o out
    state = 4 * w.dk * w.dv * (2 if w.h0_std > 0 else 1)
    return w.B * w.H * (T * per_tok + state)


def decode_bytes_per_step(w: Workload) -> float:
    """State read + write plus the step's q, k, v, g, beta in and o out."""
    e = 4 if w.dtype == "f32" else 2
    return w.B * w.H * (2 * 4 * w.dk * w.dv + e * (3 * w.dk + 2 * w.dv + 1))
