"""Helpers shared by the GPU parity tests: relative L2 error and oracle runs
on the same seeded inputs the GPU sees."""
import numpy as np
import torch

import oracle
from gated_delta_rule_117_b200 import synth

# Tolerances on relative L2 error (fp64 norm over the whole tensor): 1e-5 for
# fp32 inputs, 3e-3 for bf16 inputs with fp32 state and accumulation.
TOL = {"f32": 1e-5, "bf16": 3e-3}


def rel_l2(x, ref):
    x = np.asarray(x.double().cpu().numpy() if isinstance(x, torch.Tensor) else x, dtype=np.float64)
    ref = np.asarray(ref.double().cpu().numpy() if isinstance(ref, torch.Tensor) else ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.isfinite(x).all()
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def f64(t):
    return t.double().numpy()


def oracle_prefill(x, heads=None, h0=True, scale=None):
    """Oracle o, h_T for the CPU tensors x (from synth.prefill_inputs) on the
    (b, h) pairs in ``heads`` (all when None)."""
    if heads is None:
        sel = f64  # keep [B, H, ...]
    else:
        idx_b = [b for b, _ in heads]
        idx_h = [h for _, h in heads]
        sel = lambda t: f64(t[idx_b, idx_h])  # [n, ...]
    o, hT = oracle.recurrent(sel(x["q"]), sel(x["k"]), sel(x["v"]), sel(x["g"]), sel(x["beta"]),
                             sel(x["h0"]) if h0 else None, scale=scale)
    return o, hT


def to_dev(x):
    return {k: v.cuda() for k, v in x.items()}
