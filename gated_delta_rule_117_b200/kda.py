"""ctypes binding of libkda (include/kda.h).

Argument marshalling only: the raw functions carry the C names and take
integer device pointers; the torch helpers below turn tensors into those
pointers and the current CUDA stream.  Every step of the computation runs in
libkda's kernels.  There is no fallback: if ``libkda.so`` is missing or the
device is unsupported, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(PKG, "libkda.so")

KDA_OK = 0
KDA_DTYPE_F32 = 0
KDA_DTYPE_BF16 = 1
KDA_PATH_AUTO, KDA_PATH_SIMT16, KDA_PATH_TC32 = 0, 1, 2
STATUS_NAMES = ["KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_SHAPE", "KDA_ERR_DTYPE", "KDA_ERR_ALIGNMENT",
                "KDA_ERR_ALIAS", "KDA_ERR_WORKSPACE", "KDA_ERR_CUDA", "KDA_ERR_TIMEOUT",
                "KDA_ERR_UNSUPPORTED", "KDA_ERR_DEVICE"]
EXPORTED = ["kda_chunk_fwd_plan", "kda_chunk_fwd_workspace_size", "kda_chunk_fwd", "kda_recurrent_step",
            "kda_status_string", "kda_get_device_status", "kda_version", "kda_chunk_fwd_noalloc",
            "kda_noalloc_scratch_bytes", "kda_chunk_fwd_ckpt", "kda_chunk_fwd_gated", "kda_output_gate",
            "kda_kcp_compose", "kda_spec_replay_verify", "kda_debug_set_wait_limit", "kda_debug_inject_stall",
            "kda_chunk_fwd_outgate", "kda_chunk_transition", "kda_spec_replay_verify_fused"]


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__("%s%s" % (kda_status_string(status), (" (" + what + ")") if what else ""))


class kda_plan_t(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("chunk_size", ctypes.c_int), ("segments", ctypes.c_int),
                ("launches", ctypes.c_int), ("workspace", ctypes.c_size_t), ("segment_tokens", ctypes.c_int)]


_lib = None
_lock = threading.Lock()


def load_library():
    """Load libkda.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(SO):
                raise RuntimeError("libkda.so is not built (run gated_delta_rule_117_b200.build.build())")
            lib = ctypes.CDLL(SO)
            vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            lib.kda_chunk_fwd_plan.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(kda_plan_t)]
            lib.kda_chunk_fwd_plan.restype = i
            lib.kda_chunk_fwd_workspace_size.argtypes = [i] * 7
            lib.kda_chunk_fwd_workspace_size.restype = sz
            lib.kda_chunk_fwd.argtypes = [vp] * 8 + [i] * 7 + [f, vp, sz, vp]
            lib.kda_chunk_fwd.restype = i
            lib.kda_chunk_fwd_ckpt.argtypes = [vp] * 9 + [i] * 8 + [f, vp, sz, vp]
            lib.kda_chunk_fwd_ckpt.restype = i
            lib.kda_chunk_fwd_gated.argtypes = [vp] * 5 + [f] + [vp] * 4 + [i] * 7 + [f, vp, sz, vp]
            lib.kda_chunk_fwd_gated.restype = i
            lib.kda_chunk_fwd_outgate.argtypes = [vp] * 8 + [f, vp, vp] + [i] * 7 + [f, vp, sz, vp]
            lib.kda_chunk_fwd_outgate.restype = i
            lib.kda_chunk_transition.argtypes = [vp] * 6 + [i] * 6 + [vp]
            lib.kda_chunk_transition.restype = i
            lib.kda_output_gate.argtypes = [vp, vp, vp, f, vp] + [i] * 5 + [vp]
            lib.kda_output_gate.restype = i
            lib.kda_kcp_compose.argtypes = [vp] * 4 + [i] * 5 + [vp]
            lib.kda_kcp_compose.restype = i
            lib.kda_spec_replay_verify_fused.argtypes = [vp] * 5 + [f] + [vp] * 4 + [f] + [vp] * 2 + [i] * 6 + [f, vp]
            lib.kda_spec_replay_verify_fused.restype = i
            lib.kda_spec_replay_verify.argtypes = [vp] * 8 + [i] * 6 + [f, vp]
            lib.kda_spec_replay_verify.restype = i
            lib.kda_recurrent_step.argtypes = [vp] * 7 + [i] * 5 + [f, vp]
            lib.kda_recurrent_step.restype = i
            lib.kda_status_string.argtypes = [i]
            lib.kda_status_string.restype = ctypes.c_char_p
            lib.kda_get_device_status.argtypes = [vp]
            lib.kda_get_device_status.restype = i
            lib.kda_debug_set_wait_limit.argtypes = [ctypes.c_ulonglong]
            lib.kda_debug_set_wait_limit.restype = i
            lib.kda_debug_inject_stall.argtypes = [i]
            lib.kda_debug_inject_stall.restype = i
            lib.kda_version.argtypes = []
            lib.kda_version.restype = i
            lib.kda_chunk_fwd_noalloc.argtypes = [vp] * 8 + [i] * 7 + [f, vp]
            lib.kda_chunk_fwd_noalloc.restype = i
            lib.kda_noalloc_scratch_bytes.argtypes = []
            lib.kda_noalloc_scratch_bytes.restype = sz
            _lib = lib
    return _lib


# ---- raw C-ABI calls (integer pointers) ------------------------------------

def kda_status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def kda_version() -> int:
    return load_library().kda_version()


def kda_chunk_fwd_plan(B, H, T, dk, dv, dtype, chunk_size=0):
    p = kda_plan_t()
    st = load_library().kda_chunk_fwd_plan(B, H, T, dk, dv, dtype, chunk_size, ctypes.byref(p))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_plan")
    return dict(path=p.path, chunk_size=p.chunk_size, segments=p.segments, launches=p.launches,
                workspace=p.workspace, segment_tokens=p.segment_tokens)


def kda_chunk_fwd_workspace_size(B, H, T, dk, dv, dtype, chunk_size=0) -> int:
    return load_library().kda_chunk_fwd_workspace_size(B, H, T, dk, dv, dtype, chunk_size)


def kda_chunk_fwd(q, k, v, g, beta, h0, o, h_T, B, H, T, dk, dv, dtype, chunk_size, scale,
                  workspace, workspace_bytes, stream) -> int:
    """Returns the raw kda_status_t."""
    return load_library().kda_chunk_fwd(q, k, v, g, beta, h0, o, h_T, B, H, T, dk, dv, dtype, chunk_size,
                                        scale, workspace, workspace_bytes, stream)


def kda_chunk_fwd_ckpt(q, k, v, g, beta, h0, o, h_T, ckpt, ckpt_interval, B, H, T, dk, dv, dtype, chunk_size,
                       scale, workspace, workspace_bytes, stream) -> int:
    """kda_chunk_fwd that also writes state checkpoints every ckpt_interval tokens.
    Returns the raw kda_status_t."""
    return load_library().kda_chunk_fwd_ckpt(q, k, v, g, beta, h0, o, h_T, ckpt, ckpt_interval, B, H, T, dk, dv,
                                             dtype, chunk_size, scale, workspace, workspace_bytes, stream)


def kda_chunk_fwd_gated(q, k, v, z, A_log, g_min, beta, h0, o, h_T, B, H, T, dk, dv, dtype, chunk_size, scale,
                        workspace, workspace_bytes, stream) -> int:
    """kda_chunk_fwd with the Eq. 5 decay gate fused into the loads (takes the
    logits z and log-scales A_log instead of g).  Returns the raw kda_status_t."""
    return load_library().kda_chunk_fwd_gated(q, k, v, z, A_log, g_min, beta, h0, o, h_T, B, H, T, dk, dv, dtype,
                                              chunk_size, scale, workspace, workspace_bytes, stream)


def kda_chunk_fwd_outgate(q, k, v, g, beta, h0, gate, rms_weight, eps, y, h_T, B, H, T, dk, dv, dtype, chunk_size,
                          scale, workspace, workspace_bytes, stream) -> int:
    """kda_chunk_fwd with the Eq. 6 output edge fused into the epilogue: writes
    y = Sigmoid(gate) * RMSNorm_w(o) instead of o.  Returns the raw kda_status_t."""
    return load_library().kda_chunk_fwd_outgate(q, k, v, g, beta, h0, gate, rms_weight, eps, y, h_T, B, H, T, dk, dv,
                                                dtype, chunk_size, scale, workspace, workspace_bytes, stream)


def kda_chunk_transition(k, v, g, beta, St, M, B, H, T, dk, dv, dtype, stream) -> int:
    """Segment transition (S~, M) of every chain (Eq. 17).  Returns the raw kda_status_t."""
    return load_library().kda_chunk_transition(k, v, g, beta, St, M, B, H, T, dk, dv, dtype, stream)


def kda_output_gate(o, gate, rms_weight, eps, y, B, H, T, dv, dtype, stream) -> int:
    """Eq. 6 output edge: y = Sigmoid(gate) * RMSNorm(o).  Returns the raw kda_status_t."""
    return load_library().kda_output_gate(o, gate, rms_weight, eps, y, B, H, T, dv, dtype, stream)


def kda_kcp_compose(M, St, h0, S_in, R, B, H, dk, dv, stream) -> int:
    """Cross-device KCP prefix: S_in from the gathered (M_r, S~_r) of the R earlier segments."""
    return load_library().kda_kcp_compose(M, St, h0, S_in, R, B, H, dk, dv, stream)


def kda_spec_replay_verify(q, k, v, g, beta, S, o, n_replay, B, H, W, dk, dv, dtype, scale, stream) -> int:
    """Speculative-decode replay and verify over a W-token window.  Returns the raw kda_status_t."""
    return load_library().kda_spec_replay_verify(q, k, v, g, beta, S, o, n_replay, B, H, W, dk, dv, dtype, scale,
                                                 stream)


def kda_spec_replay_verify_fused(q, k, v, z, A_log, g_min, beta, S, gate, rms_weight, eps, y, n_replay, B, H, W, dk,
                                 dv, dtype, scale, stream) -> int:
    """The replay loop with the Eq. 5 gate (z, A_log) and the Eq. 6 edge (gate,
    rms_weight -> y) folded in.  Returns the raw kda_status_t."""
    return load_library().kda_spec_replay_verify_fused(q, k, v, z, A_log, g_min, beta, S, gate, rms_weight, eps, y,
                                                       n_replay, B, H, W, dk, dv, dtype, scale, stream)


def kda_chunk_fwd_noalloc(q, k, v, g, beta, h0, o, h_T, B, H, T, dk, dv, dtype, chunk_size, scale, stream) -> int:
    """kda_chunk_fwd with libkda's own fixed scratch array (no workspace argument).
    For callers that cannot allocate device memory.  Returns the raw kda_status_t."""
    return load_library().kda_chunk_fwd_noalloc(q, k, v, g, beta, h0, o, h_T, B, H, T, dk, dv, dtype, chunk_size,
                                                scale, stream)


def kda_noalloc_scratch_bytes() -> int:
    return load_library().kda_noalloc_scratch_bytes()


def kda_recurrent_step(q, k, v, g, beta, S, o, B, H, dk, dv, dtype, scale, stream) -> int:
    return load_library().kda_recurrent_step(q, k, v, g, beta, S, o, B, H, dk, dv, dtype, scale, stream)


def kda_get_device_status(stream=None) -> int:
    return load_library().kda_get_device_status(stream)


def kda_debug_set_wait_limit(ns: int) -> int:
    return load_library().kda_debug_set_wait_limit(int(ns))


def kda_debug_inject_stall(on: bool) -> int:
    return load_library().kda_debug_inject_stall(1 if on else 0)


# ---- torch helpers ---------------------------------------------------------

def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError("q/k/v/g/beta must be bf16 or fp32, got %s" % t.dtype)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libkda takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libkda takes contiguous tensors")
    return t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def chunk_fwd(q, k, v, g, beta, h0=None, *, o=None, h_T=None, scale=0.0, chunk_size=0,
              output_final_state=True, workspace=None, stream=None, ckpt_interval=0, ckpt=None):
    """Prefill over [B, H, T, d] tensors (see kda_chunk_fwd in include/kda.h).

    Allocates o / h_T / workspace with torch when not given.  Returns (o, h_T),
    or (o, h_T, ckpt) when ckpt_interval > 0 (kda_chunk_fwd_ckpt: ckpt is
    [B, H, T // ckpt_interval, dk, dv] fp32, the state at every multiple of
    ckpt_interval tokens).
    """
    import torch
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if h_T is None and output_final_state:
        h_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    ws = kda_chunk_fwd_workspace_size(B, H, T, dk, dv, dt, chunk_size)
    if ws == (1 << 64) - 1:
        raise KdaError(2, "kda_chunk_fwd_workspace_size")
    if ws > 0 and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if ckpt_interval:
        if ckpt is None:
            ckpt = torch.empty(B, H, T // ckpt_interval, dk, dv, dtype=torch.float32, device=q.device)
        st = kda_chunk_fwd_ckpt(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o), _ptr(h_T),
                                _ptr(ckpt), ckpt_interval, B, H, T, dk, dv, dt, chunk_size, float(scale),
                                _ptr(workspace), wbytes, _stream(stream))
        if st != KDA_OK:
            raise KdaError(st, "kda_chunk_fwd_ckpt")
        return o, h_T, ckpt
    st = kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o), _ptr(h_T),
                       B, H, T, dk, dv, dt, chunk_size, float(scale), _ptr(workspace), wbytes, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd")
    return o, h_T


def chunk_transition(k, v, g, beta, *, out=None, stream=None):
    """(S~, M) of every chain's segment: S~ [B, H, dk, dv] and M [B, H, dk, dk]
    fp32 (kda_chunk_transition).  `out`, if given, is one fp32 buffer of
    B*H*(dk*dk + dk*dv) elements that receives M then S~ (so a rank can
    publish both with one collective); the returned tensors are views of it."""
    import torch
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    n = B * H
    if out is None:
        out = torch.empty(n * (dk * dk + dk * dv), dtype=torch.float32, device=k.device)
    m = out[:n * dk * dk].view(B, H, dk, dk)
    st = out[n * dk * dk:n * (dk * dk + dk * dv)].view(B, H, dk, dv)
    code = kda_chunk_transition(_ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(st), _ptr(m), B, H, T, dk, dv,
                                _dtype_code(k), _stream(stream))
    if code != KDA_OK:
        raise KdaError(code, "kda_chunk_transition")
    return st, m


def chunk_fwd_outgate(q, k, v, g, beta, gate, rms_weight, h0=None, *, eps=1e-6, y=None, h_T=None, scale=0.0,
                      chunk_size=0, output_final_state=True, workspace=None, stream=None):
    """Prefill with the fused Eq. 6 output edge: gate [B, H, T, dv] (dtype of q),
    rms_weight [H, dv] fp32.  Allocates y / h_T / workspace when not given.
    Returns (y, h_T)."""
    import torch
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if y is None:
        y = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if h_T is None and output_final_state:
        h_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    ws = kda_chunk_fwd_workspace_size(B, H, T, dk, dv, dt, chunk_size)
    if ws == (1 << 64) - 1:
        raise KdaError(2, "kda_chunk_fwd_workspace_size")
    if ws > 0 and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = kda_chunk_fwd_outgate(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(gate), _ptr(rms_weight),
                               float(eps), _ptr(y), _ptr(h_T), B, H, T, dk, dv, dt, chunk_size, float(scale),
                               _ptr(workspace), wbytes, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_outgate")
    return y, h_T


def chunk_fwd_gated(q, k, v, z, A_log, beta, h0=None, *, g_min=-5.0, o=None, h_T=None, scale=0.0, chunk_size=0,
                    output_final_state=True, workspace=None, stream=None):
    """Prefill with the fused Eq. 5 gate: z [B, H, T, dk] (dtype of q), A_log
    [H, dk] fp32.  Allocates o / h_T / workspace when not given.  Returns (o, h_T)."""
    import torch
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if h_T is None and output_final_state:
        h_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    ws = kda_chunk_fwd_workspace_size(B, H, T, dk, dv, dt, chunk_size)
    if ws == (1 << 64) - 1:
        raise KdaError(2, "kda_chunk_fwd_workspace_size")
    if ws > 0 and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = kda_chunk_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log), float(g_min), _ptr(beta), _ptr(h0),
                             _ptr(o), _ptr(h_T), B, H, T, dk, dv, dt, chunk_size, float(scale), _ptr(workspace),
                             wbytes, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_gated")
    return o, h_T


def output_gate(o, gate, rms_weight, eps=1e-6, *, y=None, stream=None):
    """Eq. 6 output edge over [B, H, T, dv] tensors; rms_weight [H, dv] fp32.  Returns y."""
    import torch
    B, H, T, dv = o.shape
    if y is None:
        y = torch.empty_like(o)
    st = kda_output_gate(_ptr(o), _ptr(gate), _ptr(rms_weight), float(eps), _ptr(y), B, H, T, dv, _dtype_code(o),
                         _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_output_gate")
    return y


def spec_replay_verify(q, k, v, g, beta, S, n_replay, *, o=None, scale=0.0, stream=None):
    """Window of W tokens per sequence ([B, H, W, d]): replay the first
    n_replay[b] (accepted, committed to S in place), verify the rest (o).
    n_replay: [B] int32 CUDA tensor.  Returns o."""
    import torch
    B, H, W, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.zeros(B, H, W, dv, dtype=q.dtype, device=q.device)
    st = kda_spec_replay_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o), _ptr(n_replay),
                                B, H, W, dk, dv, _dtype_code(q), float(scale), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_spec_replay_verify")
    return o


def recurrent_step(q, k, v, g, beta, S, *, o=None, scale=0.0, stream=None):
    """One decode step over [B, H, d] tensors; S [B, H, dk, dv] fp32 updated in place.  Returns o."""
    import torch
    B, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    st = kda_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o), B, H, dk, dv,
                            _dtype_code(q), float(scale), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_recurrent_step")
    return o


def spec_replay_verify_fused(q, k, v, z, A_log, beta, S, gate, rms_weight, n_replay, *, g_min=-5.0, eps=1e-6, y=None,
                             scale=0.0, stream=None):
    """spec_replay_verify with the Eq. 5 gate on the inputs (z [B, H, W, dk],
    A_log [H, dk] fp32) and the Eq. 6 edge on the verified outputs (gate
    [B, H, W, dv], rms_weight [H, dv] fp32).  Returns y (zeros for replayed tokens)."""
    import torch
    B, H, W, dk = q.shape
    dv = v.shape[-1]
    if y is None:
        y = torch.zeros(B, H, W, dv, dtype=q.dtype, device=q.device)
    st = kda_spec_replay_verify_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log), float(g_min), _ptr(beta),
                                      _ptr(S), _ptr(gate), _ptr(rms_weight), float(eps), _ptr(y), _ptr(n_replay), B, H,
                                      W, dk, dv, _dtype_code(q), float(scale), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_spec_replay_verify_fused")
    return y
