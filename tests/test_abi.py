"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function include/kda.h declares, plans calls, and rejects bad arguments
synchronously with the documented status codes before touching a device."""
import ctypes
import os
import re

import pytest
import torch

from gated_delta_rule_117_b200 import build as kbuild
from gated_delta_rule_117_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert "kda_chunk_fwd" in names and "kda_recurrent_step" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(kda.EXPORTED)


def test_status_strings(lib):
    for code, name in enumerate(kda.STATUS_NAMES):
        assert kda.kda_status_string(code).startswith(name)
    assert kda.kda_status_string(999) == "KDA_ERR_UNKNOWN"
    assert kda.kda_version() >= 100


def test_plan(lib):
    p = kda.kda_chunk_fwd_plan(1, 2, 64, 16, 16, kda.KDA_DTYPE_F32, 16)
    assert p["chunk_size"] == 16 and p["launches"] == 1 and p["segments"] >= 1
    assert p["path"] == kda.KDA_PATH_SIMT16
    p = kda.kda_chunk_fwd_plan(1, 16, 4096, 128, 128, kda.KDA_DTYPE_BF16, 0)
    assert p["path"] == kda.KDA_PATH_TC32 and p["chunk_size"] == 32
    p = kda.kda_chunk_fwd_plan(1, 16, 4096, 128, 128, kda.KDA_DTYPE_F32, 0)
    assert p["path"] == kda.KDA_PATH_SIMT16
    with pytest.raises(kda.KdaError) as e:
        kda.kda_chunk_fwd_plan(1, 2, 64, 24, 16, kda.KDA_DTYPE_F32, 0)
    assert e.value.status == 2
    assert kda.kda_chunk_fwd_workspace_size(1, 2, 64, 24, 16, 0, 0) == (1 << 64) - 1


@pytest.mark.parametrize("B,H,T", [(1, 16, 4096), (1, 16, 1 << 20), (1, 8, 1024), (2, 2, 300), (1, 74, 512),
                                   (8, 32, 8192), (1, 75, 1 << 16), (1, 1, 511), (3, 5, 2000)])
def test_context_parallel_plan_and_workspace(lib, B, H, T):
    # the tensor-core plan: P = min(148 // BH, T // 256) segments of whole 32-token chunks when
    # BH <= 74 and P >= 2, else one CTA per chain; the workspace holds P - 1 transitions, P - 1
    # states from zero and P entering states per chain (64 KiB fp32 each) and two 32-bit flags
    # per transition, rounded up to 16 bytes
    p = kda.kda_chunk_fwd_plan(B, H, T, 128, 128, kda.KDA_DTYPE_BF16, 0)
    BH = B * H
    P = min(148 // BH, T // 256) if BH <= 74 else 1
    if P >= 2:
        seg = -(-(-(-T // P)) // 32) * 32
        P = -(-T // seg)
        assert (p["segments"], p["segment_tokens"], p["launches"]) == (P, seg, 4)
        flags = -(-(2 * BH * (P - 1) * 4) // 16) * 16
        assert p["workspace"] == BH * (3 * P - 2) * 65536 + flags
        assert (P - 1) * seg < T <= P * seg  # every segment holds tokens
    else:
        assert (p["segments"], p["segment_tokens"], p["launches"], p["workspace"]) == (1, T, 1, 0)
    assert kda.kda_chunk_fwd_workspace_size(B, H, T, 128, 128, kda.KDA_DTYPE_BF16, 0) == p["workspace"]


# Fake, never-dereferenced device addresses: validation must reject bad
# arguments before any CUDA call.
BASE = 1 << 40
N = 1 * 2 * 64 * 16 * 4  # bytes of one [1, 2, 64, 16] fp32 tensor


def _call(**over):
    B, H, T, dk, dv = 1, 2, 64, 16, 16
    n = N
    a = dict(q=BASE, k=BASE + n, v=BASE + 2 * n, g=BASE + 3 * n, beta=BASE + 4 * n, h0=BASE + 5 * n,
             o=BASE + 6 * n, h_T=BASE + 7 * n, B=B, H=H, T=T, dk=dk, dv=dv, dtype=0, chunk_size=16,
             scale=0.0, workspace=None, workspace_bytes=0, stream=None)
    a.update(over)
    return kda.kda_chunk_fwd(**a)


@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(T=-1), 1), (dict(scale=float("nan")), 1),
    (dict(dk=24), 2), (dict(dv=256), 2), (dict(chunk_size=64), 2), (dict(chunk_size=32, dtype=1), 2),
    (dict(dtype=7), 3), (dict(chunk_size=32), 3),
    (dict(k=BASE + N + 2), 4), (dict(h0=BASE + 5 * N + 8), 4), (dict(beta=BASE + 4 * N + 2), 4),
    (dict(o=BASE + 100 * 16), 5),           # o overlaps q
    (dict(h_T=BASE + 3 * N), 5),            # h_T == g
    (dict(h_T=BASE + 5 * N + 16), 5),       # h_T partially overlaps h0
])
def test_chunk_fwd_rejects(lib, over, code):
    assert _call(**over) == code


def test_chunk_fwd_allows_inplace_state(lib):
    st = _call(h_T=BASE + 5 * N)
    # valid arguments: on a machine without a GPU the call fails only at the device check
    if not torch.cuda.is_available():
        assert st in (7, 9)


def test_chunk_fwd_empty_batch_is_noop(lib):
    assert _call(B=0) == 0 and _call(H=0, q=None) == 0


def _ccall(**over):
    # kda_chunk_fwd_ckpt: the valid arguments of _call plus a checkpoint buffer past h_T
    n = N
    a = dict(q=BASE, k=BASE + n, v=BASE + 2 * n, g=BASE + 3 * n, beta=BASE + 4 * n, h0=BASE + 5 * n,
             o=BASE + 6 * n, h_T=BASE + 7 * n, ckpt=BASE + 8 * n, ckpt_interval=64, B=1, H=2, T=64, dk=16, dv=16,
             dtype=0, chunk_size=16, scale=0.0, workspace=None, workspace_bytes=0, stream=None)
    a.update(over)
    return kda.kda_chunk_fwd_ckpt(**a)


@pytest.mark.parametrize("over,code", [
    (dict(ckpt_interval=0), 1), (dict(ckpt_interval=32), 1), (dict(ckpt_interval=100), 1),
    (dict(ckpt=None), 1),                    # one snapshot due (T = 64) but no buffer
    (dict(ckpt=BASE + 8 * N + 4), 4),
    (dict(ckpt=BASE + 7 * N), 5),            # checkpoints overlap h_T
    (dict(ckpt=BASE + 2 * N), 5),            # checkpoints overlap v
    (dict(dk=24), 2),
])
def test_chunk_fwd_ckpt_rejects(lib, over, code):
    assert _ccall(**over) == code


def test_chunk_fwd_ckpt_needs_no_buffer_without_a_boundary(lib):
    st = _ccall(ckpt=None, T=63)
    if not torch.cuda.is_available():
        assert st in (7, 9)


def _gcall(**over):
    # kda_chunk_fwd_gated: _call's arguments with z in place of g plus A_log after h_T
    n = N
    a = dict(q=BASE, k=BASE + n, v=BASE + 2 * n, z=BASE + 3 * n, A_log=BASE + 8 * n, g_min=-5.0, beta=BASE + 4 * n,
             h0=BASE + 5 * n, o=BASE + 6 * n, h_T=BASE + 7 * n, B=1, H=2, T=64, dk=16, dv=16, dtype=0,
             chunk_size=16, scale=0.0, workspace=None, workspace_bytes=0, stream=None)
    a.update(over)
    return kda.kda_chunk_fwd_gated(**a)


@pytest.mark.parametrize("over,code", [
    (dict(g_min=-6.0), 1), (dict(g_min=0.0), 1), (dict(g_min=float("nan")), 1), (dict(A_log=None), 1),
    (dict(A_log=BASE + 8 * N + 2), 4),
    (dict(A_log=BASE + 6 * N), 5),           # A_log inside o
    (dict(z=BASE + N + 4), 4),
])
def test_chunk_fwd_gated_rejects(lib, over, code):
    assert _gcall(**over) == code


def _ocall(**over):
    n = 1 * 2 * 64 * 128 * 2  # bytes of one [1, 2, 64, 128] bf16 tensor
    a = dict(o=BASE, gate=BASE + n, rms_weight=BASE + 2 * n, eps=1e-6, y=BASE + 3 * n, B=1, H=2, T=64, dv=128,
             dtype=1, stream=None)
    a.update(over)
    return kda.kda_output_gate(**a)


@pytest.mark.parametrize("over,code", [
    (dict(o=None), 1), (dict(eps=-1.0), 1), (dict(eps=float("inf")), 1), (dict(T=-1), 1),
    (dict(dv=100), 2), (dict(dtype=4), 3),
    (dict(gate=BASE + 32768 + 8), 4), (dict(rms_weight=BASE + 65536 + 4), 4),
    (dict(y=BASE + 32768), 5),          # y overlaps gate
    (dict(y=BASE + 16), 5),             # y partially overlaps o
])
def test_output_gate_rejects(lib, over, code):
    assert _ocall(**over) == code


def test_output_gate_in_place_and_empty(lib):
    assert _ocall(B=0) == 0
    st = _ocall(y=BASE)  # y == o: in place is allowed
    if not torch.cuda.is_available():
        assert st in (7, 9)


@pytest.mark.parametrize("over,code", [
    (dict(R=-1), 1), (dict(S_in=None), 1), (dict(M=None), 1), (dict(dk=24), 2),
    (dict(St=BASE + (1 << 20) + 4), 4),
    (dict(S_in=BASE), 5),                 # S_in overlaps M
])
def test_kcp_compose_rejects(lib, over, code):
    a = dict(M=BASE, St=BASE + (1 << 20), h0=BASE + (2 << 20), S_in=BASE + (3 << 20), R=2, B=1, H=2, dk=64, dv=64,
             stream=None)
    a.update(over)
    assert kda.kda_kcp_compose(**a) == code


@pytest.mark.parametrize("over,code", [
    (dict(W=-1), 1), (dict(n_replay=None), 1), (dict(dk=8), 2), (dict(dtype=3), 3),
    (dict(S=BASE + (1 << 22) + 8), 4), (dict(n_replay=BASE + (3 << 22) + 2), 4),
    (dict(o=BASE + (1 << 22)), 5),       # o inside S
])
def test_spec_replay_verify_rejects(lib, over, code):
    a = dict(q=BASE, k=BASE + 65536, v=BASE + 2 * 65536, g=BASE + 3 * 65536, beta=BASE + 4 * 65536, S=BASE + (1 << 22),
             o=BASE + (2 << 22), n_replay=BASE + (3 << 22), B=2, H=2, W=4, dk=64, dv=64, dtype=1, scale=0.0,
             stream=None)
    a.update(over)
    assert kda.kda_spec_replay_verify(**a) == code


def _dcall(**over):
    B, H, dk, dv = 4, 2, 16, 16
    n = 4096
    a = dict(q=BASE, k=BASE + n, v=BASE + 2 * n, g=BASE + 3 * n, beta=BASE + 4 * n, S=BASE + 5 * n,
             o=BASE + 5 * n + B * H * dk * dv * 4, B=B, H=H, dk=dk, dv=dv, dtype=1, scale=0.0, stream=None)
    a.update(over)
    return kda.kda_recurrent_step(**a)


@pytest.mark.parametrize("over,code", [
    (dict(S=None), 1), (dict(B=-1), 1), (dict(scale=float("inf")), 1),
    (dict(dk=8), 2), (dict(dtype=5), 3),
    (dict(S=BASE + 5 * 4096 + 4), 4), (dict(beta=BASE + 4 * 4096 + 1), 4),
    (dict(o=BASE + 5 * 4096), 5),   # o inside S
    (dict(S=BASE + 2 * 4096), 5),   # S overlaps v..beta
])
def test_recurrent_step_rejects(lib, over, code):
    assert _dcall(**over) == code


def test_no_cpu_fallback_without_gpu(lib):
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert _dcall() in (7, 9)
