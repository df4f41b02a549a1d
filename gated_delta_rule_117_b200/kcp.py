"""Cross-device KDA context parallelism (Kimi K3 report, section 5.1.2, Eq. 17).

One long sequence is split over the ranks of a process group: rank r holds
tokens [r*T_r, (r+1)*T_r) of every chain.  A segment maps its entering state S
to S~ + M S (the recurrence is linear in S), so

1. every rank computes (S~_r, M_r) of its own segment: S~ is the final state of
   a prefill from a zero state, M the final state of a prefill from h0 = I with
   v = 0 (dk == dv);
2. one exchange: all-gather of the pairs (2 x 64 KiB fp32 per chain per rank
   at d = 128), NCCL over NVLink on a GPU group;
3. rank R composes the state entering its segment from h0 and the pairs of
   ranks < R (kda_kcp_compose, on the device);
4. rank R runs its prefill from that state: its outputs, and on the last rank
   the sequence's final state.

The compute steps run in libkda's kernels; this module only orders them around
the collective.  `ops` exists so the orchestration can be exercised with CPU
stand-ins on a gloo group.
"""
from __future__ import annotations

from . import kda


class LibkdaOps:
    """The steps of KCP on the device, through libkda's C ABI."""

    @staticmethod
    def transition(q, k, v, g, beta, scale=0.0):
        import torch
        B, H, T, dk = q.shape
        if v.shape[-1] != dk:
            raise ValueError("cross-device KCP needs dk == dv (M is taken as the state from h0 = I)")
        _, st = kda.chunk_fwd(q, k, v, g, beta, None, scale=scale)
        eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, H, dk, dk).contiguous()
        _, m = kda.chunk_fwd(q, k, torch.zeros_like(v), g, beta, eye, scale=scale)
        return st, m

    @staticmethod
    def compose(ms, sts, h0, like):
        import torch
        B, H, dk, dv = like.shape
        s_in = torch.empty_like(like)
        R = len(ms)
        m = torch.stack(ms).contiguous() if R else None
        st = torch.stack(sts).contiguous() if R else None
        code = kda.kda_kcp_compose(kda._ptr(m), kda._ptr(st), kda._ptr(h0), kda._ptr(s_in), R, B, H, dk, dv,
                                   kda._stream(None))
        if code != kda.KDA_OK:
            raise kda.KdaError(code, "kda_kcp_compose")
        return s_in

    @staticmethod
    def prefill(q, k, v, g, beta, h0, scale=0.0):
        return kda.chunk_fwd(q, k, v, g, beta, h0, scale=scale)


def kcp_prefill(q, k, v, g, beta, h0=None, *, group=None, scale=0.0, ops=LibkdaOps):
    """This rank's part of a prefill whose sequence is split over `group` in
    rank order.  q, k, v, g, beta: this rank's tokens ([B, H, T_r, d]); h0: the
    state entering the whole sequence (the same on every rank, or None).
    Returns (o for this rank's tokens, state after this rank's segment): the
    last rank's state is the sequence's final state.  Every rank takes the
    same collective steps (two all-gathers)."""
    import torch
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    st, m = ops.transition(q, k, v, g, beta, scale)
    st_all = [torch.empty_like(st) for _ in range(world)]
    m_all = [torch.empty_like(m) for _ in range(world)]
    dist.all_gather(st_all, st.contiguous(), group=group)
    dist.all_gather(m_all, m.contiguous(), group=group)
    like = st if h0 is None else h0
    s_in = ops.compose(m_all[:rank], st_all[:rank], h0, like)
    return ops.prefill(q, k, v, g, beta, s_in, scale)
