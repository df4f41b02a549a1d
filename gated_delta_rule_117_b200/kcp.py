"""Cross-device KDA context parallelism (Kimi K3 report, section 5.1.2, Eq. 17).

One long sequence is split over the ranks of a process group: rank r holds
tokens [r*T_r, (r+1)*T_r) of every chain.  A segment maps its entering state S
to S~ + M S (the recurrence is linear in S), so

1. every rank computes (S~_r, M_r) of its own segment: S~ is the final state of
   the segment run from a zero state, M = M_T ... M_1 the product of its token
   transitions; on the tensor-core path one transition-only launch gives both
   (no q loads, no outputs); elsewhere two prefills give them (S~ from a zero
   state, M from h0 = I with v = 0, dk == dv);
2. one exchange: one all-gather of each rank's packed pair [M | S~] (2 x 64 KiB
   fp32 per chain at d = 128), NCCL over NVLink on a GPU group;
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


def pack(m, st):
    """One flat buffer [M | S~] per rank (the payload of the single all-gather)."""
    import torch
    return torch.cat([m.reshape(-1), st.reshape(-1)])


def unpack(flat, B, H, dk, dv):
    n = B * H * dk * dk
    return flat[:n].view(B, H, dk, dk), flat[n:n + B * H * dk * dv].view(B, H, dk, dv)


class LibkdaOps:
    """The steps of KCP on the device, through libkda's C ABI."""

    @staticmethod
    def transition_packed(q, k, v, g, beta, scale=0.0):
        """This rank's [M | S~] as one flat fp32 tensor."""
        import torch
        B, H, T, dk = q.shape
        dv = v.shape[-1]
        if q.dtype == torch.bfloat16 and dk == 128 and dv == 128:
            flat = torch.empty(B * H * (dk * dk + dk * dv), dtype=torch.float32, device=q.device)
            kda.chunk_transition(k, v, g, beta, out=flat)
            return flat
        if dv != dk:
            raise ValueError("cross-device KCP on the CUDA-core path needs dk == dv (M is the state from h0 = I)")
        _, st = kda.chunk_fwd(q, k, v, g, beta, None, scale=scale)
        eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, H, dk, dk).contiguous()
        _, m = kda.chunk_fwd(q, k, torch.zeros_like(v), g, beta, eye, scale=scale)
        return pack(m, st)

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
    same collective step: one all-gather."""
    import torch
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, H, _, dk = q.shape
    dv = v.shape[-1]
    flat = ops.transition_packed(q, k, v, g, beta, scale).contiguous()
    gathered = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(gathered, flat, group=group)
    pairs = [unpack(gathered[r], B, H, dk, dv) for r in range(rank)]
    like = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device) if h0 is None else h0
    s_in = ops.compose([m for m, _ in pairs], [st for _, st in pairs], h0, like)
    return ops.prefill(q, k, v, g, beta, s_in, scale)
