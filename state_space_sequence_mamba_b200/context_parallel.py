"""Prefill split along the sequence over the ranks of a process group (context parallelism).

Rank k holds tokens [k L_r, (k + 1) L_r) of every sequence. The recurrence is linear in the
state ("Mamba-3: Improved Sequence Modeling using State Space Principles", Sec. 3.1.1 Prop. 1)
and its frame is an accumulated rotation of B and C (Sec. 3.2.2 Prop. 4), so the ranks need
one exchange of compact per-segment summaries, not of the tokens:

1. ``last_token``: every rank's last token (raw B per head, x) is all-gathered; rank k takes
   rank k-1's as its previous token.
2. ``segment_state``: every rank runs its own tokens without output (m3_scan_state): rank 0
   from the true initial state, every other rank from zero with angle 0 at its start and the
   previous token folded in. The end states (h, angle sum, summed log-decay: about
   N P + N / 2 + 1 floats per unit) are all-gathered.
3. ``finish``: rank k combines the end states of ranks 0 .. k-1 into the state at its start
   (m3_state_combine) and runs the full scan (m3_scan_fwd) from there. The last rank's final
   state is the sequence's.

Every step runs in the library's kernels; this module only moves tensors between ranks. The
phases are separate functions so that a single device can run the ranks one after another.
"""
from __future__ import annotations

import torch

from . import binding as m3


class DeviceOps:
    """The library's kernels (the default); tests may pass stand-ins with the same methods."""

    def scan_state(self, t, init, chunk, bc_norm, scalar):
        return m3.scan_state(**t, init=init, chunk=chunk, bc_norm=bc_norm, **scalar)

    def state_combine(self, h, phi, lam_sum):
        return m3.state_combine(h.contiguous(), phi.contiguous(), lam_sum.contiguous())

    def scan_fwd(self, t, init, final, chunk, bc_norm, scalar):
        return m3.scan_fwd(**t, init=init, final=final, chunk=chunk, bc_norm=bc_norm, **scalar)


def last_token(t):
    """This rank's last token as the next rank's stored previous token: raw B expanded per head
    [b, H, R, N] and x [b, H, R, P]."""
    x, B = t["x"], t["B"]
    H, G = x.shape[2], B.shape[2]
    heads = torch.arange(H, device=B.device) // (H // G)
    return B[:, -1].index_select(1, heads).contiguous(), x[:, -1].contiguous()


def segment_state(rank, t, init, prev, chunk, bc_norm, scalar, ops):
    """This rank's end state from its own start: the true initial state on rank 0, else zero
    (angle 0) with the previous rank's last token ``prev`` = (B, x) folded in."""
    if rank == 0:
        start = init
    else:
        pB, px = prev
        b, H, R, N = pB.shape
        P = px.shape[-1]
        start = m3.State(torch.zeros(b, H, N, P, device=pB.device),
                         torch.zeros(b, H, N // 2, device=pB.device), pB, px)
    return ops.scan_state(t, start, chunk, bc_norm, scalar)


def finish(rank, world, t, init, prev, seg_h, seg_phi, seg_lam, chunk, bc_norm, scalar, ops):
    """The full scan of this rank's tokens from the state at its start, combined from the
    gathered end states of ranks 0 .. rank-1 (stacked on dim 0). Returns (y, final state; the
    latter on the last rank only, else None)."""
    if rank == 0:
        start = init
    else:
        h0, phi0 = ops.state_combine(seg_h[:rank], seg_phi[:rank], seg_lam[:rank])
        start = m3.State(h0, phi0, prev[0], prev[1])
    return ops.scan_fwd(t, start, rank == world - 1, chunk, bc_norm, scalar)


def _all_gather(dist, group, tensor, world):
    out = [torch.empty_like(tensor) for _ in range(world)]
    dist.all_gather(out, tensor.contiguous(), group=group)
    return out


def scan_context_parallel(x, B, C, theta, dt, A, lam, B_bias=None, C_bias=None, init=None,
                          chunk=64, bc_norm=False, dt_bias=None, flags=0, group=None,
                          ops=None):
    """Prefill of this rank's tokens of every sequence, with the earlier ranks' tokens taken
    into account through one exchange (two all-gathers). ``init`` (rank 0 only) is the state
    before the sequence. Returns (y of this rank's tokens, the final state on the last rank,
    else None). Every rank must call it, in the same order as its other collectives."""
    import torch.distributed as dist
    ops = ops or DeviceOps()
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    t = dict(x=x, B=B, C=C, theta=theta, dt=dt, A=A, lam=lam, B_bias=B_bias, C_bias=C_bias)
    scalar = dict(dt_bias=dt_bias, flags=flags)
    lb, lx = last_token(t)
    gB, gx = _all_gather(dist, group, lb, world), _all_gather(dist, group, lx, world)
    prev = (gB[rank - 1], gx[rank - 1]) if rank > 0 else None
    h, phi, lsum = segment_state(rank, t, init, prev, chunk, bc_norm, scalar, ops)
    seg_h = torch.stack(_all_gather(dist, group, h, world))
    seg_phi = torch.stack(_all_gather(dist, group, phi, world))
    seg_lam = torch.stack(_all_gather(dist, group, lsum, world))
    return finish(rank, world, t, init, prev, seg_h, seg_phi, seg_lam, chunk, bc_norm, scalar,
                  ops)
