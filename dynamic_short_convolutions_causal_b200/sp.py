"""Sequence-parallel plumbing for the low-rank dynamic short convolution.

A sequence of length P*T is split into P consecutive shards of T tokens, shard i on
position i of ``seq_ranks`` (by default the process group's ranks in order).  The
causal window ("Convolucoes Curtas Dinamicas Melhoram Transformers", Metodologia:
Mecanismo, y_t = x_t + sum_{k<W} w(t)_k x_{t-k}) reaches W-1 tokens back, so shards
need only a (W-1)-row halo from their neighbours:
  forward:  the previous shard's last W-1 rows of x;
  backward: the next shard's first W-1 rows of dy and z (and the previous shard's x,
            for the filter gradient of the first W-1 rows).
Each rank runs the library's kernels on its own shard and then the halo fix-up entry
points (dsc_fwd_lowrank_halo / dsc_bwd_lowrank_halo), which recompute or complete the
W-1 affected rows; dU is then summed over the ranks like a data-parallel gradient.

These helpers move halos with torch.distributed point-to-point calls (NCCL between
GPUs, gloo on CPU) and call the binding; they do no arithmetic of the method.  A halo
exchange is one hop, so every shard must hold at least W-1 tokens.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def _ranks(seq_ranks: Optional[Sequence[int]]):
    if seq_ranks is not None:
        ranks = list(seq_ranks)
    elif dist.is_available() and dist.is_initialized():
        ranks = list(range(dist.get_world_size()))
    else:
        ranks = [0]
    me = dist.get_rank() if (dist.is_available() and dist.is_initialized()) else 0
    if me not in ranks:
        raise ValueError("sp: this rank (%d) is not in seq_ranks %s" % (me, ranks))
    return ranks, ranks.index(me)


def shard_tokens(T_total: int, rank_pos: int, n_shards: int) -> range:
    """Tokens of a sequence of T_total held by shard `rank_pos` of `n_shards` (equal
    shards; T_total must divide evenly)."""
    if T_total % n_shards:
        raise ValueError("sp: sequence length %d does not split into %d equal shards" % (T_total, n_shards))
    T = T_total // n_shards
    return range(rank_pos * T, (rank_pos + 1) * T)


def _exchange(send_fwd: Optional[torch.Tensor], send_bwd: Sequence[torch.Tensor], like_fwd: torch.Tensor,
              like_bwd: Sequence[torch.Tensor], ranks, pos):
    """One round of point-to-point halo traffic.  send_fwd goes to the next shard and the
    previous shard's comes back; each tensor of send_bwd goes to the previous shard and
    the next shard's come back.  Returns (from_prev or None, [from_next...] or None)."""
    ops = []
    prev = ranks[pos - 1] if pos > 0 else None
    nxt = ranks[pos + 1] if pos + 1 < len(ranks) else None
    from_prev, from_next = None, None
    if send_fwd is not None:
        if nxt is not None:
            ops.append(dist.P2POp(dist.isend, send_fwd.contiguous(), nxt))
        if prev is not None:
            from_prev = torch.empty_like(like_fwd)
            ops.append(dist.P2POp(dist.irecv, from_prev, prev))
    if send_bwd:
        if prev is not None:
            for t in send_bwd:
                ops.append(dist.P2POp(dist.isend, t.contiguous(), prev))
        if nxt is not None:
            from_next = [torch.empty_like(t) for t in like_bwd]
            for t in from_next:
                ops.append(dist.P2POp(dist.irecv, t, nxt))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    return from_prev, from_next


def exchange_prev(x: torch.Tensor, W: int, seq_ranks: Optional[Sequence[int]] = None) -> Optional[torch.Tensor]:
    """x [B,T,D] of this shard -> x_prev [B,W-1,D], the previous shard's last W-1 rows
    (None on the first shard, or when W = 1)."""
    ranks, pos = _ranks(seq_ranks)
    if W == 1 or len(ranks) == 1:
        return None
    if x.shape[1] < W - 1:
        raise ValueError("sp: a shard of %d tokens is shorter than the W-1 = %d row halo" % (x.shape[1], W - 1))
    tail = x[:, x.shape[1] - (W - 1):, :].contiguous()
    from_prev, _ = _exchange(tail, [], tail, [], ranks, pos)
    return from_prev


def exchange_next(dy: torch.Tensor, z: torch.Tensor, W: int, seq_ranks: Optional[Sequence[int]] = None
                  ) -> Tuple[Optional[torch.Tensor], Optional[torch.Tensor]]:
    """dy [B,T,D], z [B,T,R] of this shard -> (dy_next [B,W-1,D], z_next [B,W-1,R]), the
    next shard's first W-1 rows ((None, None) on the last shard, or when W = 1)."""
    ranks, pos = _ranks(seq_ranks)
    if W == 1 or len(ranks) == 1:
        return None, None
    if dy.shape[1] < W - 1:
        raise ValueError("sp: a shard of %d tokens is shorter than the W-1 = %d row halo" % (dy.shape[1], W - 1))
    heads = [dy[:, :W - 1, :].contiguous(), z[:, :W - 1, :].contiguous()]
    _, from_next = _exchange(None, heads, heads[0], heads, ranks, pos)
    if from_next is None:
        return None, None
    return from_next[0], from_next[1]


def fwd_lowrank(x, z, U, y, G: int, W: int, seq_ranks=None):
    """Forward of this rank's shard: the shard's own call, the x halo from the previous
    shard, and the fix-up of rows t < W-1.  Returns (y, x_prev) (x_prev is kept for the
    backward; None on the first shard)."""
    import dynamic_short_convolutions_causal_b200 as dsc
    x_prev = exchange_prev(x, W, seq_ranks)
    dsc.dsc_fwd_lowrank(x, z, U, y, G, W)
    if x_prev is not None:
        dsc.dsc_fwd_lowrank_halo(x, z, U, x_prev, y, G, W)
    return y, x_prev


def bwd_lowrank(x, z, U, dy, dx, dz, dU, workspace, G: int, W: int, x_prev=None, seq_ranks=None,
                sum_dU: bool = True):
    """Backward of this rank's shard: the shard's own call, the dy / z halo from the next
    shard, the fix-ups (dx rows t >= T-(W-1); dz rows t < W-1 and dU with x_prev), and,
    when sum_dU, dU summed over the process group (every rank must call it)."""
    import dynamic_short_convolutions_causal_b200 as dsc
    from . import dp
    dy_next, z_next = exchange_next(dy, z, W, seq_ranks)
    dsc.dsc_bwd_lowrank(x, z, U, dy, dx, dz, dU, workspace, G, W)
    if x_prev is not None or dy_next is not None:
        dsc.dsc_bwd_lowrank_halo(x_prev, z, U, dy, dy_next, z_next, dx, dz, dU, G, W)
    if sum_dU:
        dp.allreduce_weight_grad(dU)
    return dx, dz, dU
