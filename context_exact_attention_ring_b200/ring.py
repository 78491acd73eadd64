"""Ring attention across GPUs: the send/receive loop of "Lesson 8: Context
Parallelism", section 2, with one process per GPU (torch.distributed).

Rank r keeps its query shard fixed.  At step t it holds the K/V block that
started on rank (r - t) mod P and folds it into its (m, l, O) state with
ring_attn_step, while the same block is already on its way to rank r+1 and
the next one is arriving from rank r-1 (a double buffer: the transfer of the
next block overlaps the step).  Blocks land in this GPU's own memory before a
kernel reads them: every kernel reads local memory only.  The backward runs
the same loop with ring_attn_step_bwd; the dK, dV sums of a block travel with
it and take one last hop home.  helix_decode is the decode's
exchange: per-shard partials, one all-gather, and the merge on every rank.
ring_attention puts the forward and backward loops under torch autograd.

The chunk ownership follows the splits of ring_attn_fwd (see split_chunks);
the step functions default to this package's kernels and can be replaced
(tests drive the loop on CPU ranks with a stand-in step).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def split_chunks(P: int, layout: str) -> list[list[int]]:
    """Chunk ids owned by each rank, in shard order.  'contiguous[k]': rank r
    owns chunks r*k .. r*k+k-1; 'zigzag[k]' (k >= 2, default 2): slot j of rank
    r is chunk (j//2)*P + r for even j and P*k-1-(j//2)*P-r for odd j;
    'striped': rank r owns its stripe, numbered r (token t on rank t mod P)."""
    name = layout.rstrip("0123456789")
    k = int(layout[len(name):] or (2 if name == "zigzag" else 1))
    if name == "contiguous":
        return [[r * k + j for j in range(k)] for r in range(P)]
    if name == "zigzag":
        if k < 2:
            raise ValueError(layout)
        return [[(j // 2) * P + r if j % 2 == 0 else P * k - 1 - (j // 2) * P - r for j in range(k)]
                for r in range(P)]
    if name == "striped" and k == 1:
        return [[r] for r in range(P)]
    raise ValueError(layout)


def shard_rows(S: int, P: int, layout: str, rank: int) -> torch.Tensor:
    """Token positions of rank `rank`'s shard, in shard order."""
    if layout.startswith("striped"):
        return torch.arange(rank, S, P)
    own = split_chunks(P, layout)
    C = S // (P * len(own[0]))
    return torch.cat([torch.arange(c * C, (c + 1) * C) for c in own[rank]])


class Ring:
    """Neighbour exchange on a process group: rank r sends to r+1, receives from r-1."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def _global(self, r: int) -> int:
        return r if self.group is None else dist.get_global_rank(self.group, r)

    def shift(self, send: list, recv: list) -> list:
        """Post sends of `send` to the next rank and receives into `recv` from
        the previous one; returns the requests (wait on them before using
        `recv` or reusing `send`)."""
        if self.world == 1:
            return []
        nxt, prv = self._global((self.rank + 1) % self.world), self._global((self.rank - 1) % self.world)
        ops = [dist.P2POp(dist.isend, t, nxt, self.group) for t in send]
        ops += [dist.P2POp(dist.irecv, t, prv, self.group) for t in recv]
        return dist.batch_isend_irecv(ops)


def _wait(reqs):
    for r in reqs:
        r.wait()


def ring_forward(q_shard, k_block, v_block, layout="zigzag", causal=True, scale=None, ring=None, step=None,
                 new_state=None, finalize=None):
    """Attention of this rank's query shard against every rank's K/V block.

    q_shard [B, S_loc, Hq, D], k_block, v_block [B, S_loc, Hkv, D]: this rank's
    shard (its chunks stacked in split_chunks order, or its stripe).  Returns
    (out [B, S_loc, Hq, D], lse [B, Hq, S_loc]) for the shard."""
    from . import new_state as _new_state, ring_attn_state_finalize, ring_attn_step
    ring = ring or Ring()
    step = step or ring_attn_step
    P, r = ring.world, ring.rank
    own = split_chunks(P, layout)
    C = q_shard.shape[1] // len(own[r])
    stripes = P if layout.startswith("striped") else 0
    B, S_loc, Hq, D = q_shard.shape
    m, l, O = (new_state or _new_state)(B, Hq, S_loc, D, device=q_shard.device)
    cur = [k_block.contiguous(), v_block.contiguous()]
    # received blocks alternate between two buffers of the loop's own: the caller's block is
    # only ever sent, never overwritten
    bufs = [[torch.empty_like(x) for x in cur] for _ in range(min(2, P - 1))]
    for t in range(P):
        src = (r - t) % P
        nxt = bufs[t % 2] if t < P - 1 else None
        reqs = ring.shift(cur, nxt) if t < P - 1 else []
        step(q_shard, cur[0], cur[1], m, l, O, own[r], own[src], C, causal=causal, scale=scale, stripes=stripes)
        _wait(reqs)
        if t < P - 1:
            cur = nxt
    return (finalize or ring_attn_state_finalize)(m, l, O, dtype=q_shard.dtype)


def ring_backward(q_shard, k_block, v_block, out_shard, lse_shard, dout_shard, layout="zigzag", causal=True,
                  scale=None, ring=None, step=None, delta_fn=None):
    """Gradients (dq, dk, dv) of this rank's shard.  dK, dV of a block are
    summed by every rank it visits, then sent home.  float32 sums; the results
    take the dtype of q.

    A block's running sums travel one hop behind it: at step t this rank
    computes its own contribution to the block it holds into a fresh buffer
    while the sums the previous ranks made for that block arrive from rank
    r-1; it then adds the two and sends them on to rank r+1, where they arrive
    during the next step.  Only the last hop home is not hidden behind a step."""
    from . import ring_attn_bwd_delta, ring_attn_step_bwd
    ring = ring or Ring()
    step = step or ring_attn_step_bwd
    P, r = ring.world, ring.rank
    own = split_chunks(P, layout)
    C = q_shard.shape[1] // len(own[r])
    stripes = P if layout.startswith("striped") else 0
    delta = (delta_fn or ring_attn_bwd_delta)(out_shard, dout_shard)
    f32 = dict(device=q_shard.device, dtype=torch.float32)
    dq = torch.zeros(q_shard.shape, **f32)
    kv = [k_block.contiguous(), v_block.contiguous()]
    # as in ring_forward: the caller's block is only sent; received blocks alternate between two
    # buffers of the loop's own
    kv_bufs = [[torch.empty_like(x) for x in kv] for _ in range(min(2, P - 1))]
    # this step's contribution to the held block's dK, dV (two buffers: the one sent at step t is
    # not touched before that send has completed, at step t+1), and the sums arriving for it
    mine = [[torch.empty(k_block.shape, **f32), torch.empty(v_block.shape, **f32)] for _ in range(min(2, P))]
    g_in = [torch.empty(k_block.shape, **f32), torch.empty(v_block.shape, **f32)]
    g_reqs = []
    for t in range(P):
        src = (r - t) % P
        kv_nxt = kv_bufs[t % 2] if t < P - 1 else None
        reqs = ring.shift(kv, kv_nxt) if t < P - 1 else []   # the next block arrives during the step
        g = mine[t % 2]
        g[0].zero_()
        g[1].zero_()
        step(q_shard, kv[0], kv[1], dout_shard, lse_shard, delta, dq, g[0], g[1], own[r], own[src], C,
             causal=causal, scale=scale, stripes=stripes)
        if t > 0:
            _wait(g_reqs)                  # the sums of this block from the ranks it visited before
            g[0].add_(g_in[0])
            g[1].add_(g_in[1])
        if P > 1:
            # the block's sums follow it to rank r+1 (home after step P-1); the sums of the block
            # held at step t+1 come from rank r-1
            g_reqs = ring.shift(g, g_in)
        _wait(reqs)
        if t < P - 1:
            kv = kv_nxt
    if P > 1:
        _wait(g_reqs)                      # this rank's own block, summed by every rank
        g = g_in
    return dq.to(q_shard.dtype), g[0].to(k_block.dtype), g[1].to(v_block.dtype)


class RingAttention(torch.autograd.Function):
    """Autograd over the cross-GPU ring: forward is ring_forward, backward is
    ring_backward on the saved shard, out and lse (the dK, dV of this rank's
    block come home with it).  fwd_kw / bwd_kw pass the optional step
    functions of the two loops."""

    @staticmethod
    def forward(ctx, q_shard, k_block, v_block, layout, causal, scale, ring, fwd_kw, bwd_kw):
        q_shard, k_block, v_block = q_shard.contiguous(), k_block.contiguous(), v_block.contiguous()
        out, lse = ring_forward(q_shard, k_block, v_block, layout, causal, scale, ring, **(fwd_kw or {}))
        ctx.save_for_backward(q_shard, k_block, v_block, out, lse)
        ctx.cfg = (layout, causal, scale, ring, bwd_kw or {})
        return out

    @staticmethod
    def backward(ctx, dout):
        q_shard, k_block, v_block, out, lse = ctx.saved_tensors
        layout, causal, scale, ring, bwd_kw = ctx.cfg
        dq, dk, dv = ring_backward(q_shard, k_block, v_block, out, lse, dout.to(q_shard.dtype).contiguous(), layout,
                                   causal, scale, ring, **bwd_kw)
        return dq, dk, dv, None, None, None, None, None, None


def ring_attention(q_shard, k_block, v_block, layout="zigzag", causal=True, scale=None, ring=None, fwd_kw=None,
                   bwd_kw=None):
    """This rank's output of the cross-GPU ring, differentiable by autograd
    (RingAttention).  Every rank calls it, and later its backward, in step."""
    return RingAttention.apply(q_shard, k_block, v_block, layout, causal, scale, ring, fwd_kw, bwd_kw)


def helix_decode(q, k_shard, v_shard, shard_len, scale=None, group=None, partial=None, merge=None, gather=None):
    """Split-KV single-token decode across GPUs ("NVIDIA unveils Helix
    Parallelism", Phase 1, KV parallelism): rank r holds shard r of every
    sequence's KV cache and computes, over its shard, the normalised partial
    (O_r, lse_r) of every query head; the ranks exchange the partials with one
    all-gather of B*Hq*(D+1) floats each, and every rank merges them with the
    section-3 update of "Lesson 8" applied to whole partial states:
        lse = m* + ln sum_r e^(lse_r - m*),  out = sum_r e^(lse_r - lse) O_r.

    q [B, Hq, D] (the same on every rank); k_shard, v_shard [B, C, Hkv, D]
    with the first shard_len[b] rows of sequence b valid (int32 [B], e.g. the
    fill counts of ring_attn_kv_append); an empty shard gives lse_r = -inf and
    O_r = 0.  Returns (out [B, Hq, D], lse [B, Hq]), the same on every rank.
    The step functions default to this package's kernels (the decode over one
    chunk, and the merge) and can be replaced (tests run the exchange on CPU
    ranks with stand-ins).  gather(t) returns every rank's t in rank order; it
    defaults to one all_gather over `group`."""
    from . import ring_attn_decode_partial, ring_attn_merge
    if partial is None:
        def partial(q_, k_, v_, lens_, scale_):
            return ring_attn_decode_partial(q_, k_, v_, lens_, 1, scale_)
    if merge is None:
        def merge(parts_, lses_):
            return ring_attn_merge(parts_, lses_, dtype=q.dtype)
    if gather is None:
        def gather(t):
            got = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
            dist.all_gather(got, t, group=group)
            return got
    part, plse = partial(q, k_shard, v_shard, shard_len, scale)          # [B, Hq, 1, D], [B, Hq, 1]
    B, Hq, D = part.shape[0], part.shape[1], part.shape[-1]
    mine = torch.cat([part.reshape(B, Hq, D), plse.reshape(B, Hq, 1)], dim=-1).contiguous()
    allp = torch.stack(gather(mine), dim=2)                               # [B, Hq, P, D + 1]
    return merge(allp[..., :D].contiguous(), allp[..., D].contiguous())
