"""Sequence parallelism of the DiT attention across GPUs (one process per GPU).

The ReGenVC decoder shards each window's tokens over 8 GPUs with unified
sequence parallelism (blog page, "Methodology -- deep read": Ulysses U = 4 x
Ring R = 2) and stays exact ("Technical innovations"):

* Ulysses: an all-to-all turns a rank's sequence shard of every head into the
  whole sequence of its share of the heads (and back after the attention);
* Ring: each rank keeps its queries while the key/value shards travel around
  the ring; the partial attention over each visiting shard is merged into the
  running result by its log-sum-exp (regen_lse_merge), which is exact.

torch.distributed carries the data (NCCL over NVLink on GPUs): all_to_all_single
for Ulysses, batched isend/irecv to the ring neighbours for Ring, the next
shard received while the current one is computed. The attention and the merge
run in the library's kernels; the two functions that compute them are
parameters, so that the exchange logic can also run on CPU ranks (gloo) with
another implementation of the same arithmetic.

Layouts: [B, H, S, D] per rank, as everywhere in this library. Sequence shards
are contiguous token ranges; a rank's RoPE positions are its token offset plus
the local index (regen_rope3d_shard).
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist


def _kernel_attn(q, k, v, scale):
    from . import attn_fwd
    return attn_fwd(q, k, v, scale)


def _kernel_merge(o_a, lse_a, o_b, lse_b):
    from . import lse_merge
    return lse_merge(o_a, lse_a, o_b, lse_b)


def _kernel_bwd(q, k, v, out, lse, dout, scale, dq, dk, dv, acc_dq, acc_dkdv):
    from . import attn_bwd
    return attn_bwd(q, k, v, out, lse, dout, scale, dq=dq, dk=dk, dv=dv, accumulate_dq=acc_dq,
                    accumulate_dkdv=acc_dkdv)


def shard_range(S: int, index: int, count: int):
    """Token range [start, stop) of shard `index` of `count` equal shards of S tokens."""
    if S % count:
        raise ValueError(f"{S} tokens do not split into {count} equal shards")
    n = S // count
    return index * n, (index + 1) * n


def ring_attention(q, k, v, group=None, scale=None, attn=None, merge=None):
    """Exact attention of this rank's queries over the keys of every rank in `group`.

    q [B, H, Sq_local, D]; k, v [B, H, Skv_local, D] this rank's key shard.
    Returns (out [B, H, Sq_local, D], lse [B, H, Sq_local]). Step s computes the
    partial attention over the shard of rank (r - s) mod R while the next
    shard arrives from rank r - 1 and the current one leaves for rank r + 1."""
    attn = attn or _kernel_attn
    merge = merge or _kernel_merge
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (r + 1) % R) if group is not None else (r + 1) % R
    prv = dist.get_global_rank(group, (r - 1) % R) if group is not None else (r - 1) % R
    cur_k, cur_v = k.contiguous(), v.contiguous()
    out = lse = None
    for step in range(R):
        reqs = []
        if step < R - 1:
            nk, nv = torch.empty_like(cur_k), torch.empty_like(cur_v)
            ops = [dist.P2POp(dist.isend, cur_k, nxt, group), dist.P2POp(dist.irecv, nk, prv, group),
                   dist.P2POp(dist.isend, cur_v, nxt, group), dist.P2POp(dist.irecv, nv, prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        o_s, l_s = attn(q, cur_k, cur_v, scale)
        out, lse = (o_s, l_s) if out is None else merge(out, lse, o_s, l_s)
        for req in reqs:
            req.wait()
        if step < R - 1:
            cur_k, cur_v = nk, nv
    return out, lse


def ring_attention_bwd(q, k, v, out, lse, dout, group=None, scale=None, bwd=None):
    """Gradients (dq, dk, dv) of ring_attention for this rank's q, k, v shards.

    out, lse: this rank's ring_attention result (the attention over every
    rank's keys); dout: its upstream gradient. Step s: the key shard of rank
    (r - s) mod R visits together with the dk, dv that the ranks before have
    accumulated for it; this rank adds its queries' contribution (the gradient
    kernel with the merged out and lse, accumulating into the visiting dk, dv)
    and its own dq gathers that shard's share. The key shards travel on while
    the step is computed; the accumulators follow once it is done, and a last
    hop returns each shard's dk, dv to its owner.

    bwd(q, k, v, out, lse, dout, scale, dq, dk, dv, acc_dq, acc_dkdv) -> (dq, dk, dv)
    computes (or accumulates, when acc_*) one step; by default the library's
    regen_attn_bwd."""
    bwd = bwd or _kernel_bwd
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (r + 1) % R) if group is not None else (r + 1) % R
    prv = dist.get_global_rank(group, (r - 1) % R) if group is not None else (r - 1) % R
    q, out, dout = q.contiguous(), out.contiguous(), dout.contiguous()
    cur_k, cur_v = k.contiguous(), v.contiguous()
    dq, cur_dk, cur_dv = torch.empty_like(q), torch.empty_like(cur_k), torch.empty_like(cur_v)
    for step in range(R):
        reqs = []
        if step < R - 1:
            nk, nv = torch.empty_like(cur_k), torch.empty_like(cur_v)
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, cur_k, nxt, group),
                                           dist.P2POp(dist.irecv, nk, prv, group),
                                           dist.P2POp(dist.isend, cur_v, nxt, group),
                                           dist.P2POp(dist.irecv, nv, prv, group)])
        dq, cur_dk, cur_dv = bwd(q, cur_k, cur_v, out, lse, dout, scale, dq, cur_dk, cur_dv, step > 0, step > 0)
        ndk, ndv = torch.empty_like(cur_dk), torch.empty_like(cur_dv)
        reqs += dist.batch_isend_irecv([dist.P2POp(dist.isend, cur_dk.contiguous(), nxt, group),
                                        dist.P2POp(dist.irecv, ndk, prv, group),
                                        dist.P2POp(dist.isend, cur_dv.contiguous(), nxt, group),
                                        dist.P2POp(dist.irecv, ndv, prv, group)])
        for req in reqs:
            req.wait()
        cur_dk, cur_dv = ndk, ndv
        if step < R - 1:
            cur_k, cur_v = nk, nv
    return dq, cur_dk, cur_dv


def seq_to_heads(x, group=None):
    """Ulysses all-to-all: [B, H, S_local, ...] (this rank's tokens, every head)
    -> [B, H/U, U*S_local, ...] (every token of the group, this rank's heads)."""
    U = dist.get_world_size(group)
    B, H = x.shape[:2]
    rest = x.shape[2:]
    if H % U:
        raise ValueError(f"{H} heads do not split over {U} ranks")
    send = x.reshape(B, U, H // U, *rest).movedim(1, 0).contiguous()        # [U][B][H/U][S_local]...
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)                          # recv[u]: rank u's tokens
    return recv.movedim(0, 2).reshape(B, H // U, U * rest[0], *rest[1:]).contiguous()


def heads_to_seq(x, group=None):
    """The inverse all-to-all: [B, H/U, S, ...] -> [B, H, S/U, ...]."""
    U = dist.get_world_size(group)
    B, Hl, S = x.shape[:3]
    rest = x.shape[3:]
    if S % U:
        raise ValueError(f"{S} tokens do not split over {U} ranks")
    send = x.reshape(B, Hl, U, S // U, *rest).movedim(2, 0).contiguous()   # [U][B][H/U][S/U]...: rank u's tokens
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)                          # recv[u]: rank u's heads
    return recv.movedim(0, 1).reshape(B, U * Hl, S // U, *rest).contiguous()


def usp_groups(ulysses: int, ring: int):
    """Process groups of unified sequence parallelism over ulysses * ring ranks:
    rank = ring_index * ulysses + ulysses_index. Returns (ulysses_group,
    ring_group) containing this rank. Every rank must call this (collective)."""
    world = dist.get_world_size()
    if ulysses * ring != world:
        raise ValueError(f"{ulysses} x {ring} != {world} ranks")
    rank = dist.get_rank()
    mine_u = mine_r = None
    for j in range(ring):
        g = dist.new_group([j * ulysses + u for u in range(ulysses)])
        if rank // ulysses == j:
            mine_u = g
    for u in range(ulysses):
        g = dist.new_group([j * ulysses + u for j in range(ring)])
        if rank % ulysses == u:
            mine_r = g
    return mine_u, mine_r


def usp_attention(q, k, v, ulysses_group, ring_group, scale=None, attn=None, merge=None):
    """Exact self-attention of a window whose tokens are sharded over ulysses x
    ring ranks: this rank holds tokens shard_range(S, rank, U*R) of every head
    (q, k, v [B, H, S/(U R), D], RoPE already applied at their positions).
    Returns (out [B, H, S/(U R), D], lse [B, H, S/(U R)]) for the same tokens."""
    qh, kh, vh = (seq_to_heads(t, ulysses_group) for t in (q, k, v))       # [B, H/U, S/R, D]
    out, lse = ring_attention(qh, kh, vh, ring_group, scale, attn, merge)
    return heads_to_seq(out, ulysses_group), heads_to_seq(lse, ulysses_group)


class _USPAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, ulysses_group, ring_group, scale, attn, merge, bwd):
        qh, kh, vh = (seq_to_heads(t.contiguous(), ulysses_group) for t in (q, k, v))
        oh, lh = ring_attention(qh, kh, vh, ring_group, scale, attn, merge)
        ctx.save_for_backward(qh, kh, vh, oh, lh)
        ctx.groups, ctx.scale, ctx.bwd = (ulysses_group, ring_group), scale, bwd
        return heads_to_seq(oh, ulysses_group)

    @staticmethod
    def backward(ctx, dout):
        qh, kh, vh, oh, lh = ctx.saved_tensors
        ug, rg_ = ctx.groups
        # the all-to-all is a permutation of the data over the ranks: its
        # adjoint is the inverse all-to-all
        doh = seq_to_heads(dout.contiguous(), ug)
        dqh, dkh, dvh = ring_attention_bwd(qh, kh, vh, oh, lh, doh, rg_, ctx.scale, ctx.bwd)
        return (heads_to_seq(dqh, ug), heads_to_seq(dkh, ug), heads_to_seq(dvh, ug),
                None, None, None, None, None, None)


def usp_attention_autograd(q, k, v, ulysses_group, ring_group, scale=None, attn=None, merge=None, bwd=None):
    """usp_attention as a differentiable function of this rank's q, k, v
    shards (RoPE already applied): the backward runs the Ulysses all-to-alls
    in reverse around ring_attention_bwd. Returns this rank's out shard."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    return _USPAttention.apply(q, k, v, ulysses_group, ring_group, float(scale), attn, merge, bwd)
