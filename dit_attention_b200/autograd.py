"""torch.autograd glue over the library's forward and gradient kernels.

Argument marshalling only: the forward runs regen_rope3d, regen_attn_fwd and
regen_attn_fwd_kv2, the backward runs regen_attn_bwd, regen_attn_bwd_kv2 and
regen_rope3d_bwd; no arithmetic happens here. Tensors are bf16 [B, H, S, D] on
the GPU.

    dit_attention(q, k, v, grid=None, theta=10000.0, scale=None) -> out
        self-attention of q over (k, v); with a latent grid (T, Hh, Ww), q and
        k are first rotated by the 3D RoPE (on copies: the inputs are left as
        they are). Gradients flow to q, k and v, back through the RoPE.

    dit_cross_attention(q, (k_a, v_a), (k_b, v_b), scale=None) -> out
        one softmax over the keys of two separately held sources (the DiT's
        reference-frame latents and conditioning tokens, ReGenVC blog page,
        "Methodology -- deep read"), in one launch over both (regen_attn_fwd_kv2).
        Its gradient (regen_attn_bwd_kv2) takes each source's P as its slice
        of the joint softmax, from the joint output and LSE, and accumulates
        dq over both sources' keys.
"""
from __future__ import annotations

import math

import torch

from . import attn_bwd, attn_bwd_kv2, attn_fwd, attn_fwd_kv2, rope3d_, rope3d_bwd_


def _scale(scale, q):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


class _SelfAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, grid, theta, scale):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        if grid is not None:          # the RoPE works in place: rotate copies
            q, k = q.clone(), k.clone()
            rope3d_(q, k, grid, theta)
        out, lse = attn_fwd(q, k, v, scale)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.grid, ctx.theta, ctx.scale = grid, theta, scale
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = attn_bwd(q, k, v, out, lse, dout.contiguous(), ctx.scale)
        if ctx.grid is not None:
            rope3d_bwd_(dq, dk, ctx.grid, ctx.theta)
        return dq, dk, dv, None, None, None


class _TwoSourceAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k_a, v_a, k_b, v_b, scale):
        q, k_a, v_a, k_b, v_b = (t.contiguous() for t in (q, k_a, v_a, k_b, v_b))
        out, lse = attn_fwd_kv2(q, k_a, v_a, k_b, v_b, scale)
        ctx.save_for_backward(q, k_a, v_a, k_b, v_b, out, lse)
        ctx.scale = scale
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k_a, v_a, k_b, v_b, out, lse = ctx.saved_tensors
        dq, dk_a, dv_a, dk_b, dv_b = attn_bwd_kv2(q, k_a, v_a, k_b, v_b, out, lse, dout.contiguous(), ctx.scale)
        return dq, dk_a, dv_a, dk_b, dv_b, None


def dit_attention(q, k, v, grid=None, theta=10000.0, scale=None):
    """Self-attention (with the 3D RoPE on q, k when `grid` is given), differentiable."""
    return _SelfAttention.apply(q, k, v, tuple(grid) if grid is not None else None, float(theta), _scale(scale, q))


def dit_cross_attention(q, source_a, source_b, scale=None):
    """Attention of q over the keys of two sources, one softmax, differentiable."""
    (k_a, v_a), (k_b, v_b) = source_a, source_b
    return _TwoSourceAttention.apply(q, k_a, v_a, k_b, v_b, _scale(scale, q))
