"""Run one kernel of the hot path a few times on a synthetic shape, for profilers.

    python -m dit_attention_b200.profile_case --kernel attn --heads 8 --seq 31200 --iters 2

No timing is done here (use bench.py); this only gives ncu a small, bounded
launch sequence of one kernel: --kernel attn (self-attention with the 77-frame
window's sequence length, or --kv for cross-attention), rope (3D RoPE on the
latent grid of that sequence length), merge (two-block LSE merge) or bwd (one
forward, then --iters gradient calls: prep, dK/dV and dQ launches each) or
fp8 (quantisation of Q, K, V once, then --iters FP8 attention calls).
"""
from __future__ import annotations

import argparse
import math

import numpy as np
import torch

import dit_attention_b200 as rg
from dit_attention_b200 import synth

GRIDS = {31200: (20, 30, 52), 10920: (7, 30, 52), 1024: (1, 32, 32)}


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--kernel", choices=["attn", "rope", "merge", "bwd", "fp8"], default="attn")
    p.add_argument("--heads", type=int, default=8)
    p.add_argument("--seq", type=int, default=31200)
    p.add_argument("--kv", type=int, default=0, help="key count (default: --seq)")
    p.add_argument("--dim", type=int, default=128)
    p.add_argument("--iters", type=int, default=2)
    a = p.parse_args()
    skv = a.kv or a.seq
    w = synth.Workload("profile", B=1, H=a.heads, D=a.dim, Sq=a.seq, Skv=skv, seed=7)
    q, k, v = synth.make_inputs(w)

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)

    dq, dk, dv = dev(q), dev(k), dev(v)
    rg.load()
    if a.kernel == "bwd":
        scale = 1.0 / math.sqrt(a.dim)
        out, lse = rg.attn_fwd(dq, dk, dv, scale)
        g = dev(synth.make_dout(w))
    if a.kernel == "fp8":
        quant = [rg.quant_e4m3(x) for x in (dq, dk, dv)]
    for _ in range(a.iters):
        if a.kernel == "fp8":
            rg.attn_fwd_fp8(*quant[0], *quant[1], *quant[2], 1.0 / math.sqrt(a.dim))
        elif a.kernel == "attn":
            rg.attn_fwd(dq, dk, dv, 1.0 / math.sqrt(a.dim))
        elif a.kernel == "bwd":
            rg.attn_bwd(dq, dk, dv, out, lse, g, scale)
        elif a.kernel == "rope":
            rg.rope3d_(dq, dk, GRIDS[a.seq])
        else:
            lse = torch.zeros((1, a.heads, a.seq), dtype=torch.float32, device="cuda")
            rg.lse_merge(dq, lse, dk[:, :, :a.seq], lse)
    torch.cuda.synchronize()
    rc, site = rg.regen_last_device_error()
    if rc != 0:
        raise SystemExit(f"device error {rc} at wait site {site}")


if __name__ == "__main__":
    main()
