"""Sequence parallelism (dit_attention_b200.usp): Ring and Ulysses exchanges on
2 and 4 ranks.

CPU tests: gloo ranks run the exchange logic with the oracle as the per-rank
attention and merge (fp64), and every rank's result must equal the oracle's
attention over the whole window -- the exactness the sharding promises. The GPU
test runs two ranks on one GPU with the library's kernels as the per-rank
compute; the shards travel through gloo (host memory), since two ranks cannot
share one GPU under NCCL.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from dit_attention_b200 import synth, usp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_attn(q, k, v, scale):
    out, lse = oracle.attention(q.numpy(), k.numpy(), v.numpy(), scale)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _oracle_merge(oa, la, ob, lb):
    out, lse = oracle.lse_merge(oa.numpy(), la.numpy(), ob.numpy(), lb.numpy())
    return torch.from_numpy(out), torch.from_numpy(lse)


def _window(B=1, H=4, S=96, D=16, seed=5):
    rng = np.random.default_rng(seed)
    return [rng.normal(size=(B, H, S, D)) * f for f in (1.5, 1.5, 1.0)]


def _run(world, fn, *args):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out, fn, args), nprocs=world, start_method="spawn", join=True)
        return dict(out)


def _worker(rank, world, port, out, fn, args):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = fn(rank, world, *args)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _ring_case(rank, world, S):
    q, k, v = _window(S=S)
    scale = 0.25
    a, b = usp.shard_range(S, rank, world)
    o, l = usp.ring_attention(torch.from_numpy(q[:, :, a:b].copy()), torch.from_numpy(k[:, :, a:b].copy()),
                              torch.from_numpy(v[:, :, a:b].copy()), None, scale, _oracle_attn, _oracle_merge)
    ref, rl = oracle.attention(q, k, v, scale)
    return float(np.abs(o.numpy() - ref[:, :, a:b]).max()), float(np.abs(l.numpy() - rl[:, :, a:b]).max())


@pytest.mark.parametrize("world", [2, 4])
def test_ring_attention_is_exact(world):
    res = _run(world, _ring_case, 96)
    assert sorted(res) == list(range(world))
    for r, (eo, el) in res.items():
        assert eo < 1e-12 and el < 1e-12, (r, eo, el)


def _ulysses_case(rank, world):
    x = _window(H=4, S=64)[0]
    a, b = usp.shard_range(64, rank, world)
    mine = torch.from_numpy(x[:, :, a:b].copy())
    heads = usp.seq_to_heads(mine, None)
    hq = 4 // world
    # this rank's heads, every token
    ok_fwd = np.array_equal(heads.numpy(), x[:, rank * hq:(rank + 1) * hq])
    back = usp.heads_to_seq(heads, None)
    lse_like = torch.from_numpy(x[..., 0][:, :, a:b].copy())           # [B, H, S_local]: 3-dim tensors too
    lse_back = usp.heads_to_seq(usp.seq_to_heads(lse_like, None), None)
    return ok_fwd, bool(torch.equal(back, mine)), bool(torch.equal(lse_back, lse_like))


def test_ulysses_all_to_all_round_trip():
    res = _run(2, _ulysses_case)
    for r, (f, b, lse_ok) in res.items():
        assert f and b and lse_ok, r


def _usp_case(rank, world, U, R):
    ug, rg_ = usp.usp_groups(U, R)
    q, k, v = _window(H=4, S=96)
    scale = 0.25
    a, b = usp.shard_range(96, rank, world)
    args = [torch.from_numpy(t[:, :, a:b].copy()) for t in (q, k, v)]
    o, l = usp.usp_attention(*args, ug, rg_, scale, _oracle_attn, _oracle_merge)
    ref, rl = oracle.attention(q, k, v, scale)
    return float(np.abs(o.numpy() - ref[:, :, a:b]).max()), float(np.abs(l.numpy() - rl[:, :, a:b]).max())


def test_unified_sequence_parallel_ulysses2_ring2():
    # the pages' layout scaled down: 2 (Ulysses) x 2 (Ring) ranks
    res = _run(4, _usp_case, 2, 2)
    for r, (eo, el) in res.items():
        assert eo < 1e-12 and el < 1e-12, (r, eo, el)


def _oracle_bwd(q, k, v, out, lse, dout, scale, dq, dk, dv, acc_dq, acc_dkdv):
    sq, sk, sv = (torch.from_numpy(x) for x in oracle.attention_bwd_block(
        q.numpy(), k.numpy(), v.numpy(), out.numpy(), lse.numpy(), dout.numpy(), scale))
    return (dq + sq if acc_dq else sq), (dk + sk if acc_dkdv else sk), (dv + sv if acc_dkdv else sv)


def _dout(B=1, H=4, S=96, D=16, seed=6):
    return np.random.default_rng(seed).normal(size=(B, H, S, D))


def _rel(a, b):
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def _ring_bwd_case(rank, world, S):
    q, k, v = _window(S=S)
    g = _dout(S=S)
    scale = 0.25
    a, b = usp.shard_range(S, rank, world)
    sl = lambda x: torch.from_numpy(x[:, :, a:b].copy())  # noqa: E731
    o, l = usp.ring_attention(sl(q), sl(k), sl(v), None, scale, _oracle_attn, _oracle_merge)
    dq, dk, dv = usp.ring_attention_bwd(sl(q), sl(k), sl(v), o, l, sl(g), None, scale, _oracle_bwd)
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, scale)
    return (_rel(dq.numpy(), rq[:, :, a:b]), _rel(dk.numpy(), rk[:, :, a:b]), _rel(dv.numpy(), rv[:, :, a:b]))


@pytest.mark.parametrize("world", [2, 4])
def test_ring_attention_backward_is_exact(world):
    # every rank's dq, dk, dv of its own shards equal the oracle's gradient of
    # the whole window: the key shards and their accumulators went all the way round
    res = _run(world, _ring_bwd_case, 96)
    assert sorted(res) == list(range(world))
    for r, errs in res.items():
        assert max(errs) < 1e-10, (r, errs)


def _usp_autograd_case(rank, world, U, R):
    ug, rg_ = usp.usp_groups(U, R)
    q, k, v = _window(H=4, S=96)
    g = _dout(H=4, S=96)
    scale = 0.25
    a, b = usp.shard_range(96, rank, world)
    leaf = lambda x: torch.from_numpy(x[:, :, a:b].copy()).requires_grad_(True)  # noqa: E731
    tq, tk, tv = leaf(q), leaf(k), leaf(v)
    out = usp.usp_attention_autograd(tq, tk, tv, ug, rg_, scale, _oracle_attn, _oracle_merge, _oracle_bwd)
    out.backward(torch.from_numpy(g[:, :, a:b].copy()))
    ref, _ = oracle.attention(q, k, v, scale)
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, scale)
    return (_rel(out.detach().numpy(), ref[:, :, a:b]), _rel(tq.grad.numpy(), rq[:, :, a:b]),
            _rel(tk.grad.numpy(), rk[:, :, a:b]), _rel(tv.grad.numpy(), rv[:, :, a:b]))


def test_unified_sequence_parallel_autograd_ulysses2_ring2():
    # forward and backward through the all-to-alls and the ring on 2 x 2 ranks
    res = _run(4, _usp_autograd_case, 2, 2)
    for r, errs in res.items():
        assert max(errs) < 1e-10, (r, errs)


def test_shard_range():
    assert usp.shard_range(31200, 3, 8) == (11700, 15600)
    with pytest.raises(ValueError):
        usp.shard_range(10, 1, 3)


# ------------------------------------------------- with the GPU kernels ---

def _gpu_ring_case(rank, world):
    import dit_attention_b200 as rg
    torch.cuda.set_device(0)
    w = synth.Workload("usp", B=1, H=4, D=128, Sq=1040, Skv=1040, seed=9, grid=(2, 20, 26), rope=True, rmsnorm=True)
    q, k, v = synth.make_inputs(w)
    a, b = usp.shard_range(w.Sq, rank, world)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    tq, tk, tv = dev(q[:, :, a:b]), dev(k[:, :, a:b]), dev(v[:, :, a:b])
    T, Hh, Ww = w.grid
    rg.regen_rope3d_shard(tq, tk, T, Hh, Ww, w.theta, w.B, w.H, w.D, a, b - a, 0)   # RoPE at global positions

    # per-rank compute in the library's kernels; the shards travel as host tensors
    def attn(qh, kh, vh, scale):
        o, l = rg.attn_fwd(qh.cuda(), kh.cuda(), vh.cuda(), scale)
        return o.cpu(), l.cpu()

    def merge(oa, la, ob, lb):
        o, l = rg.lse_merge(oa.cuda(), la.cuda(), ob.cuda(), lb.cuda())
        return o.cpu(), l.cpu()

    o, l = usp.ring_attention(tq.cpu(), tk.cpu(), tv.cpu(), None, w.scale, attn, merge)
    torch.cuda.synchronize()
    return (o.contiguous().view(torch.int16).numpy().view(np.uint16), l.numpy(), a, b,
            tq.cpu().contiguous().view(torch.int16).numpy().view(np.uint16),
            tk.cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


@pytest.mark.gpu
def test_ring_attention_with_kernels_two_ranks_one_gpu():
    from util import check_attention
    assert torch.cuda.is_available()
    res = _run(2, _gpu_ring_case)
    w = synth.Workload("usp", B=1, H=4, D=128, Sq=1040, Skv=1040, seed=9, grid=(2, 20, 26), rope=True, rmsnorm=True)
    q, k, v = synth.make_inputs(w)
    qr, kr = oracle.rope3d(q, w.grid, w.theta), oracle.rope3d(k, w.grid, w.theta)
    ref, rl = oracle.attention(qr, kr, v, w.scale)
    for r, (o, l, a, b, gq, gk) in res.items():
        # the sharded RoPE equals the whole-grid one on these rows, bit for bit
        np.testing.assert_array_equal(gq, qr[:, :, a:b])
        np.testing.assert_array_equal(gk, kr[:, :, a:b])
        check_attention(o.reshape(-1, 128), l.reshape(-1), ref[:, :, a:b].reshape(-1, 128), rl[:, :, a:b].reshape(-1),
                        f"ring rank {r}")


def _gpu_ring_bwd_case(rank, world):
    import dit_attention_b200 as rg
    torch.cuda.set_device(0)
    w = synth.Workload("usp", B=1, H=4, D=128, Sq=1040, Skv=1040, seed=9, grid=(2, 20, 26), rope=True, rmsnorm=True)
    q, k, v = synth.make_inputs(w)
    g = synth.make_dout(w)
    a, b = usp.shard_range(w.Sq, rank, world)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    tq, tk, tv, tg = dev(q[:, :, a:b]), dev(k[:, :, a:b]), dev(v[:, :, a:b]), dev(g[:, :, a:b])
    T, Hh, Ww = w.grid
    rg.regen_rope3d_shard(tq, tk, T, Hh, Ww, w.theta, w.B, w.H, w.D, a, b - a, 0)

    # per-rank compute in the library's kernels; the shards travel as host tensors
    def attn(qh, kh, vh, scale):
        o, l = rg.attn_fwd(qh.cuda(), kh.cuda(), vh.cuda(), scale)
        return o.cpu(), l.cpu()

    def merge(oa, la, ob, lb):
        o, l = rg.lse_merge(oa.cuda(), la.cuda(), ob.cuda(), lb.cuda())
        return o.cpu(), l.cpu()

    def bwd(q_, k_, v_, out, lse, dout, scale, dq, dk, dv, acc_dq, acc_dkdv):
        c = lambda t: t.cuda()  # noqa: E731
        r = rg.attn_bwd(c(q_), c(k_), c(v_), c(out), c(lse), c(dout), scale, dq=c(dq), dk=c(dk), dv=c(dv),
                        accumulate_dq=acc_dq, accumulate_dkdv=acc_dkdv)
        return tuple(t.cpu() for t in r)

    o, l = usp.ring_attention(tq.cpu(), tk.cpu(), tv.cpu(), None, w.scale, attn, merge)
    dq, dk, dv = usp.ring_attention_bwd(tq.cpu(), tk.cpu(), tv.cpu(), o, l, tg.cpu(), None, w.scale, bwd)
    torch.cuda.synchronize()
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    return bits(dq), bits(dk), bits(dv), a, b


@pytest.mark.gpu
def test_ring_attention_backward_with_kernels_two_ranks_one_gpu():
    from util import check_grad
    assert torch.cuda.is_available()
    res = _run(2, _gpu_ring_bwd_case)
    w = synth.Workload("usp", B=1, H=4, D=128, Sq=1040, Skv=1040, seed=9, grid=(2, 20, 26), rope=True, rmsnorm=True)
    q, k, v = synth.make_inputs(w)
    g = synth.make_dout(w)
    qr, kr = oracle.rope3d(q, w.grid, w.theta), oracle.rope3d(k, w.grid, w.theta)
    rq, rk, rv = oracle.attention_bwd(qr, kr, v, g, w.scale)
    for r, (dq, dk, dv, a, b) in res.items():
        # gradients with respect to the rotated shards (RoPE's own gradient is pinned elsewhere)
        check_grad(dq, rq[:, :, a:b], f"ring dq rank {r}")
        check_grad(dk, rk[:, :, a:b], f"ring dk rank {r}")
        check_grad(dv, rv[:, :, a:b], f"ring dv rank {r}")


def _gpu_usp_case(rank, world, U, R):
    # Unified sequence parallelism as the pages lay it out, scaled down to
    # Ulysses 2 x Ring 2 ranks on one GPU: the RoPE of each rank's token shard
    # at its global positions, the Ulysses all-to-alls, the ring with its LSE
    # merges, and the backward through all of them, with the library's kernels
    # as every rank's compute (regen_rope3d_shard, regen_attn_fwd,
    # regen_lse_merge, regen_attn_bwd, and the RoPE's gradient); the shards and
    # partial results travel as host tensors over gloo.
    import dit_attention_b200 as rg
    torch.cuda.set_device(0)
    ug, rg_ = usp.usp_groups(U, R)
    w = synth.Workload("usp", B=1, H=4, D=128, Sq=1040, Skv=1040, seed=9, grid=(2, 20, 26), rope=True, rmsnorm=True)
    q, k, v = synth.make_inputs(w)
    g = synth.make_dout(w)
    a, b = usp.shard_range(w.Sq, rank, world)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    tq, tk = dev(q[:, :, a:b]), dev(k[:, :, a:b])
    T, Hh, Ww = w.grid
    rg.regen_rope3d_shard(tq, tk, T, Hh, Ww, w.theta, w.B, w.H, w.D, a, b - a, 0)   # RoPE at global positions

    def attn(qh, kh, vh, scale):
        o, l = rg.attn_fwd(qh.detach().cuda().contiguous(), kh.detach().cuda().contiguous(),
                           vh.detach().cuda().contiguous(), scale)
        return o.cpu(), l.cpu()

    def merge(oa, la, ob, lb):
        o, l = rg.lse_merge(oa.cuda(), la.cuda(), ob.cuda(), lb.cuda())
        return o.cpu(), l.cpu()

    def bwd(q_, k_, v_, out, lse, dout, scale, dq, dk, dv, acc_dq, acc_dkdv):
        c = lambda t: t.detach().cuda().contiguous()  # noqa: E731
        r = rg.attn_bwd(c(q_), c(k_), c(v_), c(out), c(lse), c(dout), scale, dq=c(dq), dk=c(dk), dv=c(dv),
                        accumulate_dq=acc_dq, accumulate_dkdv=acc_dkdv)
        return tuple(t.cpu() for t in r)

    leaf = lambda t: t.cpu().requires_grad_(True)  # noqa: E731
    lq, lk = leaf(tq), leaf(tk)
    lv = torch.from_numpy(np.ascontiguousarray(v[:, :, a:b]).view(np.int16)).view(torch.bfloat16).requires_grad_(True)
    out = usp.usp_attention_autograd(lq, lk, lv, ug, rg_, w.scale, attn, merge, bwd)
    gout = torch.from_numpy(np.ascontiguousarray(g[:, :, a:b]).view(np.int16)).view(torch.bfloat16)
    out.backward(gout)
    # the RoPE's gradient of this rank's shard, at its global positions
    gq, gk = lq.grad.cuda().contiguous(), lk.grad.cuda().contiguous()
    rg.regen_rope3d_shard(gq, gk, T, Hh, Ww, w.theta, w.B, w.H, w.D, a, b - a, 1)
    torch.cuda.synchronize()
    bits = lambda t: t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    return (bits(out), bits(lq.grad), bits(lk.grad), bits(lv.grad), bits(gq), bits(gk), bits(tq), bits(tk), a, b)


@pytest.mark.gpu
def test_usp_ulysses2_ring2_forward_and_backward_with_kernels_four_ranks_one_gpu():
    from util import check_attention, check_grad
    assert torch.cuda.is_available()
    res = _run(4, _gpu_usp_case, 2, 2)
    assert sorted(res) == [0, 1, 2, 3]
    w = synth.Workload("usp", B=1, H=4, D=128, Sq=1040, Skv=1040, seed=9, grid=(2, 20, 26), rope=True, rmsnorm=True)
    q, k, v = synth.make_inputs(w)
    g = synth.make_dout(w)
    qr, kr = oracle.rope3d(q, w.grid, w.theta), oracle.rope3d(k, w.grid, w.theta)
    ref, rl = oracle.attention(qr, kr, v, w.scale)
    rq, rk, rv = oracle.attention_bwd(qr, kr, v, g, w.scale)
    for r, (o, dq, dk, dv, gq, gk, tq, tk, a, b) in res.items():
        np.testing.assert_array_equal(tq, qr[:, :, a:b])            # sharded RoPE == whole-grid RoPE
        np.testing.assert_array_equal(tk, kr[:, :, a:b])
        check_attention(o.reshape(-1, 128), None, ref[:, :, a:b].reshape(-1, 128), rl[:, :, a:b].reshape(-1),
                        f"usp out rank {r}")
        # gradients with respect to the rotated shards, against the oracle's chain rule over the whole window
        check_grad(dq, rq[:, :, a:b], f"usp dq rank {r}")
        check_grad(dk, rk[:, :, a:b], f"usp dk rank {r}")
        check_grad(dv, rv[:, :, a:b], f"usp dv rank {r}")
        # the RoPE's gradient of the shard at its global positions, bit for bit
        full_q = np.zeros_like(q)
        full_k = np.zeros_like(k)
        full_q[:, :, a:b], full_k[:, :, a:b] = dq, dk
        np.testing.assert_array_equal(gq, oracle.rope3d_bwd(full_q, w.grid, w.theta)[:, :, a:b], f"rank {r}")
        np.testing.assert_array_equal(gk, oracle.rope3d_bwd(full_k, w.grid, w.theta)[:, :, a:b], f"rank {r}")
