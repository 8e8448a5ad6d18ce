"""GPU parity of the backward path (regen_attn_bwd, regen_rope3d_bwd) through
the C ABI against the fp64 oracle's gradients on the same seeded bf16 inputs.

The forward outputs (out, lse) the backward consumes come from the GPU's own
forward, as in training; the oracle never sees them -- it differentiates the
exact attention of q, k, v for the same dO. Gradient contract: see
util.check_grad. RoPE's gradient is compared bit for bit.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from util import bits_to_f64, check_grad, delta_bounds, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(7070)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rg.load()
    yield
    rc, site = rg.regen_last_device_error()
    assert rc == 0, f"a kernel recorded a device error: {rc} at wait site {site}"


def rand_bf16(shape, scale=1.0):
    return synth.f64_to_bf16_bits(RNG.normal(size=shape) * scale)


def gpu_fwd_bwd(q, k, v, g, scale, **kw):
    dq_, dk_, dv_, dg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    out, lse = rg.attn_fwd(dq_, dk_, dv_, scale)
    grads = rg.attn_bwd(dq_, dk_, dv_, out, lse, dg, scale, **kw)
    torch.cuda.synchronize()
    return tuple(to_bits(t) for t in grads)


def check_all(got, ref, label, inputs=None):
    """dq, dk, dv against the oracle; with inputs = (q, k, v, g, scale) the
    dq and dk allowances include the delta term (util.delta_bounds)."""
    extra = (0.0, 0.0, 0.0) if inputs is None else (*delta_bounds(*inputs), 0.0)
    return [check_grad(gt, r, f"{label} {n}", e) for gt, r, n, e in zip(got, ref, ("dq", "dk", "dv"), extra)]


# ------------------------------------------------------------- small ---

@pytest.mark.parametrize("B,H,Sq,Skv,D", [
    (1, 1, 128, 128, 128), (1, 2, 200, 300, 128), (2, 3, 77, 130, 64), (1, 1, 1, 1, 128),
    (1, 2, 257, 1, 64), (1, 1, 5, 700, 128), (1, 2, 384, 256, 64), (1, 1, 640, 515, 128),
])
def test_attn_bwd_small_shapes(B, H, Sq, Skv, D):
    q, k, v = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Skv, D)), rand_bf16((B, H, Skv, D))
    g = rand_bf16((B, H, Sq, D))
    scale = 1.0 / np.sqrt(D)
    got = gpu_fwd_bwd(q, k, v, g, scale)
    check_all(got, oracle.attention_bwd(q, k, v, g, scale), f"{B}x{H}x{Sq}x{Skv}x{D}", (q, k, v, g, scale))


@pytest.mark.parametrize("scale", [-0.09, 0.35])
def test_attn_bwd_scale_sign_and_size(scale):
    q, k, v, g = rand_bf16((1, 2, 300, 128)), rand_bf16((1, 2, 260, 128)), rand_bf16((1, 2, 260, 128)), \
        rand_bf16((1, 2, 300, 128))
    check_all(gpu_fwd_bwd(q, k, v, g, scale), oracle.attention_bwd(q, k, v, g, scale), f"scale {scale}",
              (q, k, v, g, scale))


def test_attn_bwd_zero_scale():
    # uniform P: dq = dk = 0 exactly, dv_j = mean_i dO_i
    q, k, v, g = rand_bf16((1, 1, 200, 64)), rand_bf16((1, 1, 150, 64)), rand_bf16((1, 1, 150, 64)), \
        rand_bf16((1, 1, 200, 64))
    dq, dk, dv = gpu_fwd_bwd(q, k, v, g, 0.0)
    assert not bits_to_f64(dq).any() and not bits_to_f64(dk).any()
    check_grad(dv, oracle.attention_bwd(q, k, v, g, 0.0)[2], "scale 0 dv")


def test_attn_bwd_spiky_logits():
    # softmax rows dominated by a few keys (Q x4, a few K rows x8): P near 0/1
    q = synth.f64_to_bf16_bits(synth.bf16_bits_to_f64(rand_bf16((1, 2, 260, 128))) * 4.0)
    k = rand_bf16((1, 2, 390, 128))
    kk = synth.bf16_bits_to_f64(k)
    kk[:, :, ::37] *= 8.0
    k = synth.f64_to_bf16_bits(kk)
    v, g = rand_bf16((1, 2, 390, 128)), rand_bf16((1, 2, 260, 128))
    scale = 1 / np.sqrt(128)
    d = check_all(gpu_fwd_bwd(q, k, v, g, scale), oracle.attention_bwd(q, k, v, g, scale), "spiky",
                  (q, k, v, g, scale))
    assert d[0]["max_err_over_rms"] > 0.02    # the case where the delta term is what binds


def test_attn_bwd_deterministic():
    q, k, v, g = rand_bf16((1, 4, 520, 128)), rand_bf16((1, 4, 700, 128)), rand_bf16((1, 4, 700, 128)), \
        rand_bf16((1, 4, 520, 128))
    a = gpu_fwd_bwd(q, k, v, g, 0.088)
    b = gpu_fwd_bwd(q, k, v, g, 0.088)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_attn_bwd_key_blocks_with_merged_stats():
    # keys in two blocks, forward per block + LSE merge; the backward per block
    # with the MERGED out/lse, dq accumulated, equals the gradient over all keys
    B, H, Sq, D = 1, 2, 333, 128
    s1, s2 = 270, 141
    q, g = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Sq, D))
    k, v = rand_bf16((B, H, s1 + s2, D)), rand_bf16((B, H, s1 + s2, D))
    scale = 1 / np.sqrt(D)
    tq, tg = to_dev(q), to_dev(g)
    ka, kb = to_dev(k[:, :, :s1]), to_dev(k[:, :, s1:])
    va, vb = to_dev(v[:, :, :s1]), to_dev(v[:, :, s1:])
    oa, la = rg.attn_fwd(tq, ka, va, scale)
    ob, lb = rg.attn_fwd(tq, kb, vb, scale)
    om, lm = rg.lse_merge(oa, la, ob, lb)
    dq, dka, dva = rg.attn_bwd(tq, ka, va, om, lm, tg, scale)
    _, dkb, dvb = rg.attn_bwd(tq, kb, vb, om, lm, tg, scale, dq=dq, accumulate_dq=True)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, scale)
    check_grad(to_bits(dq), rq, "merged dq (two accumulated shares)")
    check_grad(np.concatenate([to_bits(dka), to_bits(dkb)], axis=2), rk, "merged dk")
    check_grad(np.concatenate([to_bits(dva), to_bits(dvb)], axis=2), rv, "merged dv")


def test_attn_bwd_query_blocks_accumulate_dkdv():
    # queries in two blocks (as Ring attention's backward meets a key shard once
    # per rank): the second call adds its dk, dv into the first's, and the sums
    # equal the gradient over all queries; dq rows are independent per block
    B, H, Skv, D = 1, 2, 300, 128
    s1, s2 = 197, 230
    q, g = rand_bf16((B, H, s1 + s2, D)), rand_bf16((B, H, s1 + s2, D))
    k, v = rand_bf16((B, H, Skv, D)), rand_bf16((B, H, Skv, D))
    scale = 1 / np.sqrt(D)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    out, lse = rg.attn_fwd(tq, tk, tv, scale)
    c = lambda t, a, b: t[:, :, a:b].contiguous()  # noqa: E731
    dq1, dk, dv = rg.attn_bwd(c(tq, 0, s1), tk, tv, c(out, 0, s1), c(lse, 0, s1), c(tg, 0, s1), scale)
    dq2, _, _ = rg.attn_bwd(c(tq, s1, s1 + s2), tk, tv, c(out, s1, s1 + s2), c(lse, s1, s1 + s2),
                            c(tg, s1, s1 + s2), scale, dk=dk, dv=dv, accumulate_dkdv=True)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, scale)
    check_grad(np.concatenate([to_bits(dq1), to_bits(dq2)], axis=2), rq, "query-block dq")
    check_grad(to_bits(dk), rk, "dk accumulated over two query blocks")
    check_grad(to_bits(dv), rv, "dv accumulated over two query blocks")


def test_attn_bwd_empty_sides():
    t = lambda *s: torch.full(s, 3.0, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    q, out, g = t(1, 2, 0, 128), t(1, 2, 0, 128), t(1, 2, 0, 128)
    k, v = t(1, 2, 50, 128), t(1, 2, 50, 128)
    lse = torch.zeros((1, 2, 0), device="cuda")
    dq, dk, dv = rg.attn_bwd(q, k, v, out, lse, g, 0.1, dk=t(1, 2, 50, 128), dv=t(1, 2, 50, 128))
    torch.cuda.synchronize()
    assert float(dk.abs().max()) == 0.0 and float(dv.abs().max()) == 0.0     # no query: no gradient
    q, out, g = t(1, 2, 40, 128), t(1, 2, 40, 128), t(1, 2, 40, 128)
    k, v = t(1, 2, 0, 128), t(1, 2, 0, 128)
    lse = torch.zeros((1, 2, 40), device="cuda")
    dq, _, _ = rg.attn_bwd(q, k, v, out, lse, g, 0.1, dq=t(1, 2, 40, 128))
    torch.cuda.synchronize()
    assert float(dq.abs().max()) == 0.0
    dq = t(1, 2, 40, 128)
    rg.attn_bwd(q, k, v, out, lse, g, 0.1, dq=dq, accumulate_dq=True)
    torch.cuda.synchronize()
    assert float(dq.min()) == 3.0 and float(dq.max()) == 3.0                 # accumulating nothing
    q, out, g = t(1, 2, 0, 128), t(1, 2, 0, 128), t(1, 2, 0, 128)
    k, v = t(1, 2, 50, 128), t(1, 2, 50, 128)
    dk, dv = t(1, 2, 50, 128), t(1, 2, 50, 128)
    rg.attn_bwd(q, k, v, out, torch.zeros((1, 2, 0), device="cuda"), g, 0.1, dk=dk, dv=dv, accumulate_dkdv=True)
    torch.cuda.synchronize()
    assert float(torch.stack([dk, dv]).min()) == 3.0 and float(torch.stack([dk, dv]).max()) == 3.0


def test_attn_bwd_workspace_errors():
    q = torch.zeros((1, 1, 300, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 300), device="cuda")
    small = torch.empty(rg.regen_attn_bwd_workspace_bytes(1, 1, 300, 128) - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(rg.RegenError) as e:
        rg.attn_bwd(q, q.clone(), q.clone(), q.clone(), lse, q.clone(), 0.1, workspace=small)
    assert e.value.status == -1


# -------------------------------------------------------------- RoPE ---

@pytest.mark.parametrize("B,H,grid,D", [(1, 2, (3, 5, 7), 128), (2, 3, (2, 4, 6), 64), (1, 3, (7, 30, 52), 128)])
def test_rope3d_bwd_bit_exact(B, H, grid, D):
    S = grid[0] * grid[1] * grid[2]
    gq, gk = rand_bf16((B, H, S, D)), rand_bf16((B, H, S, D))
    tq, tk = to_dev(gq), to_dev(gk)
    rg.rope3d_bwd_(tq, tk, grid, 10000.0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_bits(tq), oracle.rope3d_bwd(gq, grid, 10000.0))
    np.testing.assert_array_equal(to_bits(tk), oracle.rope3d_bwd(gk, grid, 10000.0))


def test_rope_attention_chain_gradient():
    # q, k -> RoPE -> attention -> dq, dk through the attention's and the
    # RoPE's backward, against the oracle's chain rule R^T (dL/d(Rq))
    B, H, grid, D = 1, 2, (3, 6, 11), 128
    S = grid[0] * grid[1] * grid[2]
    q, k, v, g = (rand_bf16((B, H, S, D)) for _ in range(4))
    scale = 1 / np.sqrt(D)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    rg.rope3d_(tq, tk, grid)
    out, lse = rg.attn_fwd(tq, tk, tv, scale)
    dq, dk, dv = rg.attn_bwd(tq, tk, tv, out, lse, tg, scale)
    rg.rope3d_bwd_(dq, dk, grid)
    torch.cuda.synchronize()
    qr, kr = oracle.rope3d(q, grid), oracle.rope3d(k, grid)
    rq, rk, rv = oracle.attention_bwd(qr, kr, v, g, scale)
    check_grad(to_bits(dq), oracle.rope3d_bwd(rq, grid), "chain dq")
    check_grad(to_bits(dk), oracle.rope3d_bwd(rk, grid), "chain dk")
    check_grad(to_bits(dv), rv, "chain dv")


# ---------------------------------------------------- named workloads ---

def _sample(n, count, seed):
    r = np.random.default_rng(seed)
    fixed = {0, 1, 127, 128, n - 1, (n - 1) // 128 * 128}
    return np.array(sorted(fixed | set(r.choice(n, size=min(count, n), replace=False).tolist())), dtype=np.int64)


def _workload_bwd(name, heads, nq_rows=24, nk_rows=24, delta_term=False):
    """The whole workload's backward on the GPU (after its RoPE and forward);
    the given heads compared on sampled dq rows and dk/dv rows (the oracle
    computes every query row's statistics of those heads), and every head
    checked by two identities that hold at any size."""
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_inputs(w)
    g = synth.make_dout(w)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    if w.rope:
        rg.rope3d_(tq, tk, w.grid, w.theta)
    out, lse = rg.attn_fwd(tq, tk, tv, w.scale)
    dq, dk, dv = rg.attn_bwd(tq, tk, tv, out, lse, tg, w.scale)
    torch.cuda.synchronize()
    BH = w.B * w.H
    gq = to_bits(dq).reshape(BH, w.Sq, w.D)
    gk = to_bits(dk).reshape(BH, w.Skv, w.D)
    gv = to_bits(dv).reshape(BH, w.Skv, w.D)
    # identities of every head: sum_j dv_j = sum_i dO_i (rows of P sum to 1),
    # sum_j dk_j = 0 (shifting every key leaves the softmax unchanged)
    # (bounds: 4u of every summand, u = 2^-8 the bf16 unit roundoff: a few roundings)
    fv = bits_to_f64(gv)
    sg = bits_to_f64(g.reshape(BH, w.Sq, w.D)).sum(axis=1)
    assert np.all(np.abs(fv.sum(axis=1) - sg) <= 4 * 2.0 ** -8 * np.abs(fv).sum(axis=1) + 1e-3)
    fk = bits_to_f64(gk)
    assert np.all(np.abs(fk.sum(axis=1)) <= 4 * 2.0 ** -8 * np.abs(fk).sum(axis=1) + 1e-6)
    qrows, krows = _sample(w.Sq, nq_rows, 1), _sample(w.Skv, nk_rows, 2)
    qh = q.reshape(BH, w.Sq, w.D)[heads]
    kh = k.reshape(BH, w.Skv, w.D)[heads]
    if w.rope:
        qh, kh = oracle.rope3d(qh, w.grid, w.theta), oracle.rope3d(kh, w.grid, w.theta)
    vh, gh = v.reshape(BH, w.Skv, w.D)[heads], g.reshape(BH, w.Sq, w.D)[heads]
    rq, rk, rv = oracle.attention_bwd_rows(qh, kh, vh, gh, w.scale, qrows, krows)
    bq, bk = delta_bounds(qh, kh, vh, gh, w.scale, qrows, krows) if delta_term else (0.0, 0.0)
    return [check_grad(gq[heads][:, qrows], rq, f"{name} dq", bq),
            check_grad(gk[heads][:, krows], rk, f"{name} dk", bk),
            check_grad(gv[heads][:, krows], rv, f"{name} dv")]


def test_workload_bwd_tiny_full():
    w = synth.WORKLOADS["tiny_s1024"]
    q, k, v = synth.make_inputs(w)
    g = synth.make_dout(w)
    check_all(gpu_fwd_bwd(q, k, v, g, w.scale), oracle.attention_bwd(q, k, v, g, w.scale), "tiny",
              (q, k, v, g, w.scale))


def test_workload_bwd_25_frame_window_sampled():
    _workload_bwd("win25_s10920", heads=[0, 11])


def test_workload_bwd_77_frame_window_sampled():
    _workload_bwd("win77_s31200", heads=[23])


def test_workload_bwd_cross_attention_sampled():
    _workload_bwd("cross_s31200_kv2072", heads=[0, 39])


def test_workload_bwd_softmax_stress_sampled():
    # nearly one-hot softmax rows: the delta term of the allowance binds here
    _workload_bwd("stress_s10920", heads=[30], delta_term=True)
