"""GPU parity of the two-source gradient (regen_attn_bwd_kv2) through the C ABI.

The cross-attention's softmax runs over the reference-frame and the
conditioning keys together (mlsanity.com abstract; blog page, "Methodology --
deep read"), so its gradient is the attention gradient over the two key sets
concatenated, each key's dk, dv returned in its own source's buffer. The
oracle is the fp64 gradient over the concatenation; the contract is
util.check_grad's, as for regen_attn_bwd. The forward's out and lse come from
the GPU's two-source forward, as in training; the oracle never sees them.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from util import bits_to_f64, check_grad, delta_bounds, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(20261204)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rg.load()
    yield
    rc, site = rg.regen_last_device_error()
    assert rc == 0, f"a kernel recorded a device error: {rc} at wait site {site}"


def rand_bf16(shape, scale=1.0):
    return synth.f64_to_bf16_bits(RNG.normal(size=shape) * scale)


def gpu_kv2(q, ka, va, kb, vb, g, scale, **kw):
    """Two-source forward, then its gradient; (dq, dk_a, dv_a, dk_b, dv_b) as bf16 bits."""
    tq, tka, tva, tkb, tvb, tg = (to_dev(x) for x in (q, ka, va, kb, vb, g))
    out, lse = rg.attn_fwd_kv2(tq, tka, tva, tkb, tvb, scale)
    grads = rg.attn_bwd_kv2(tq, tka, tva, tkb, tvb, out, lse, tg, scale, **kw)
    torch.cuda.synchronize()
    return tuple(to_bits(t) for t in grads), (tq, tka, tva, tkb, tvb, out, lse, tg)


def check_against_oracle(grads, q, ka, va, kb, vb, g, scale, label, dq0=None):
    kc, vc = np.concatenate([ka, kb], axis=2), np.concatenate([va, vb], axis=2)
    rq, rk, rv = oracle.attention_bwd(q, kc, vc, g, scale)
    bq, bk = delta_bounds(q, kc, vc, g, scale)
    dq, dka, dva, dkb, dvb = grads
    if dq0 is not None:   # accumulated into dq0, then rounded once to bf16
        rq = rq + bits_to_f64(dq0)
        bq = bq + 2.0 ** -8 * np.abs(rq)
    check_grad(dq, rq, f"{label} dq", bq)
    check_grad(np.concatenate([bits_to_f64(dka), bits_to_f64(dkb)], axis=2), rk, f"{label} dk", bk)
    check_grad(np.concatenate([bits_to_f64(dva), bits_to_f64(dvb)], axis=2), rv, f"{label} dv")


@pytest.mark.parametrize("B,H,Sq,Skv_a,Skv_b,D", [
    (1, 1, 128, 1, 1, 128), (1, 2, 200, 24, 512, 128), (2, 1, 300, 127, 129, 64), (1, 2, 257, 130, 300, 128),
    (1, 1, 1, 300, 40, 128), (1, 3, 513, 5, 700, 64), (1, 1, 256, 256, 128, 128), (1, 1, 640, 515, 77, 128),
])
def test_bwd_kv2_against_oracle_over_concatenated_keys(B, H, Sq, Skv_a, Skv_b, D):
    q, g = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Sq, D))
    ka, va = rand_bf16((B, H, Skv_a, D)), rand_bf16((B, H, Skv_a, D))
    kb, vb = rand_bf16((B, H, Skv_b, D)), rand_bf16((B, H, Skv_b, D))
    scale = 1.0 / np.sqrt(D)
    grads, _ = gpu_kv2(q, ka, va, kb, vb, g, scale)
    check_against_oracle(grads, q, ka, va, kb, vb, g, scale, f"kv2 bwd {Skv_a}+{Skv_b}")


def test_bwd_kv2_negative_scale_and_spiky_keys():
    B, H, Sq, D = 1, 2, 300, 128
    q, g = rand_bf16((B, H, Sq, D), 2.0), rand_bf16((B, H, Sq, D))
    ka, va = rand_bf16((B, H, 150, D)), rand_bf16((B, H, 150, D))
    kb, vb = rand_bf16((B, H, 90, D)), rand_bf16((B, H, 90, D))
    kb[:, :, ::17] = synth.f64_to_bf16_bits(synth.bf16_bits_to_f64(kb[:, :, ::17]) * 6.0)   # spikes in source b
    for scale in (-0.09, 0.09):
        grads, _ = gpu_kv2(q, ka, va, kb, vb, g, scale)
        check_against_oracle(grads, q, ka, va, kb, vb, g, scale, f"kv2 bwd scale {scale}")


def test_bwd_kv2_dk_dv_equal_the_per_source_gradients_bit_for_bit():
    # each key tile's dk, dv depend only on that tile and the joint softmax's
    # per-row statistics, so they equal regen_attn_bwd's for one source given
    # the joint out and lse
    B, H, Sq, D = 1, 2, 390, 128
    q, g = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Sq, D))
    ka, va = rand_bf16((B, H, 1560 // 8, D)), rand_bf16((B, H, 1560 // 8, D))
    kb, vb = rand_bf16((B, H, 64 + 3, D)), rand_bf16((B, H, 64 + 3, D))
    scale = 1.0 / np.sqrt(D)
    grads, (tq, tka, tva, tkb, tvb, out, lse, tg) = gpu_kv2(q, ka, va, kb, vb, g, scale)
    _, dka, dva = rg.attn_bwd(tq, tka, tva, out, lse, tg, scale)
    _, dkb, dvb = rg.attn_bwd(tq, tkb, tvb, out, lse, tg, scale)
    torch.cuda.synchronize()
    for got, want, name in zip(grads[1:], (dka, dva, dkb, dvb), ("dk_a", "dv_a", "dk_b", "dv_b")):
        np.testing.assert_array_equal(got, to_bits(want), err_msg=name)


def test_bwd_kv2_accumulates_dq():
    B, H, Sq, D = 1, 2, 260, 128
    q, g = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Sq, D))
    ka, va = rand_bf16((B, H, 200, D)), rand_bf16((B, H, 200, D))
    kb, vb = rand_bf16((B, H, 70, D)), rand_bf16((B, H, 70, D))
    dq0 = rand_bf16((B, H, Sq, D), 0.05)
    scale = 1.0 / np.sqrt(D)
    grads, _ = gpu_kv2(q, ka, va, kb, vb, g, scale, dq=to_dev(dq0), accumulate_dq=True)
    check_against_oracle(grads, q, ka, va, kb, vb, g, scale, "kv2 bwd accumulate", dq0=dq0)


def test_bwd_kv2_accumulates_dk_dv_of_both_sources():
    # query blocks (Ring attention's backward): each source's dk, dv add into the given ones
    B, H, Sq, D = 1, 2, 300, 64
    q, g = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Sq, D))
    ka, va = rand_bf16((B, H, 140, D)), rand_bf16((B, H, 140, D))
    kb, vb = rand_bf16((B, H, 200, D)), rand_bf16((B, H, 200, D))
    olds = [rand_bf16(x.shape, 0.05) for x in (ka, va, kb, vb)]
    scale = 1.0 / np.sqrt(D)
    grads, _ = gpu_kv2(q, ka, va, kb, vb, g, scale, dkv=tuple(to_dev(o) for o in olds), accumulate_dkdv=True)
    kc, vc = np.concatenate([ka, kb], axis=2), np.concatenate([va, vb], axis=2)
    rq, rk, rv = oracle.attention_bwd(q, kc, vc, g, scale)
    bq, bk = delta_bounds(q, kc, vc, g, scale)
    rk = rk + np.concatenate([bits_to_f64(olds[0]), bits_to_f64(olds[2])], axis=2)
    rv = rv + np.concatenate([bits_to_f64(olds[1]), bits_to_f64(olds[3])], axis=2)
    check_grad(grads[0], rq, "kv2 acc dq", bq)
    check_grad(np.concatenate([bits_to_f64(grads[1]), bits_to_f64(grads[3])], axis=2), rk, "kv2 acc dk",
               bk + 2.0 ** -8 * np.abs(rk))
    check_grad(np.concatenate([bits_to_f64(grads[2]), bits_to_f64(grads[4])], axis=2), rv, "kv2 acc dv",
               2.0 ** -8 * np.abs(rv))


def test_bwd_kv2_one_source_empty_is_the_one_source_gradient():
    B, H, Sq, D = 1, 2, 200, 64
    q, g = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Sq, D))
    k, v = rand_bf16((B, H, 333, D)), rand_bf16((B, H, 333, D))
    empty = np.zeros((B, H, 0, D), dtype=np.uint16)
    scale = 0.125
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    out, lse = rg.attn_fwd(tq, tk, tv, scale)
    want = [to_bits(t) for t in rg.attn_bwd(tq, tk, tv, out, lse, tg, scale)]
    te = to_dev(empty)
    for first in (True, False):
        srcs = (tk, tv, te, te) if first else (te, te, tk, tv)
        dq, dka, dva, dkb, dvb = rg.attn_bwd_kv2(tq, *srcs, out, lse, tg, scale)
        torch.cuda.synchronize()
        got = [dq, dka, dva] if first else [dq, dkb, dvb]
        for a, b in zip(got, want):
            np.testing.assert_array_equal(to_bits(a), b)


def test_bwd_kv2_no_queries_zeroes_both_sources():
    D = 128
    q = torch.zeros((1, 2, 0, D), dtype=torch.bfloat16, device="cuda")
    ka, va = (to_dev(rand_bf16((1, 2, 50, D))) for _ in range(2))
    kb, vb = (to_dev(rand_bf16((1, 2, 30, D))) for _ in range(2))
    lse = torch.zeros((1, 2, 0), device="cuda")
    dq, dka, dva, dkb, dvb = rg.attn_bwd_kv2(q, ka, va, kb, vb, q, lse, q, 0.1)
    torch.cuda.synchronize()
    for t in (dka, dva, dkb, dvb):
        assert float(t.float().abs().max()) == 0.0


def test_workload_bwd_kv2_cross_attention_sampled():
    """The cross-attention workload (31200 video tokens; 1560 reference-frame +
    512 conditioning keys in two buffers): every head through the two-source
    forward and gradient; two heads compared with the oracle on sampled rows;
    every head checked by the identities sum_j dv_j = sum_i dO_i and
    sum_j dk_j = 0 over both sources' keys."""
    w = synth.WORKLOADS["cross_s31200_kv2072"]
    q, k, v = synth.make_inputs(w)
    g = synth.make_dout(w)
    na = 1560
    ka, kb, va, vb = k[:, :, :na], k[:, :, na:], v[:, :, :na], v[:, :, na:]
    (dq, dka, dva, dkb, dvb), _ = gpu_kv2(q, ka, va, kb, vb, g, w.scale)
    BH = w.B * w.H
    gk = np.concatenate([dka, dkb], axis=2).reshape(BH, w.Skv, w.D)
    gv = np.concatenate([dva, dvb], axis=2).reshape(BH, w.Skv, w.D)
    fv, fk = bits_to_f64(gv), bits_to_f64(gk)
    sg = bits_to_f64(g.reshape(BH, w.Sq, w.D)).sum(axis=1)
    assert np.all(np.abs(fv.sum(axis=1) - sg) <= 4 * 2.0 ** -8 * np.abs(fv).sum(axis=1) + 1e-3)
    assert np.all(np.abs(fk.sum(axis=1)) <= 4 * 2.0 ** -8 * np.abs(fk).sum(axis=1) + 1e-6)
    heads = [0, 39]
    r = np.random.default_rng(5)
    qrows = np.array(sorted({0, 127, 128, w.Sq - 1} | set(r.choice(w.Sq, 24, replace=False).tolist())))
    krows = np.array(sorted({0, na - 1, na, na + 127, w.Skv - 1} | set(r.choice(w.Skv, 24, replace=False).tolist())))
    qh, kh = q.reshape(BH, w.Sq, w.D)[heads], k.reshape(BH, w.Skv, w.D)[heads]
    vh, gh = v.reshape(BH, w.Skv, w.D)[heads], g.reshape(BH, w.Sq, w.D)[heads]
    rq, rk, rv = oracle.attention_bwd_rows(qh, kh, vh, gh, w.scale, qrows, krows)
    check_grad(dq.reshape(BH, w.Sq, w.D)[heads][:, qrows], rq, "cross kv2 dq")
    check_grad(gk[heads][:, krows], rk, "cross kv2 dk")
    check_grad(gv[heads][:, krows], rv, "cross kv2 dv")
