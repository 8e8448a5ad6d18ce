"""GPU parity of the two-source attention (regen_attn_fwd_kv2) through the C ABI.

The cross-attention of the video tokens reads two key sets held apart: the
reference-frame latent tokens and the conditioning tokens (mlsanity.com
abstract; blog page, "Methodology -- deep read"). Its definition is one
softmax over the two sets concatenated, so the oracle is the fp64 attention
over the concatenated keys and values. Contract as for regen_attn_fwd:
|out - ref| <= 1e-2 + 1e-2 |ref|, |lse - ref| <= 1e-3.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from util import check_attention, sample_rows, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(20261203)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rg.load()
    yield
    rc, site = rg.regen_last_device_error()
    assert rc == 0, f"a kernel recorded a device error: {rc} at wait site {site}"


def rand_bf16(shape, scale=1.0):
    return synth.f64_to_bf16_bits(RNG.normal(size=shape) * scale)


def run_kv2(q, ka, va, kb, vb, scale):
    """Two-source attention with NaN guard regions around out and lse."""
    B, H, Sq, D = q.shape
    n_out, n_lse, pad = B * H * Sq * D, B * H * Sq, 4096
    out_buf = torch.full((n_out + 2 * pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse_buf = torch.full((n_lse + 2 * pad,), float("nan"), dtype=torch.float32, device="cuda")
    out = out_buf[pad:pad + n_out].view(B, H, Sq, D)
    lse = lse_buf[pad:pad + n_lse].view(B, H, Sq)
    dka, dva, dkb, dvb = (to_dev(x) for x in (ka, va, kb, vb))
    rg.regen_attn_fwd_kv2(to_dev(q), dka, dva, dkb, dvb, out, lse, B, H, Sq, ka.shape[2], kb.shape[2], D, scale)
    torch.cuda.synchronize()
    assert torch.isnan(out_buf[:pad].float()).all() and torch.isnan(out_buf[pad + n_out:].float()).all()
    assert torch.isnan(lse_buf[:pad]).all() and torch.isnan(lse_buf[pad + n_lse:]).all()
    return to_bits(out), lse.cpu().numpy()


@pytest.mark.parametrize("B,H,Sq,Skv_a,Skv_b,D", [
    (1, 1, 128, 1, 1, 128), (1, 2, 200, 24, 512, 128), (1, 1, 129, 128, 128, 128), (2, 1, 300, 127, 129, 64),
    (1, 2, 257, 1560, 512, 128), (1, 1, 1, 300, 40, 128), (1, 3, 513, 5, 700, 64), (1, 1, 256, 256, 1, 128),
])
def test_kv2_against_oracle_over_concatenated_keys(B, H, Sq, Skv_a, Skv_b, D):
    q = rand_bf16((B, H, Sq, D))
    ka, va = rand_bf16((B, H, Skv_a, D)), rand_bf16((B, H, Skv_a, D))
    kb, vb = rand_bf16((B, H, Skv_b, D)), rand_bf16((B, H, Skv_b, D))
    scale = 1.0 / np.sqrt(D)
    out, lse = run_kv2(q, ka, va, kb, vb, scale)
    ref, rl = oracle.attention(q, np.concatenate([ka, kb], axis=2), np.concatenate([va, vb], axis=2), scale)
    check_attention(out, lse, ref, rl, f"kv2 {Skv_a}+{Skv_b}")


def test_kv2_negative_scale_and_spiky_keys():
    B, H, Sq, D = 1, 2, 300, 128
    q = rand_bf16((B, H, Sq, D), 4.0)
    ka, va = rand_bf16((B, H, 150, D)), rand_bf16((B, H, 150, D))
    kb, vb = rand_bf16((B, H, 90, D)), rand_bf16((B, H, 90, D))
    kb[:, :, ::17] = synth.f64_to_bf16_bits(synth.bf16_bits_to_f64(kb[:, :, ::17]) * 8.0)   # spikes in source b
    for scale in (-0.09, 0.09):
        out, lse = run_kv2(q, ka, va, kb, vb, scale)
        ref, rl = oracle.attention(q, np.concatenate([ka, kb], axis=2), np.concatenate([va, vb], axis=2), scale)
        check_attention(out, lse, ref, rl, f"kv2 scale {scale}")


def test_kv2_equals_one_call_over_the_concatenation_when_a_fills_whole_blocks():
    # Source a a multiple of 128 keys: the key blocks and their order are the
    # same as one call over the concatenated keys, so the bits are too.
    B, H, Sq, D = 1, 3, 400, 128
    q = rand_bf16((B, H, Sq, D))
    ka, va = rand_bf16((B, H, 256, D)), rand_bf16((B, H, 256, D))
    kb, vb = rand_bf16((B, H, 300, D)), rand_bf16((B, H, 300, D))
    out, lse = run_kv2(q, ka, va, kb, vb, 0.088)
    o1, l1 = rg.attn_fwd(to_dev(q), to_dev(np.concatenate([ka, kb], axis=2)),
                         to_dev(np.concatenate([va, vb], axis=2)), 0.088)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out, to_bits(o1))
    np.testing.assert_array_equal(lse, l1.cpu().numpy())


def test_kv2_with_an_empty_source_is_the_plain_attention():
    B, H, Sq, D = 1, 2, 130, 64
    q = rand_bf16((B, H, Sq, D))
    k, v = rand_bf16((B, H, 77, D)), rand_bf16((B, H, 77, D))
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    o1, l1 = rg.attn_fwd(dq, dk, dv, 0.125)
    for a_empty in (False, True):
        out = torch.empty_like(dq)
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device="cuda")
        if a_empty:
            rg.regen_attn_fwd_kv2(dq, None, None, dk, dv, out, lse, B, H, Sq, 0, 77, D, 0.125)
        else:
            rg.regen_attn_fwd_kv2(dq, dk, dv, None, None, out, lse, B, H, Sq, 77, 0, D, 0.125)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(to_bits(out), to_bits(o1))
        np.testing.assert_array_equal(lse.cpu().numpy(), l1.cpu().numpy())
    # both empty: the empty softmax (out 0, lse -inf)
    out = torch.full_like(dq, 1.0)
    lse = torch.zeros((B, H, Sq), dtype=torch.float32, device="cuda")
    rg.regen_attn_fwd_kv2(dq, None, None, None, None, out, lse, B, H, Sq, 0, 0, D, 0.125)
    torch.cuda.synchronize()
    assert (out.float() == 0).all() and torch.isneginf(lse).all()


def test_kv2_cross_attention_workload_sampled():
    # The cross-attention workload: 31200 video tokens, 1560 reference-frame +
    # 512 conditioning keys, 40 heads; sampled rows of 8 heads vs the oracle.
    w = synth.WORKLOADS["cross_s31200_kv2072"]
    q, k, v = synth.make_inputs(w)
    n_ref = 1560
    dq = to_dev(q)
    dka, dva = to_dev(np.ascontiguousarray(k[:, :, :n_ref])), to_dev(np.ascontiguousarray(v[:, :, :n_ref]))
    dkb, dvb = to_dev(np.ascontiguousarray(k[:, :, n_ref:])), to_dev(np.ascontiguousarray(v[:, :, n_ref:]))
    out, lse = rg.attn_fwd_kv2(dq, dka, dva, dkb, dvb, w.scale)
    torch.cuda.synchronize()
    heads = [0, 5, 11, 17, 23, 29, 35, 39]
    BH = w.B * w.H
    qh, kh, vh = (x.reshape(BH, -1, w.D)[heads] for x in (q, k, v))
    rows = sample_rows(len(heads), w.Sq, 64)
    ref, rl = oracle.attention(qh, kh, vh, w.scale, rows=rows)
    gout = to_bits(out).reshape(BH, w.Sq, w.D)[heads].reshape(-1, w.D)[rows]
    glse = lse.cpu().numpy().reshape(BH, w.Sq)[heads].reshape(-1)[rows]
    check_attention(gout, glse, ref, rl, "cross kv2")
