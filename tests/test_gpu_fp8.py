"""GPU parity of the FP8 (E4M3) variant through the C ABI: the blockwise
quantiser bit for bit against the oracle's, and the FP8 attention against the
oracle's exact attention of the dequantised inputs (contract:
util.check_fp8_attention)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from util import bits_to_f64, check_fp8_attention, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(8080)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rg.load()
    yield
    rc, site = rg.regen_last_device_error()
    assert rc == 0, f"a kernel recorded a device error: {rc} at wait site {site}"


def rand_bf16(shape, scale=1.0):
    return synth.f64_to_bf16_bits(RNG.normal(size=shape) * scale)


def quant_gpu(bits):
    codes, scales = rg.quant_e4m3(to_dev(bits))
    torch.cuda.synchronize()
    return codes, scales


def fp8_case(q, k, v, scale, rows=None, label=""):
    """GPU quantise + FP8 attention; the oracle quantises the same bits itself."""
    (q8, qs), (k8, ks), (v8, vs) = (quant_gpu(x) for x in (q, k, v))
    out, lse = rg.attn_fwd_fp8(q8, qs, k8, ks, v8, vs, scale)
    torch.cuda.synchronize()
    deq = []
    for x, c, sc in ((q, q8, qs), (k, k8, ks), (v, v8, vs)):
        oc, osc = oracle.quantize_e4m3(x)
        np.testing.assert_array_equal(c.cpu().numpy(), oc)
        np.testing.assert_array_equal(sc.cpu().numpy(), osc)
        deq.append(oracle.dequantize_e4m3(oc, osc))
    got, glse = to_bits(out), lse.cpu().numpy()
    D = q.shape[-1]
    if rows is not None:
        got, glse = got.reshape(-1, D)[rows], glse.reshape(-1)[rows]
    return check_fp8_attention(got, glse, *deq, scale, rows=rows, label=label)


@pytest.mark.parametrize("shape,D", [((1, 2, 300), 128), ((2, 1, 128), 64), ((1, 1, 1), 128), ((1, 3, 1000), 64)])
def test_quant_e4m3_bit_exact(shape, D):
    x = rand_bf16(shape + (D,), 3.0)
    xf = synth.bf16_bits_to_f64(x)
    xf[..., :1, :] *= 1e-4                                  # a block with a small row
    if shape[-1] > 256:
        xf[:, :, 128:256] = 0.0                             # an all-zero block
    x = synth.f64_to_bf16_bits(xf)
    codes, scales = quant_gpu(x)
    oc, osc = oracle.quantize_e4m3(x)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)
    np.testing.assert_array_equal(scales.cpu().numpy(), osc)


@pytest.mark.parametrize("B,H,Sq,Skv", [(1, 2, 256, 256), (1, 2, 300, 200), (2, 3, 130, 517), (1, 1, 1, 1),
                                        (1, 1, 700, 77), (1, 2, 513, 1100)])
def test_attn_fp8_small_shapes(B, H, Sq, Skv):
    q, k, v = rand_bf16((B, H, Sq, 128)), rand_bf16((B, H, Skv, 128)), rand_bf16((B, H, Skv, 128))
    fp8_case(q, k, v, 1 / np.sqrt(128), label=f"{B}x{H}x{Sq}x{Skv}")


def test_attn_fp8_block_scales_differ():
    # V blocks of very different magnitude: the per-block scales fold into P's exponent
    q, k = rand_bf16((1, 2, 260, 128)), rand_bf16((1, 2, 640, 128))
    vf = RNG.normal(size=(1, 2, 640, 128)) * np.repeat([1.0, 0.05, 8.0, 0.3, 2.0], 128)[None, None, :, None]
    fp8_case(q, k, synth.f64_to_bf16_bits(vf), 1 / np.sqrt(128), label="block scales")


@pytest.mark.parametrize("scale", [-0.07, 0.3])
def test_attn_fp8_scale_sign_and_size(scale):
    q, k, v = rand_bf16((1, 2, 300, 128)), rand_bf16((1, 2, 420, 128)), rand_bf16((1, 2, 420, 128))
    fp8_case(q, k, v, scale, label=f"scale {scale}")


def test_attn_fp8_spiky_logits():
    q = synth.f64_to_bf16_bits(synth.bf16_bits_to_f64(rand_bf16((1, 2, 260, 128))) * 4.0)
    kk = synth.bf16_bits_to_f64(rand_bf16((1, 2, 390, 128)))
    kk[:, :, ::37] *= 8.0
    fp8_case(q, synth.f64_to_bf16_bits(kk), rand_bf16((1, 2, 390, 128)), 1 / np.sqrt(128), label="spiky")


def test_attn_fp8_empty_kv():
    q8 = torch.zeros((1, 2, 50, 128), dtype=torch.uint8, device="cuda")
    qs = torch.ones((1, 2, 1), device="cuda")
    k8 = torch.zeros((1, 2, 0, 128), dtype=torch.uint8, device="cuda")
    ks = torch.ones((1, 2, 0), device="cuda")
    out, lse = rg.attn_fwd_fp8(q8, qs, k8, ks, k8, ks, 0.1)
    torch.cuda.synchronize()
    assert float(out.float().abs().max()) == 0.0 and bool(torch.isneginf(lse).all())


def _workload_fp8(name, heads, per_head=48):
    """RoPE (when the workload has it) and quantisation on the GPU, FP8 attention
    for the whole workload; sampled rows of the given heads checked."""
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_inputs(w)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    if w.rope:
        rg.rope3d_(tq, tk, w.grid, w.theta)
    (q8, qs), (k8, ks), (v8, vs) = rg.quant_e4m3(tq), rg.quant_e4m3(tk), rg.quant_e4m3(tv)
    out, lse = rg.attn_fwd_fp8(q8, qs, k8, ks, v8, vs, w.scale)
    torch.cuda.synchronize()
    BH = w.B * w.H
    qh, kh = q.reshape(BH, w.Sq, w.D)[heads], k.reshape(BH, w.Skv, w.D)[heads]
    vh = v.reshape(BH, w.Skv, w.D)[heads]
    if w.rope:
        qh, kh = oracle.rope3d(qh, w.grid, w.theta), oracle.rope3d(kh, w.grid, w.theta)
    deq = [oracle.dequantize_e4m3(*oracle.quantize_e4m3(x)) for x in (qh, kh, vh)]
    # the GPU's codes and scales of those heads equal the oracle's
    for gc, gs, x in ((q8, qs, qh), (k8, ks, kh), (v8, vs, vh)):
        oc, osc = oracle.quantize_e4m3(x)
        np.testing.assert_array_equal(gc.cpu().numpy().reshape((BH,) + gc.shape[2:])[heads], oc)
        np.testing.assert_array_equal(gs.cpu().numpy().reshape(BH, -1)[heads], osc)
    rng = np.random.default_rng(0)
    local = np.sort(np.unique(np.concatenate([[0, 127, 128, w.Sq - 1], rng.choice(w.Sq, per_head, replace=False)])))
    rows = (np.arange(len(heads))[:, None] * w.Sq + local[None, :]).reshape(-1)
    got = to_bits(out).reshape(BH, w.Sq, w.D)[heads].reshape(-1, w.D)[rows]
    glse = lse.cpu().numpy().reshape(BH, w.Sq)[heads].reshape(-1)[rows]
    return check_fp8_attention(got, glse, *deq, w.scale, rows=rows, label=name)


def test_workload_fp8_25_frame_window_sampled():
    _workload_fp8("win25_s10920", [0, 7, 11])


def test_workload_fp8_77_frame_window_sampled():
    _workload_fp8("win77_s31200", [0, 19, 39])


def test_workload_fp8_cross_attention_sampled():
    _workload_fp8("cross_s31200_kv2072", [0, 39])


def test_workload_fp8_softmax_stress_sampled():
    _workload_fp8("stress_s10920", [3, 30])
