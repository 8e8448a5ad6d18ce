"""GPU parity of the torch.autograd glue (dit_attention_b200.autograd): the
forward against the oracle's attention, and the gradients that autograd
returns against the oracle's chain rule, on seeded bf16 inputs with ragged
tiles. Contracts: util.check_attention and util.check_grad."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from dit_attention_b200.autograd import dit_attention, dit_cross_attention  # noqa: E402
from util import check_attention, check_grad, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(8181)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rg.load()
    yield
    rc, site = rg.regen_last_device_error()
    assert rc == 0, f"a kernel recorded a device error: {rc} at wait site {site}"


def rand_bf16(shape):
    return synth.f64_to_bf16_bits(RNG.normal(size=shape))


def leaf(bits):
    return to_dev(bits).requires_grad_(True)


def test_self_attention_with_rope_forward_and_gradients():
    B, H, grid, D = 1, 2, (3, 6, 11), 128
    S = grid[0] * grid[1] * grid[2]
    q, k, v, g = (rand_bf16((B, H, S, D)) for _ in range(4))
    tq, tk, tv = leaf(q), leaf(k), leaf(v)
    out = dit_attention(tq, tk, tv, grid=grid)
    out.backward(to_dev(g))
    torch.cuda.synchronize()
    # the inputs are left unrotated
    np.testing.assert_array_equal(to_bits(tq.detach()), q)
    qr, kr = oracle.rope3d(q, grid), oracle.rope3d(k, grid)
    scale = 1 / np.sqrt(D)
    ref, _ = oracle.attention(qr, kr, v, scale)
    check_attention(to_bits(out.detach()).reshape(-1, D), None, ref.reshape(-1, D), None, "autograd forward")
    rq, rk, rv = oracle.attention_bwd(qr, kr, v, g, scale)
    check_grad(to_bits(tq.grad), oracle.rope3d_bwd(rq, grid), "autograd dq")
    check_grad(to_bits(tk.grad), oracle.rope3d_bwd(rk, grid), "autograd dk")
    check_grad(to_bits(tv.grad), rv, "autograd dv")


def test_self_attention_without_rope_scale_given():
    B, H, Sq, Skv, D = 2, 1, 300, 200, 64
    q, g = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Sq, D))
    k, v = rand_bf16((B, H, Skv, D)), rand_bf16((B, H, Skv, D))
    tq, tk, tv = leaf(q), leaf(k), leaf(v)
    out = dit_attention(tq, tk, tv, scale=0.2)
    out.backward(to_dev(g))
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, 0.2)
    check_grad(to_bits(tq.grad), rq, "dq")
    check_grad(to_bits(tk.grad), rk, "dk")
    check_grad(to_bits(tv.grad), rv, "dv")


def test_two_source_cross_attention_forward_and_gradients():
    # one softmax over [source a; source b], as the oracle computes it on the
    # concatenated keys
    B, H, Sq, D = 1, 2, 333, 128
    s1, s2 = 270, 141
    q, g = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Sq, D))
    k, v = rand_bf16((B, H, s1 + s2, D)), rand_bf16((B, H, s1 + s2, D))
    tq = leaf(q)
    ka, kb = leaf(k[:, :, :s1]), leaf(k[:, :, s1:])
    va, vb = leaf(v[:, :, :s1]), leaf(v[:, :, s1:])
    out = dit_cross_attention(tq, (ka, va), (kb, vb))
    out.backward(to_dev(g))
    torch.cuda.synchronize()
    scale = 1 / np.sqrt(D)
    ref, _ = oracle.attention(q, k, v, scale)
    check_attention(to_bits(out.detach()).reshape(-1, D), None, ref.reshape(-1, D), None, "two-source forward")
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, scale)
    check_grad(to_bits(tq.grad), rq, "two-source dq")
    check_grad(np.concatenate([to_bits(ka.grad), to_bits(kb.grad)], axis=2), rk, "two-source dk")
    check_grad(np.concatenate([to_bits(va.grad), to_bits(vb.grad)], axis=2), rv, "two-source dv")
