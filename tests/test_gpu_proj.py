"""GPU parity of the DiT block's projections around the attention through the
C ABI (regen_qkv_proj with its fused per-head RMSNorm and 3D RoPE, and
regen_out_proj reading the attention output in place) against the oracle's
fp64 projections on the same bf16 inputs (contract: util.check_proj)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from util import check_attention, check_proj, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(9090)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rg.load()
    yield
    rc, site = rg.regen_last_device_error()
    assert rc == 0, f"a kernel recorded a device error: {rc} at wait site {site}"


def rand_bf16(shape, scale=1.0):
    return synth.f64_to_bf16_bits(RNG.normal(size=shape) * scale)


def f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def qkv_case(B, grid, C, H, with_bias=True, with_gamma=True, rows=None, theta=10000.0):
    S = grid[0] * grid[1] * grid[2]
    x = rand_bf16((B, S, C))
    w = rand_bf16((3 * H * 128, C), 1 / np.sqrt(C))
    bias = (RNG.normal(size=3 * H * 128) * 0.1).astype(np.float32) if with_bias else None
    gq = (1 + 0.1 * RNG.normal(size=H * 128)).astype(np.float32) if with_gamma else None
    gk = (1 + 0.1 * RNG.normal(size=H * 128)).astype(np.float32) if with_gamma else None
    q, k, v = rg.qkv_proj(to_dev(x), to_dev(w), H, grid, None if bias is None else f32(bias),
                          None if gq is None else f32(gq), None if gk is None else f32(gk), theta=theta)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_proj(x, w, bias, gq, gk, H, grid, theta, 1e-6, rows=rows)
    # the GPU writes [B, H, S, D]; the oracle returns [rows, H, D]
    sel = (lambda a: a.transpose(0, 2, 1, 3).reshape(B * S, H, 128)) if rows is None else \
        (lambda a: a.transpose(0, 2, 1, 3).reshape(B * S, H, 128)[rows])
    return [check_proj(sel(to_bits(g)), r, n) for g, r, n in ((q, rq, "q"), (k, rk, "k"), (v, rv, "v"))]


def test_qkv_proj_small():
    qkv_case(1, (3, 4, 5), 256, 2)


def test_qkv_proj_ragged_everything():
    # S = 132 (a 4-row second token tile, batch boundary inside no tile), C = 200
    # (a partial last K block), H = 3 (N = 1152: the last feature tile half empty)
    qkv_case(2, (2, 6, 11), 200, 3, theta=500.0)


def test_qkv_proj_without_bias_or_gamma():
    qkv_case(1, (2, 5, 13), 128, 2, with_bias=False, with_gamma=False)


def test_qkv_proj_wan14b_77_frame_window_sampled():
    # the 14B-class DiT's projection on the 77-frame window: S = 31200, C = 5120, H = 40
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 31199], RNG.choice(31200, 27, replace=False)]))
    qkv_case(1, (20, 30, 52), 5120, 40, rows=rows)


def out_case(B, H, S, N, with_bias=True, rows=None):
    o = rand_bf16((B, H, S, 128))
    w = rand_bf16((N, H * 128), 1 / np.sqrt(H * 128))
    bias = (RNG.normal(size=N) * 0.1).astype(np.float32) if with_bias else None
    y = rg.out_proj(to_dev(o), to_dev(w), None if bias is None else f32(bias))
    torch.cuda.synchronize()
    ref = oracle.out_proj(o, w, bias, rows=rows)
    got = to_bits(y).reshape(B * S, N)
    return check_proj(got if rows is None else got[rows], ref, "out")


@pytest.mark.parametrize("B,H,S,N", [(1, 2, 256, 256), (2, 3, 130, 200), (1, 1, 1, 8), (1, 4, 300, 520)])
def test_out_proj_small(B, H, S, N):
    out_case(B, H, S, N)


def test_out_proj_without_bias():
    out_case(1, 2, 200, 264, with_bias=False)


def test_out_proj_wan14b_77_frame_window_sampled():
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 31199], RNG.choice(31200, 27, replace=False)]))
    out_case(1, 40, 31200, 5120, rows=rows)


def test_dit_attention_block_chain():
    # x -> fused QKV projection (RMSNorm, RoPE) -> attention -> output projection,
    # against the oracle's chain with its own bf16 rounding of q, k, v and o
    B, grid, C, H, N = 1, (2, 8, 16), 256, 2, 256
    S = grid[0] * grid[1] * grid[2]
    x = rand_bf16((B, S, C))
    w = rand_bf16((3 * H * 128, C), 1 / np.sqrt(C))
    wo = rand_bf16((N, H * 128), 1 / np.sqrt(H * 128))
    q, k, v = rg.qkv_proj(to_dev(x), to_dev(w), H, grid)
    o, lse = rg.attn_fwd(q, k, v)
    y = rg.out_proj(o, to_dev(wo))
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_proj(x, w, None, None, None, H, grid, 10000.0, 1e-6)
    to_bhsd = lambda a: oracle.f64_to_bf16(a.reshape(B, S, H, 128).transpose(0, 2, 1, 3))  # noqa: E731
    ro, rl = oracle.attention(to_bhsd(rq), to_bhsd(rk), to_bhsd(rv), 1 / np.sqrt(128))
    check_attention(to_bits(o).reshape(-1, 128), lse.cpu().numpy().reshape(-1), ro.reshape(-1, 128),
                    rl.reshape(-1), "chain attention")
    ry = oracle.out_proj(oracle.f64_to_bf16(ro), wo, None)
    got = to_bits(y).reshape(B * S, N)
    err = np.abs(synth.bf16_bits_to_f64(got) - ry)
    # o differs from the oracle's by the attention's own contract: bound its effect
    assert err.max() <= 0.05 * np.sqrt(np.mean(ry ** 2)) + 2.0 ** -7 * np.abs(ry).max(), err.max()
