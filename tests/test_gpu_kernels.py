"""GPU parity: rope3d, lse_merge and attention through the C ABI vs the fp64 oracle.

Every expected value comes from ``oracle`` on the same seeded bf16 inputs.
Accuracy contract (bf16 outputs): |out - ref| <= 1e-2 + 1e-2 |ref|;
fp32 LSE: |lse - ref| <= 1e-3. RoPE is compared bit for bit (both sides round
the fp64 rotation once to bf16, nearest-even).
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from util import bits_to_f64, check_attention, sample_rows, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(20261202)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rg.load()
    yield
    rc, site = rg.regen_last_device_error()
    assert rc == 0, f"a kernel recorded a device error: {rc} at wait site {site}"


def rand_bf16(shape, scale=1.0):
    return synth.f64_to_bf16_bits(RNG.normal(size=shape) * scale)


# ------------------------------------------------------------------ RoPE ---

@pytest.mark.parametrize("B,H,grid,D", [
    (1, 2, (3, 5, 7), 128), (2, 3, (2, 4, 6), 64), (1, 1, (1, 1, 9), 8), (1, 5, (4, 3, 2), 24),
    (1, 3, (7, 30, 52), 128),
])
def test_rope3d_bit_exact(B, H, grid, D):
    S = grid[0] * grid[1] * grid[2]
    q = rand_bf16((B, H, S, D))
    k = rand_bf16((B, H, S, D))
    dq, dk = to_dev(q), to_dev(k)
    rg.rope3d_(dq, dk, grid, 10000.0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_bits(dq), oracle.rope3d(q, grid, 10000.0))
    np.testing.assert_array_equal(to_bits(dk), oracle.rope3d(k, grid, 10000.0))


def test_rope3d_q_only_and_theta():
    grid = (2, 3, 5)
    q = rand_bf16((1, 2, 30, 64))
    dq = to_dev(q)
    rg.rope3d_(dq, None, grid, 500.0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_bits(dq), oracle.rope3d(q, grid, 500.0))


def test_rope3d_full_77_frame_window_sampled_heads():
    w = synth.WORKLOADS["win77_s31200"]
    q, k, _ = synth.make_inputs(w)
    dq, dk = to_dev(q), to_dev(k)
    rg.rope3d_(dq, dk, w.grid, w.theta)
    torch.cuda.synchronize()
    heads = [0, 17, 39]
    gq, gk = to_bits(dq), to_bits(dk)
    for h in heads:
        np.testing.assert_array_equal(gq[0, h], oracle.rope3d(q[0, h], w.grid, w.theta))
        np.testing.assert_array_equal(gk[0, h], oracle.rope3d(k[0, h], w.grid, w.theta))


def _all_finite_bf16_patterns(n_rows, D, seed):
    """Every finite bf16 bit pattern (zeros, subnormals, up to +-max) once,
    shuffled, then filled up with random ones: [n_rows, D]."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]                   # drop inf and NaN
    rng = np.random.default_rng(seed)
    need = n_rows * D
    assert need >= bits.size
    fill = rng.choice(bits, size=need - bits.size)
    return rng.permutation(np.concatenate([bits, fill])).reshape(n_rows, D)


def test_rope3d_every_finite_bf16_pattern_bit_exact():
    # The rotation runs in fp32 and proves per pair that it rounds like fp64,
    # else redoes the pair in fp64: across every finite bf16 magnitude
    # (subnormals, values whose products overflow fp32, exact zeros) the bits
    # must equal the oracle's fp64 rotation, forward and inverse.
    grid, D, H = (3, 5, 7), 128, 6          # 105 tokens x 128 x 6 heads = 80640 values
    S = grid[0] * grid[1] * grid[2]
    q = _all_finite_bf16_patterns(H * S, D, 1).reshape(1, H, S, D)
    k = _all_finite_bf16_patterns(H * S, D, 2).reshape(1, H, S, D)
    for theta in (10000.0, 3.0):
        dq, dk = to_dev(q), to_dev(k)
        rg.rope3d_(dq, dk, grid, theta)
        torch.cuda.synchronize()
        gq, gk = to_bits(dq), to_bits(dk)
        np.testing.assert_array_equal(gq, oracle.rope3d(q, grid, theta))
        np.testing.assert_array_equal(gk, oracle.rope3d(k, grid, theta))
        rg.rope3d_bwd_(dq, None, grid, theta)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(to_bits(dq), oracle.rope3d_bwd(gq, grid, theta))


# ------------------------------------------------------------- LSE merge ---

@pytest.mark.parametrize("rows,D", [(1, 128), (2, 128), (777, 128), (4096, 64), (33, 8)])
def test_lse_merge(rows, D):
    oa, ob = rand_bf16((rows, D)), rand_bf16((rows, D))
    la = (RNG.normal(size=rows) * 20).astype(np.float32)
    lb = (RNG.normal(size=rows) * 20).astype(np.float32)
    la[::7] = -np.inf
    lb[::11] = -np.inf
    out, lse = rg.lse_merge(to_dev(oa), torch.from_numpy(la).cuda(), to_dev(ob), torch.from_numpy(lb).cuda())
    torch.cuda.synchronize()
    ref, rl = oracle.lse_merge(oa, la.astype(np.float64), ob, lb.astype(np.float64))
    got = bits_to_f64(to_bits(out))
    # fp32 weights, one bf16 rounding: within one bf16 ulp of the fp64 value
    np.testing.assert_array_less(np.abs(got - ref), np.abs(ref) * 2.0 ** -7 + 1e-30)
    gl = lse.cpu().numpy().astype(np.float64)
    both = np.isneginf(rl)
    assert np.array_equal(np.isneginf(gl), both)
    if (~both).any():
        np.testing.assert_allclose(gl[~both], rl[~both], rtol=0, atol=2e-5 * max(1.0, np.abs(rl[~both]).max()))
    assert np.all(got[both] == 0)


def test_lse_merge_in_place():
    rows, D = 300, 128
    oa, ob = rand_bf16((rows, D)), rand_bf16((rows, D))
    la = RNG.normal(size=rows).astype(np.float32)
    lb = RNG.normal(size=rows).astype(np.float32)
    da = to_dev(oa)
    rg.lse_merge(da, torch.from_numpy(la).cuda(), to_dev(ob), torch.from_numpy(lb).cuda(), out=da)
    torch.cuda.synchronize()
    ref, _ = oracle.lse_merge(oa, la.astype(np.float64), ob, lb.astype(np.float64))
    np.testing.assert_array_less(np.abs(bits_to_f64(to_bits(da)) - ref), np.abs(ref) * 2.0 ** -7 + 1e-30)


# ------------------------------------------------------------- attention ---

def run_attention(q, k, v, scale, guard=True):
    """GPU attention with NaN-filled outputs inside guard regions; checks that
    nothing outside out/lse was written. Returns (out bits, lse)."""
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    n_out, n_lse = B * H * Sq * D, B * H * Sq
    pad = 4096
    out_buf = torch.full((n_out + 2 * pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse_buf = torch.full((n_lse + 2 * pad,), float("nan"), dtype=torch.float32, device="cuda")
    out = out_buf[pad:pad + n_out].view(B, H, Sq, D)
    lse = lse_buf[pad:pad + n_lse].view(B, H, Sq)
    rg.regen_attn_fwd(dq, dk, dv, out, lse, B, H, Sq, Skv, D, scale)
    torch.cuda.synchronize()
    if guard:
        assert torch.isnan(out_buf[:pad].float()).all() and torch.isnan(out_buf[pad + n_out:].float()).all()
        assert torch.isnan(lse_buf[:pad]).all() and torch.isnan(lse_buf[pad + n_lse:]).all()
    return to_bits(out), lse.cpu().numpy()


@pytest.mark.parametrize("B,H,Sq,Skv,D", [
    (1, 1, 128, 128, 128), (1, 1, 1, 1, 128), (1, 2, 2, 2, 64), (1, 1, 127, 129, 128),
    (1, 1, 129, 127, 128), (2, 1, 255, 255, 128), (1, 1, 256, 2072, 128), (1, 1, 300, 1, 64),
    (1, 2, 257, 384, 64), (3, 1, 100, 1000, 128), (1, 1, 513, 130, 128),
])
def test_attention_small_shapes(B, H, Sq, Skv, D):
    q, k, v = rand_bf16((B, H, Sq, D)), rand_bf16((B, H, Skv, D)), rand_bf16((B, H, Skv, D))
    scale = 1.0 / math.sqrt(D)
    out, lse = run_attention(q, k, v, scale)
    ref, rl = oracle.attention(q, k, v, scale)
    check_attention(out, lse, ref, rl, f"B{B} H{H} Sq{Sq} Skv{Skv} D{D}")


def test_attention_many_heads_more_ctas_than_sms():
    B, H, S, D = 2, 100, 300, 128        # 400 CTAs over 148 SMs
    q, k, v = rand_bf16((B, H, S, D)), rand_bf16((B, H, S, D)), rand_bf16((B, H, S, D))
    out, lse = run_attention(q, k, v, 1 / math.sqrt(D))
    rows = sample_rows(B * H, S, 4)
    ref, rl = oracle.attention(q, k, v, 1 / math.sqrt(D), rows=rows)
    check_attention(out.reshape(-1, D)[rows], lse.reshape(-1)[rows], ref, rl, "many heads")


@pytest.mark.parametrize("scale", [0.0, -0.125, 0.5])
def test_attention_scale_edge_cases(scale):
    q, k, v = rand_bf16((1, 2, 200, 128)), rand_bf16((1, 2, 333, 128)), rand_bf16((1, 2, 333, 128))
    out, lse = run_attention(q, k, v, scale)
    ref, rl = oracle.attention(q, k, v, scale)
    check_attention(out, lse, ref, rl, f"scale {scale}")


def test_attention_spiky_logits_rescale_path():
    # logits spanning ~100 (log2) units force O rescaling in later key blocks
    q = rand_bf16((1, 1, 256, 128), 4.0)
    k = rand_bf16((1, 1, 1024, 128))
    kk = synth.bf16_bits_to_f64(k)
    kk[0, 0, 900:910] *= 8.0      # the large logits arrive late
    k = synth.f64_to_bf16_bits(kk)
    v = rand_bf16((1, 1, 1024, 128))
    out, lse = run_attention(q, k, v, 1 / math.sqrt(128))
    ref, rl = oracle.attention(q, k, v, 1 / math.sqrt(128))
    check_attention(out, lse, ref, rl, "spiky")


def test_attention_empty_kv_and_no_queries():
    q = rand_bf16((1, 2, 64, 128))
    dq = to_dev(q)
    out = torch.full_like(dq, float("nan"))
    lse = torch.zeros((1, 2, 64), dtype=torch.float32, device="cuda")
    rg.regen_attn_fwd(dq, None, None, out, lse, 1, 2, 64, 0, 128, 0.1)
    torch.cuda.synchronize()
    assert (out.float() == 0).all() and torch.isneginf(lse).all()
    rg.regen_attn_fwd(dq, dq, dq, out, lse, 1, 2, 0, 64, 128, 0.1)   # Sq = 0: no-op


def test_attention_lse_optional():
    q, k, v = rand_bf16((1, 1, 130, 64)), rand_bf16((1, 1, 130, 64)), rand_bf16((1, 1, 130, 64))
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    out = torch.empty_like(dq)
    rg.regen_attn_fwd(dq, dk, dv, out, None, 1, 1, 130, 130, 64, 0.125)
    torch.cuda.synchronize()
    ref, rl = oracle.attention(q, k, v, 0.125)
    check_attention(to_bits(out), rl, ref, rl, "lse=NULL")


# --------------------------------------------- the five named workloads ---

def _workload(name, per_head, heads=None):
    """Run RoPE (when the workload has it) and attention on the GPU for the whole
    workload; compare the given heads (default all) against the oracle, on
    every row (per_head None) or on sampled rows."""
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_inputs(w)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    if w.rope:
        rg.rope3d_(dq, dk, w.grid, w.theta)
    out, lse = rg.attn_fwd(dq, dk, dv, w.scale)
    torch.cuda.synchronize()
    BH = w.B * w.H
    heads = list(range(BH)) if heads is None else heads
    qh = q.reshape(BH, w.Sq, w.D)[heads]
    kh = k.reshape(BH, w.Skv, w.D)[heads]
    vh = v.reshape(BH, w.Skv, w.D)[heads]
    if w.rope:   # the oracle rotates its own copy of the inputs
        qh = oracle.rope3d(qh, w.grid, w.theta)
        kh = oracle.rope3d(kh, w.grid, w.theta)
    gout = to_bits(out).reshape(BH, w.Sq, w.D)[heads].reshape(-1, w.D)
    glse = lse.cpu().numpy().reshape(BH, w.Sq)[heads].reshape(-1)
    rows = None if per_head is None else sample_rows(len(heads), w.Sq, per_head)
    ref, rl = oracle.attention(qh, kh, vh, w.scale, rows=rows)
    if rows is not None:
        gout, glse = gout[rows], glse[rows]
    else:
        ref, rl = ref.reshape(-1, w.D), rl.reshape(-1)
    return check_attention(gout, glse, ref, rl, name)


SPREAD_HEADS = [0, 5, 11, 17, 23, 29, 35, 39]


def test_workload_tiny_full():
    _workload("tiny_s1024", None)


def test_workload_25_frame_window_sampled():
    _workload("win25_s10920", 48)


def test_workload_77_frame_window_sampled():
    _workload("win77_s31200", 48, heads=SPREAD_HEADS)


def test_workload_cross_attention_sampled():
    _workload("cross_s31200_kv2072", 64, heads=SPREAD_HEADS)


def test_workload_softmax_stress_and_two_block_merge():
    w = synth.WORKLOADS["stress_s10920"]
    q, k, v = synth.make_inputs(w)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    out, lse = rg.attn_fwd(dq, dk, dv, w.scale)
    # the same attention as two KV blocks of 5460 keys merged by their LSE
    s = w.merge_split
    oa, la = rg.attn_fwd(dq, dk[:, :, :s].contiguous(), dv[:, :, :s].contiguous(), w.scale)
    ob, lb = rg.attn_fwd(dq, dk[:, :, s:].contiguous(), dv[:, :, s:].contiguous(), w.scale)
    om, lm = rg.lse_merge(oa, la, ob, lb)
    torch.cuda.synchronize()
    rows = sample_rows(w.B * w.H, w.Sq, 24)
    ref, rl = oracle.attention(q, k, v, w.scale, rows=rows)
    d1 = check_attention(to_bits(out).reshape(-1, w.D)[rows], lse.cpu().numpy().reshape(-1)[rows], ref, rl,
                         "stress")
    d2 = check_attention(to_bits(om).reshape(-1, w.D)[rows], lm.cpu().numpy().reshape(-1)[rows], ref, rl,
                         "stress two-block merge")
    assert d1["rms_ref"] > 0.1      # spiky logits: outputs of order one, so the rtol term binds
    assert d2["max_lse_err"] <= 1e-3


# ------------------------------------------------ the kernel's FMA exp2 ---

def test_selftest_exp2_against_cuda_exp2f_and_fp64():
    # 2^x over the range the softmax feeds it (x <= 8 with the stale-max rule),
    # compared with CUDA's exp2f (torch.exp2 on the GPU) and with fp64.
    x = torch.cat([torch.linspace(-126.0, 8.5, 1 << 20), torch.tensor([-127.0, -200.0, -1e30, 0.0, -0.5, 0.5]),
                   torch.rand(1 << 16) * -30.0]).float().cuda()
    if x.numel() % 2:
        x = torch.cat([x, torch.zeros(1, device="cuda")])
    y = torch.empty_like(x)
    rg.regen_selftest_exp2(x, y, x.numel())
    torch.cuda.synchronize()
    ref64 = torch.exp2(x.double())
    cuda32 = torch.exp2(x)
    normal = x >= -125.5
    rel = ((y.double() - ref64) / ref64)[normal].abs().max().item()
    rel_cuda = ((y.double() - cuda32.double()) / ref64)[normal].abs().max().item()
    assert rel < 4e-6, rel            # fitted bound 2.9e-6 plus fp32 rounding of the reduction
    assert rel_cuda < 4e-6, rel_cuda
    low = x <= -127.0                 # clamped: exactly zero, never negative or NaN
    assert (y[low] == 0).all()
    tiny = (~normal) & (~low)
    assert (y[tiny] >= 0).all() and (y[tiny] < 2.0 ** -124).all()


# ------------------------------------------------- RoPE fused into Q load ---

@pytest.mark.parametrize("B,H,grid,D", [
    (1, 2, (2, 5, 13), 128), (2, 1, (3, 7, 11), 64), (1, 3, (1, 16, 16), 128), (1, 1, (4, 30, 52), 128),
])
def test_rope3d_fused_equals_unfused(B, H, grid, D):
    S = grid[0] * grid[1] * grid[2]
    q, k, v = rand_bf16((B, H, S, D)), rand_bf16((B, H, S, D)), rand_bf16((B, H, S, D))
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    out, lse = rg.attn_fwd_rope3d(dq, dk, dv, grid)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_bits(dq), q)            # inputs untouched
    np.testing.assert_array_equal(to_bits(dk), k)
    uq, uk = dq.clone(), dk.clone()
    rg.rope3d_(uq, uk, grid)
    ref_out, ref_lse = rg.attn_fwd(uq, uk, dv)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_bits(out), to_bits(ref_out))
    np.testing.assert_array_equal(lse.cpu().numpy(), ref_lse.cpu().numpy())


def test_rope3d_fused_25_frame_window_vs_oracle():
    w = synth.WORKLOADS["win25_s10920"]
    q, k, v = synth.make_inputs(w)
    out, lse = rg.attn_fwd_rope3d(to_dev(q), to_dev(k), to_dev(v), w.grid, w.theta)
    torch.cuda.synchronize()
    heads = [0, 5, 11]
    qh = oracle.rope3d(q.reshape(12, w.Sq, w.D)[heads], w.grid, w.theta)
    kh = oracle.rope3d(k.reshape(12, w.Skv, w.D)[heads], w.grid, w.theta)
    rows = sample_rows(len(heads), w.Sq, 64)
    ref, rl = oracle.attention(qh, kh, v.reshape(12, w.Skv, w.D)[heads], w.scale, rows=rows)
    gout = to_bits(out).reshape(12, w.Sq, w.D)[heads].reshape(-1, w.D)[rows]
    glse = lse.cpu().numpy().reshape(12, w.Sq)[heads].reshape(-1)[rows]
    check_attention(gout, glse, ref, rl, "fused rope, 25-frame window")


def test_rope3d_fused_workspace_errors():
    grid = (2, 3, 4)
    q = to_dev(rand_bf16((1, 1, 24, 128)))
    need = rg.regen_attn_fwd_rope3d_workspace_bytes(1, 1, *grid, 128)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(rg.RegenError) as e:
        rg.attn_fwd_rope3d(q, q.clone(), q.clone(), grid, workspace=small)
    assert e.value.status == -1
    ws = torch.empty(need + 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(rg.RegenError) as e:
        rg.attn_fwd_rope3d(q, q.clone(), q.clone(), grid, workspace=ws[16:])
    assert e.value.status == -3


@pytest.mark.parametrize("B,H,Sq,Skv", [(1, 2, 257, 300), (1, 3, 513, 129), (2, 2, 700, 1000), (1, 1, 1024, 77),
                                        (1, 2, 1500, 2072)])
def test_attention_ragged_multi_tile(B, H, Sq, Skv):
    q, k, v = rand_bf16((B, H, Sq, 128)), rand_bf16((B, H, Skv, 128)), rand_bf16((B, H, Skv, 128))
    out, lse = rg.attn_fwd(to_dev(q), to_dev(k), to_dev(v), 1 / math.sqrt(128))
    torch.cuda.synchronize()
    ref, rl = oracle.attention(q, k, v, 1 / math.sqrt(128))
    check_attention(to_bits(out).reshape(-1, 128), lse.cpu().numpy().reshape(-1), ref.reshape(-1, 128),
                    rl.reshape(-1), f"{B}x{H}x{Sq}x{Skv}")


def test_calls_from_a_fresh_host_thread():
    # A thread on which no CUDA call has run has no current context (a torch
    # autograd worker, a user's own thread). Every entry point binds the device
    # that holds its data first: the same calls there give the same bits, after
    # the main thread has already used the library.
    import threading
    B, H, S, D = 1, 2, 300, 128
    q, k, v, g = (synth.f64_to_bf16_bits(RNG.normal(size=(B, H, S, D))) for _ in range(4))
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    out, lse = rg.attn_fwd(tq, tk, tv)
    grads = rg.attn_bwd(tq, tk, tv, out, lse, tg)
    torch.cuda.synchronize()
    res = {}

    def worker():
        try:
            o2, l2 = rg.attn_fwd(tq, tk, tv)
            g2 = rg.attn_bwd(tq, tk, tv, o2, l2, tg)
            torch.cuda.synchronize()
            res["ok"] = (o2, l2) + tuple(g2)
        except Exception as e:  # reported below, on the main thread
            res["err"] = repr(e)

    t = threading.Thread(target=worker)
    t.start()
    t.join()
    assert "err" not in res, res.get("err")
    for a, b in zip((out, lse) + tuple(grads), res["ok"]):
        assert torch.equal(a, b)


def test_forward_step_under_cuda_graph_capture():
    # The step's five launches (RoPE, self-attention, two cross-attention
    # calls, merge) captured once into a CUDA graph and replayed on new inputs
    # copied into the captured buffers: the same bits as eager calls. (Capture
    # runs each entry point's host work once: argument checks, device binding,
    # descriptor encoding; the descriptors travel in the kernel parameters.)
    B, H, D, grid = 1, 2, 128, (2, 6, 11)
    S = grid[0] * grid[1] * grid[2]
    n_ref, n_ctx = 150, 70

    def inputs():
        q, k, v = (synth.f64_to_bf16_bits(RNG.normal(size=(B, H, S, D))) for _ in range(3))
        kc, vc = (synth.f64_to_bf16_bits(RNG.normal(size=(B, H, n_ref + n_ctx, D))) for _ in range(2))
        return [to_dev(x) for x in (q, k, v, kc[:, :, :n_ref], vc[:, :, :n_ref], kc[:, :, n_ref:], vc[:, :, n_ref:])]

    def step(q, k, v, kr, vr, kx, vx, o):
        rg.rope3d_(q, k, grid)
        rg.attn_fwd(q, k, v, out=o["out"], lse=o["lse"])
        rg.attn_fwd(q, kr, vr, out=o["oa"], lse=o["la"])
        rg.attn_fwd(q, kx, vx, out=o["ob"], lse=o["lb"])
        rg.lse_merge(o["oa"], o["la"], o["ob"], o["lb"], out=o["oc"], lse_out=o["lc"])

    def outs():
        o = {n: torch.empty((B, H, S, D), dtype=torch.bfloat16, device="cuda") for n in ("out", "oa", "ob", "oc")}
        o.update({n: torch.empty((B, H, S), dtype=torch.float32, device="cuda") for n in ("lse", "la", "lb", "lc")})
        return o

    static_in, static_out = inputs(), outs()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                 # warm up off the capture (one-time setup)
        step(*[t.clone() for t in static_in], outs())
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(*static_in, static_out)
    for _ in range(2):
        fresh = inputs()
        for dst, src in zip(static_in, fresh):
            dst.copy_(src)
        graph.replay()
        eager = outs()
        step(*fresh, eager)
        torch.cuda.synchronize()
        for n in static_out:
            assert torch.equal(static_out[n], eager[n]), n
