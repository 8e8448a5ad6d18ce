"""The allocation-free RoPE-fused attention entry point.

regen_attn_fwd_rope3d_noalloc exists for callers that may not allocate device
memory (a plug-in inside an application that owns all device allocations, or
a serving loop where cudaMalloc/cudaFree are off limits). It uses a fixed
scratch array inside the library instead of a caller workspace. These tests
call it through the C ABI twice in a row -- the second call finds the first
call's leftovers in the shared array -- and compare each result with the
workspace entry point's on the same inputs. Kept in a file of its own that
pytest collects last; it also passes alone in a fresh process, where its first
call is the one that looks up the array's device address.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from util import ATOL, LSE_ATOL, RTOL, bits_to_f64, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu


def _with_workspace(dq, dk, dv, grid, theta):
    B, H, S, D = dq.shape
    return rg.attn_fwd_rope3d(dq, dk, dv, grid, theta)


def _no_alloc(dq, dk, dv, grid, theta):
    B, H, S, D = dq.shape
    out = torch.empty_like(dq)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dq.device)
    rg.regen_attn_fwd_rope3d_noalloc(dq, dk, dv, out, lse, B, H, S, S, D, 1.0 / math.sqrt(D), None, *grid, theta)
    return out, lse


def test_no_alloc_matches_workspace_entry_on_two_calls_in_a_row():
    rng = np.random.default_rng(77)
    w25 = synth.WORKLOADS["win25_s10920"]
    cases = [
        (synth.make_inputs(w25), w25.grid, w25.theta),                     # 12 x 10920 x 128: 33.5 MB of scratch
        (tuple(synth.f64_to_bf16_bits(rng.normal(size=(2, 3, 231, 64))) for _ in range(3)), (3, 7, 11), 500.0),
    ]
    for (q, k, v), grid, theta in cases:                                   # two calls in a row
        dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
        out, lse = _no_alloc(dq, dk, dv, grid, theta)
        ref_out, ref_lse = _with_workspace(dq, dk, dv, grid, theta)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(to_bits(dq), q)                      # inputs untouched
        np.testing.assert_array_equal(to_bits(dk), k)
        a, b = bits_to_f64(to_bits(out)), bits_to_f64(to_bits(ref_out))
        assert np.all(np.abs(a - b) <= ATOL + RTOL * np.abs(b))            # the tests' tolerance ...
        la, lb = lse.cpu().numpy(), ref_lse.cpu().numpy()
        assert np.all(np.abs(la - lb) <= LSE_ATOL)
        np.testing.assert_array_equal(to_bits(out), to_bits(ref_out))      # ... and in fact the same bits
        np.testing.assert_array_equal(la, lb)
    assert rg.regen_last_device_error() == (0, 0)


def test_no_alloc_call_leaves_device_memory_unchanged():
    # After a first call in this context (which may load the module and looks
    # up the array's address), a call takes no device memory: the device's
    # free bytes are the same before and after it.
    w25 = synth.WORKLOADS["win25_s10920"]
    q, k, v = synth.make_inputs(w25)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    out, lse = _no_alloc(dq, dk, dv, w25.grid, w25.theta)       # first call: set-up
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    B, H, S, D = dq.shape
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    rg.regen_attn_fwd_rope3d_noalloc(dq, dk, dv, out2, lse2, B, H, S, S, D, 1.0 / math.sqrt(D), None,
                                     *w25.grid, w25.theta)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before
    np.testing.assert_array_equal(to_bits(out2), to_bits(out))
    assert rg.regen_last_device_error() == (0, 0)


def test_no_alloc_rejects_problems_larger_than_its_scratch():
    # 40 heads of 31200 tokens need ~320 MB of rotated K: more than the 64 MiB array
    need = rg.regen_attn_fwd_rope3d_workspace_bytes(1, 40, 20, 30, 52, 128)
    assert need > rg.regen_noalloc_scratch_bytes()
    fake = 0x7F0000000000
    with pytest.raises(rg.RegenError) as e:
        rg.regen_attn_fwd_rope3d_noalloc(fake, fake + (1 << 30), fake + (2 << 30), fake + (3 << 30),
                                         fake + (4 << 30), 1, 40, 31200, 31200, 128, 0.088, None, 20, 30, 52, 1e4)
    assert e.value.status == -2 and "needs" in str(e.value)
