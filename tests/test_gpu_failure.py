"""Failure detection without a GPU fault: a bounded wait that nothing completes
expires, the kernel records REGEN_ERR_TIMEOUT and returns, and the context
stays usable for the next call."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import dit_attention_b200 as rg  # noqa: E402
from dit_attention_b200 import synth  # noqa: E402
from util import check_attention, to_bits, to_dev  # noqa: E402

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_survives():
    assert rg.regen_last_device_error() == (0, 0)
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    rg.regen_selftest_bounded_wait(50_000_000, done)        # 50 ms, on a barrier nobody completes
    torch.cuda.synchronize()
    assert int(done.item()) == 1                             # returned after giving up
    assert rg.regen_last_device_error() == (-5, 10)          # REGEN_ERR_TIMEOUT at the self-test site
    assert rg.regen_last_device_error() == (0, 0)            # the record is cleared
    # the context is still usable: a normal attention call runs and is correct
    rng = np.random.default_rng(3)
    q, k, v = (synth.f64_to_bf16_bits(rng.normal(size=(1, 2, 200, 128))) for _ in range(3))
    out, lse = rg.attn_fwd(to_dev(q), to_dev(k), to_dev(v), 1 / math.sqrt(128))
    torch.cuda.synchronize()
    ref, rl = oracle.attention(q, k, v, 1 / math.sqrt(128))
    check_attention(to_bits(out), lse.cpu().numpy(), ref, rl, "after timeout")
    assert rg.regen_last_device_error() == (0, 0)


def test_bounded_wait_argument_checks():
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(rg.RegenError):
        rg.regen_selftest_bounded_wait(0, done)
    with pytest.raises(rg.RegenError):
        rg.regen_selftest_bounded_wait(10_000_000_000, done)
