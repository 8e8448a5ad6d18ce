"""bench.py's accuracy diagnostic (CPU): the GPU rows of the last timed step
against the oracle's rows on the same bf16 inputs. An output equal to the
oracle's, rounded to bf16, is within the attention contract; a planted error
in one output element or one LSE is reported."""
import numpy as np

import bench
import oracle
from dit_attention_b200 import synth


def _case():
    rng = np.random.default_rng(3)
    B, H, S, D = 1, 2, 64, 32
    q, k, v = (synth.f64_to_bf16_bits(rng.normal(size=(B, H, S, D))) for _ in range(3))
    out, lse = oracle.attention(q, k, v, 0.2)
    snap = dict(q=q, k=k, v=v, out=oracle.f64_to_bf16(out), lse=lse.astype(np.float32), scale=0.2)
    rows = np.array([0, 5, 63, 64, 100, 127])
    ref, ref_lse = oracle.attention(q, k, v, 0.2, rows=rows)
    return snap, dict(rows=rows, out=ref, lse=ref_lse)


def test_accuracy_within_contract():
    snap, kept = _case()
    acc = bench.accuracy(snap, kept)
    assert acc["rows"] == 6 and acc["within_contract"] and not acc["flag_mean_err_over_rms_5e-3"]
    assert acc["mean_err_over_rms"] < 2.0 ** -8 and acc["max_lse_err"] < 1e-6


def test_accuracy_reports_planted_errors():
    snap, kept = _case()
    flat = snap["out"].reshape(-1, 32)
    flat[100, 7] = oracle.f64_to_bf16(np.array([oracle.bf16_to_f64(flat[100:101, 7])[0] + 0.5]))[0]
    acc = bench.accuracy(snap, kept)
    assert not acc["within_contract"] and acc["flag_mean_err_over_rms_5e-3"]
    snap, kept = _case()
    snap["lse"].reshape(-1)[63] += 0.01
    acc = bench.accuracy(snap, kept)
    assert not acc["within_contract"] and acc["max_lse_err"] > 5e-3
