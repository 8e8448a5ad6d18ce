"""Helpers shared by the GPU parity tests (marshalling only; no method arithmetic)."""
import numpy as np

ATOL, RTOL, LSE_ATOL = 1e-2, 1e-2, 1e-3   # the accuracy contract for bf16 outputs / fp32 LSE


def to_dev(bits: np.ndarray):
    """uint16 bf16 bit array -> CUDA bf16 tensor (same bytes)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def to_bits(t) -> np.ndarray:
    """CUDA bf16 tensor -> uint16 bit array."""
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sample_rows(BH: int, Sq: int, per_head: int, seed: int = 0) -> np.ndarray:
    """Global row ids bh*Sq + i: every head's first and last 4 rows, the rows of
    its last (ragged) 128-row tile boundary, plus `per_head` random rows."""
    rng = np.random.default_rng(seed)
    rows = []
    last_tile = (Sq - 1) // 128 * 128
    for bh in range(BH):
        fixed = {0, 1, 2, 3, Sq - 4, Sq - 3, Sq - 2, Sq - 1, last_tile, min(Sq - 1, 127), min(Sq - 1, 128),
                 min(Sq - 1, 255), min(Sq - 1, 256)}
        fixed = {r for r in fixed if 0 <= r < Sq}
        rnd = rng.choice(Sq, size=min(per_head, Sq), replace=False)
        for r in sorted(fixed | set(rnd.tolist())):
            rows.append(bh * Sq + r)
    return np.array(rows, dtype=np.int64)


def check_attention(out_bits, lse_gpu, ref_out, ref_lse, label=""):
    """Assert the contract |out - ref| <= atol + rtol|ref| and |lse - ref| <= 1e-3,
    plus a tighter error-budget check relative to RMS(ref) (bf16 rounding of P
    and of out gives ~0.3% of RMS; 5% flags a real defect). Returns diagnostics."""
    out = bits_to_f64(out_bits).reshape(ref_out.shape)
    err = np.abs(out - ref_out)
    bound = ATOL + RTOL * np.abs(ref_out)
    bad = err > bound
    lse_err = np.abs(np.asarray(lse_gpu, dtype=np.float64).reshape(ref_lse.shape) - ref_lse)
    rms = float(np.sqrt(np.mean(ref_out ** 2))) or 1.0
    diag = {"max_abs_err": float(err.max()), "max_err_over_rms": float(err.max() / rms),
            "max_lse_err": float(lse_err.max()), "rms_ref": rms}
    assert not bad.any(), f"{label}: {int(bad.sum())} outputs out of tolerance; {diag}"
    assert np.all(np.isfinite(lse_err)) and lse_err.max() <= LSE_ATOL, f"{label}: lse {diag}"
    assert diag["max_err_over_rms"] < 0.05, f"{label}: error budget {diag}"
    return diag


# Gradient contract. dV sums P rounded to bf16; dK and dQ sum dS rounded to
# bf16, whose delta term uses the forward's bf16 output; each result is
# rounded once more. That is a handful of independent roundings of unit
# roundoff u = 2^-9 per summand, so the error of one element behaves like a
# few u times the RMS of the gradient, and its maximum over ~1e6 elements stays
# below ~20u = 0.04 of the RMS; a relative term of 10u = 0.02 covers the large
# elements. The mean error is the sharper signal: a few u, bounded by 0.01.
GRAD_ATOL_RMS, GRAD_RTOL, GRAD_MEAN_RMS = 4e-2, 2e-2, 1e-2


def check_grad(got, ref, label=""):
    """Assert |got - ref| <= 0.04 rms(ref) + 0.02 |ref| elementwise and
    mean |got - ref| <= 0.01 rms(ref); got is bf16 bits or float64."""
    g = bits_to_f64(got) if np.asarray(got).dtype == np.uint16 else np.asarray(got, dtype=np.float64)
    g = g.reshape(ref.shape)
    err = np.abs(g - ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    diag = {"max_err_over_rms": float(err.max() / rms) if rms else float(err.max()),
            "mean_err_over_rms": float(err.mean() / rms) if rms else float(err.mean()), "rms_ref": rms}
    assert np.all(np.isfinite(g)), f"{label}: non-finite gradient"
    if rms == 0.0:
        assert err.max() == 0.0, f"{label}: expected exact zeros; {diag}"
        return diag
    bad = err > GRAD_ATOL_RMS * rms + GRAD_RTOL * np.abs(ref)
    assert not bad.any(), f"{label}: {int(bad.sum())} of {bad.size} gradients out of tolerance; {diag}"
    assert diag["mean_err_over_rms"] <= GRAD_MEAN_RMS, f"{label}: mean error {diag}"
    return diag
