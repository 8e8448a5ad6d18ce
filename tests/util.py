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
    if lse_gpu is None:     # a caller that has no LSE (the autograd glue returns none)
        lse_err = np.zeros(1)
    else:
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
# roundoff u = 2^-8 (bf16 keeps 8 significant bits) per summand, so the error
# of one element behaves like a few u times the RMS of the gradient, and its
# maximum over ~1e6 elements stays below ~10u = 0.04 of the RMS; a relative
# term of 5u = 0.02 covers the large elements. The mean error is the sharper
# signal: about u, bounded by 0.01.
GRAD_ATOL_RMS, GRAD_RTOL, GRAD_MEAN_RMS = 4e-2, 2e-2, 1e-2


def check_grad(got, ref, label="", extra=0.0):
    """Assert |got - ref| <= 0.04 rms(ref) + 0.02 |ref| + extra elementwise and
    mean |got - ref| <= 0.01 rms(ref) + mean(extra); got is bf16 bits or float64.

    extra (scalar or per element): the error inherited through delta, see
    delta_bounds; where the exact gradient is identically zero it is the
    whole allowance."""
    g = bits_to_f64(got) if np.asarray(got).dtype == np.uint16 else np.asarray(got, dtype=np.float64)
    g = g.reshape(ref.shape)
    extra = np.broadcast_to(np.asarray(extra, dtype=np.float64), ref.shape)
    err = np.abs(g - ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    diag = {"max_err_over_rms": float(err.max() / rms) if rms else float(err.max()),
            "mean_err_over_rms": float(err.mean() / rms) if rms else float(err.mean()), "rms_ref": rms,
            "max_err_over_bound": float((err / (GRAD_ATOL_RMS * rms + GRAD_RTOL * np.abs(ref) + extra + 1e-300)).max())}
    assert np.all(np.isfinite(g)), f"{label}: non-finite gradient"
    if rms == 0.0:
        assert np.all(err <= extra), f"{label}: expected zeros up to the delta bound; {diag}"
        return diag
    bad = err > GRAD_ATOL_RMS * rms + GRAD_RTOL * np.abs(ref) + extra
    assert not bad.any(), f"{label}: {int(bad.sum())} of {bad.size} gradients out of tolerance; {diag}"
    assert err.mean() <= GRAD_MEAN_RMS * rms + extra.mean(), f"{label}: mean error {diag}"
    return diag


U_BF16 = 2.0 ** -8   # bf16 unit roundoff: 8 significant bits, round to nearest


def delta_bounds(q, k, v, g, scale, qrows=None, krows=None):
    """Per-element bounds (bq for dq, bk for dk) on the error a backward
    inherits from delta_i = <dO_i, O_i> evaluated with the forward's bf16
    output, as every FlashAttention-style backward does. |O_bf16 - O| is at
    most ~2u sum_j P_ij |v_j| (the forward's rounding of P and of O), and the
    fp32 sums of delta and dP add 2 D 2^-24 of the same magnitude; so with
    A_i = sum_j P_ij |v_j| and c_i = 3u sum_d |dO_id| A_id:
        |d dS_ij| <= P_ij c_i
        |d dq_id| <= |scale| c_i sum_j P_ij |k_jd|,  |d dk_jd| <= |scale| sum_i P_ij c_i |q_id|
    It is small where softmax rows are diffuse and dominates where they are
    nearly one-hot (dP_ij* ~ delta_i: cancellation). Every sum of P above is
    the oracle's own attention (values |v|, |k|) or the dv leg of its backward
    (upstream gradient c_i |q_i|). qrows / krows: the query rows for bq and
    the key rows for bk, the same in every head (all if None)."""
    import oracle
    from dit_attention_b200 import synth
    absbits = lambda x: np.asarray(x, dtype=np.uint16) & np.uint16(0x7FFF)  # noqa: E731  |bf16| exactly
    A, _ = oracle.attention(q, k, absbits(v), scale)
    G = bits_to_f64(g).reshape(A.shape)
    D = A.shape[-1]
    c = (3 * U_BF16 + 2 * D * 2.0 ** -24) * np.sum(np.abs(G) * A, axis=-1)
    if qrows is None:
        Kabs, _ = oracle.attention(q, k, absbits(k), scale)
        bq = abs(scale) * c[..., None] * Kabs
    else:
        Sq = A.shape[-2]
        heads = int(np.prod(A.shape[:-2]))
        qrows = np.asarray(qrows, dtype=np.int64)
        glob = (np.arange(heads, dtype=np.int64)[:, None] * Sq + qrows[None, :]).reshape(-1)
        Kabs, _ = oracle.attention(q, k, absbits(k), scale, rows=glob)
        bq = abs(scale) * c.reshape(heads, Sq)[:, qrows].reshape(A.shape[:-2] + (qrows.size, 1)) * \
            Kabs.reshape(A.shape[:-2] + (qrows.size, D))
    X = synth.f64_to_bf16_bits(c[..., None] * bits_to_f64(absbits(q)).reshape(A.shape) * (1 + 2.0 ** -7))
    if krows is None:
        bk = oracle.attention_bwd(q, k, v, X, scale)[2]
    else:
        bk = oracle.attention_bwd_rows(q, k, v, X, scale, [], krows)[2]
    return bq, abs(scale) * bk


def check_fp8_attention(out_bits, lse_gpu, qd, kd, vd, scale, rows=None, label=""):
    """FP8 attention contract, against the oracle's exact attention of the
    DEQUANTISED inputs qd, kd, vd (fp64, code * block scale).

    The kernel rounds P to E4M3 before P V: p_j (1 + e_j) with |e_j| <= 2^-4,
    errors of different keys independent, so out_d carries an error of standard
    deviation at most sigma_d = 2^-4 / sqrt(3) * sqrt(sum_j p_j^2 v_jd^2), and
    sum_j p_j^2 v_jd^2 = exp(lse2 - 2 lse) out2_d with (out2, lse2) the
    oracle's attention of values v^2 at twice the scale. Asserted: |err| <=
    6 sigma + 2^-8 |ref| (bf16 output) + 1e-5 (keys whose P lands in E4M3's
    subnormals) elementwise, mean |err| <= mean sigma + 2^-8 mean |ref|, and
    |lse - ref| <= 1e-3 (the row sum uses P before rounding)."""
    import oracle
    ref, rl = oracle.attention(qd, kd, vd, scale, rows=rows)
    out2, rl2 = oracle.attention(qd, kd, vd * vd, 2.0 * scale, rows=rows)
    D = ref.shape[-1]
    ref, rl = ref.reshape(-1, D), rl.reshape(-1)
    out2, rl2 = out2.reshape(-1, D), rl2.reshape(-1)
    sigma = 2.0 ** -4 / np.sqrt(3.0) * np.sqrt(np.maximum(out2, 0.0) * np.exp(rl2 - 2.0 * rl)[:, None])
    got = bits_to_f64(out_bits).reshape(-1, D)
    err = np.abs(got - ref)
    allow = 6.0 * sigma + 2.0 ** -8 * np.abs(ref) + 1e-5
    lse_err = np.abs(np.asarray(lse_gpu, dtype=np.float64).reshape(-1) - rl)
    diag = {"max_err_over_sigma": float((err / (sigma + 1e-30)).max()),
            "mean_err_over_mean_sigma": float(err.mean() / max(sigma.mean(), 1e-30)),
            "max_abs_err": float(err.max()), "max_lse_err": float(lse_err.max()),
            "rms_ref": float(np.sqrt(np.mean(ref ** 2)))}
    assert np.all(np.isfinite(got)), f"{label}: non-finite output"
    bad = err > allow
    assert not bad.any(), f"{label}: {int(bad.sum())} of {bad.size} outputs outside 6 sigma; {diag}"
    assert err.mean() <= sigma.mean() + 2.0 ** -8 * np.abs(ref).mean(), f"{label}: mean error {diag}"
    assert lse_err.max() <= LSE_ATOL, f"{label}: lse {diag}"
    return diag


def check_proj(got_bits, ref, label=""):
    """Projection contract: bf16 x bf16 products are exact in fp32, sums in fp32
    (relative ~1e-6 of the sum of |products|), one rounding of the result to
    bf16 (2^-8 relative): |got - ref| <= 2^-8 |ref| + 2e-3 rms(ref)."""
    got = bits_to_f64(got_bits).reshape(ref.shape)
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    diag = {"max_err_over_rms": float(err.max() / rms), "mean_err_over_rms": float(err.mean() / rms), "rms_ref": rms}
    bad = err > 2.0 ** -8 * np.abs(ref) + 2e-3 * rms
    assert np.all(np.isfinite(got)), f"{label}: non-finite"
    assert not bad.any(), f"{label}: {int(bad.sum())} of {bad.size} out of tolerance; {diag}"
    return diag
