"""Seeded synthetic inputs for the DiT attention hot path.

This module only *generates data*: a counter-based random stream, normal
variates, the bf16 rounding of those variates, and the per-head RMSNorm that
prepares Q/K before they reach the attention (the DiT applies a QK-norm ahead
of RoPE; it is input preparation here, not part of the kernels under test).
It holds none of the attention, RoPE or merge arithmetic. Both the CUDA path's
tests/bench and the fp64 oracle consume the same bf16 bytes produced here.

Random stream (defined here, independent of torch's and numpy's RNGs):

* splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): state advances by the golden-ratio increment
  0x9E3779B97F4A7C15 and each output is the state passed through the
  variant-13 finaliser (xor-shift 30, multiply 0xBF58476D1CE4E5B9,
  xor-shift 27, multiply 0x94D049BB133111EB, xor-shift 31).
* The state of element i of stream (seed, stream, sub) starts from
  key = mix(seed * 2^40 + stream * 2^32 + sub) and is key + (i + 1) * gamma,
  so any element can be produced without producing the ones before it.
* Uniform u in (0, 1]: ((x >> 11) + 1) * 2^-53.
* Normal pairs by Box-Muller: for pair p with u1 = U(2p), u2 = U(2p+1),
  z(2p) = sqrt(-2 ln u1) cos(2 pi u2), z(2p+1) = sqrt(-2 ln u1) sin(2 pi u2).

Streams: q = 0, k = 1, v = 2, spike-row choice = 3, upstream gradient dO = 4.

The workloads are the latent-token shapes of the ReGenVC decoder's DiT
(Wan2.1-class, head dim 128, latent grid 30 x 52 per latent frame): a 25-frame
window is T = 7 latent frames (S = 10920 tokens), a 77-frame clip is T = 20
(S = 31200 tokens); cross-attention keys are 1560 reference-frame latent
tokens plus 512 conditioning tokens.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_Q, STREAM_K, STREAM_V, STREAM_SPIKE, STREAM_DOUT = 0, 1, 2, 3, 4

_CHUNK = 1 << 16  # normal pairs per chunk (cache-sized temporaries)


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser on a uint64 array, in place (wrapping arithmetic)."""
    t = z >> np.uint64(30)
    z ^= t
    z *= _M1
    np.right_shift(z, np.uint64(27), out=t)
    z ^= t
    z *= _M2
    np.right_shift(z, np.uint64(31), out=t)
    z ^= t
    return z


def stream_key(seed: int, stream: int, sub: int = 0) -> np.uint64:
    """Starting state of stream (seed, stream, sub)."""
    raw = ((seed << 40) + (stream << 32) + sub) & 0xFFFFFFFFFFFFFFFF
    return _mix(np.array([raw], dtype=np.uint64))[0]


def splitmix64(key: np.uint64, start: int, n: int) -> np.ndarray:
    """Outputs start .. start+n-1 of the splitmix64 sequence that begins at key."""
    z = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    z *= GAMMA
    z += np.uint64(key)
    return _mix(z)


def uniform(key: np.uint64, start: int, n: int) -> np.ndarray:
    """Uniform doubles in (0, 1] from outputs start .. start+n-1."""
    x = splitmix64(key, start, n)
    x >>= np.uint64(11)
    x += np.uint64(1)
    u = x.astype(np.float64)
    u *= 2.0 ** -53
    return u


def _normal_into(key: np.uint64, first: int, out: np.ndarray) -> None:
    """Fill out (even length) with normals 2*p .. for pairs starting at `first`."""
    npairs = out.size // 2
    u = uniform(key, 2 * first, 2 * npairs).reshape(npairs, 2)
    r = np.log(u[:, 0])
    r *= -2.0
    np.sqrt(r, out=r)
    ang = u[:, 1]
    ang *= 2.0 * math.pi
    z = out.reshape(npairs, 2)
    np.cos(ang, out=z[:, 0])
    np.sin(ang, out=z[:, 1])
    z[:, 0] *= r
    z[:, 1] *= r


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1))
    return _POOL


_POOL = None


def normal(seed: int, stream: int, n: int, sub: int = 0) -> np.ndarray:
    """n standard normal doubles (Box-Muller over the stream's uniforms)."""
    key = stream_key(seed, stream, sub)
    out = np.empty(n + (n & 1), dtype=np.float64)
    step = 2 * _CHUNK
    list(_pool().map(lambda lo: _normal_into(key, lo // 2, out[lo:lo + step]),
                     range(0, out.size, step)))
    return out[:n]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round doubles to bf16 (round to nearest, ties to even), as uint16 bits.

    Exact: the double is first rounded to fp32 *to odd* (truncate, then set
    the last bit when anything was dropped), and that fp32 is rounded to
    nearest-even bf16; with 16 spare bits the two-step rounding equals one
    correct rounding (Boldo & Melquiond, "Emulation of FMA and correctly
    rounded sums: proved algorithms using rounding to odd", IEEE TC 2008).
    Zeros, infinities and NaN are kept; values in the fp32 subnormal range
    raise, since no generator here produces them.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    flat_x = x.reshape(-1)
    flat_o = out.reshape(-1)
    step = 1 << 18

    def work(lo):
        flat_o[lo:lo + step] = _round_chunk(flat_x[lo:lo + step])

    list(_pool().map(work, range(0, flat_x.size, step)))
    return out


def bf16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to doubles (exact)."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def rmsnorm_rows(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """Per-row RMSNorm over the last axis with unit weight: x / sqrt(mean(x^2) + eps)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps)


def _normal_bf16(seed: int, stream: int, shape, rmsnorm: bool, sub: int = 0) -> np.ndarray:
    """Normals of the given shape, optionally RMSNormed per row, rounded to bf16."""
    n = int(np.prod(shape))
    D = shape[-1]
    key = stream_key(seed, stream, sub)
    out = np.empty(n, dtype=np.uint16)
    rows_per = max(1, (2 * _CHUNK) // D)
    step = rows_per * D                    # whole rows, even (D is even)

    def work(lo):
        hi = min(n, lo + step)
        z = np.empty(hi - lo, dtype=np.float64)
        _normal_into(key, lo // 2, z)
        if rmsnorm:
            z = rmsnorm_rows(z.reshape(-1, D)).reshape(-1)
        out[lo:hi] = _round_chunk(z)

    if D % 2:
        raise ValueError("head dim must be even")
    list(_pool().map(work, range(0, n, step)))
    return out.reshape(shape)


def _round_chunk(xs: np.ndarray) -> np.ndarray:
    """Round-to-odd to fp32, then nearest-even to bf16 (see f64_to_bf16_bits)."""
    a = np.abs(xs)
    if np.any((a < 2.0 ** -126) & (a > 0)):
        raise ValueError("value in the fp32 subnormal range")
    with np.errstate(over="ignore", invalid="ignore"):
        f = xs.astype(np.float32)
    bits = f.view(np.uint32).copy()
    back = np.abs(f.astype(np.float64))
    finite = np.isfinite(xs)
    bits -= ((back > a) & finite).astype(np.uint32)      # rounded away from zero: step back
    bits |= ((back != a) & finite).astype(np.uint32)     # sticky bit
    bits += np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))
    res = (bits >> np.uint32(16)).astype(np.uint16)
    res[np.isnan(xs)] = 0x7FC0
    return res


def spike_rows(seed: int, bh: int, S: int, count: int) -> np.ndarray:
    """Distinct key rows chosen by a seeded Fisher-Yates shuffle (first `count`)."""
    key = stream_key(seed, STREAM_SPIKE, bh)
    perm = np.arange(S, dtype=np.int64)
    draws = splitmix64(key, 0, count)
    for i in range(count):
        j = i + int(draws[i] % np.uint64(S - i))
        perm[i], perm[j] = perm[j], perm[i]
    return np.sort(perm[:count])


@dataclass(frozen=True)
class Workload:
    """One synthetic attention workload in [B, H, S, D] bf16 layout."""
    name: str
    B: int
    H: int
    D: int
    Sq: int
    Skv: int
    seed: int
    grid: tuple | None = None        # latent grid (T, Hh, Ww) when RoPE applies
    rope: bool = False
    rmsnorm: bool = False
    theta: float = 10000.0
    q_mult: float = 1.0              # power of two: exact in bf16
    spike_mult: float = 1.0          # power of two: exact in bf16
    spike_frac: float = 0.0
    merge_split: int = 0             # KV split point for the two-block LSE merge
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs of one forward: QK^T and PV, 2 flops per MAC."""
        return 4.0 * self.B * self.H * self.Sq * self.Skv * self.D

    @property
    def spike_count(self) -> int:
        return int(round(self.spike_frac * self.Skv))


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_s1024", B=1, H=2, D=64, Sq=1024, Skv=1024, seed=0, grid=(1, 32, 32),
                 note="B1 H2 D64, 32x32 latent grid, N(0,1), scale 1/8, no RoPE"),
        Workload("win25_s10920", B=1, H=12, D=128, Sq=10920, Skv=10920, seed=1, grid=(7, 30, 52),
                 rope=True, rmsnorm=True,
                 note="25-frame window, 1.3B-class DiT: RMSNorm Q/K + 3D RoPE 44/42/42"),
        Workload("win77_s31200", B=1, H=40, D=128, Sq=31200, Skv=31200, seed=2, grid=(20, 30, 52),
                 rope=True, rmsnorm=True,
                 note="77-frame clip, 14B-class DiT: RMSNorm Q/K + 3D RoPE 44/42/42"),
        Workload("cross_s31200_kv2072", B=1, H=40, D=128, Sq=31200, Skv=2072, seed=3,
                 note="video tokens -> 1560 reference-frame + 512 conditioning tokens, no RoPE"),
        Workload("stress_s10920", B=2, H=16, D=128, Sq=10920, Skv=10920, seed=4, grid=(7, 30, 52),
                 q_mult=4.0, spike_mult=8.0, spike_frac=0.01, merge_split=5460,
                 note="spiky logits: Q x4, 1% of K rows x8; KV split 2 x 5460 for the merge"),
    ]
}


def make_inputs(w: Workload, seed_offset: int = 0):
    """bf16 bit arrays q [B,H,Sq,D], k and v [B,H,Skv,D] for workload w.

    RMSNorm (when w.rmsnorm) is applied to q and k in fp64 before rounding.
    RoPE is *not* applied here: it is a step of the path under test.
    """
    seed = w.seed + seed_offset
    q = _normal_bf16(seed, STREAM_Q, (w.B, w.H, w.Sq, w.D), w.rmsnorm)
    k = _normal_bf16(seed, STREAM_K, (w.B, w.H, w.Skv, w.D), w.rmsnorm)
    v = _normal_bf16(seed, STREAM_V, (w.B, w.H, w.Skv, w.D), False)
    if w.q_mult != 1.0:
        q = f64_to_bf16_bits(bf16_bits_to_f64(q) * w.q_mult)
    if w.spike_frac > 0:
        kk = k.reshape(w.B * w.H, w.Skv, w.D)
        for bh in range(w.B * w.H):
            rows = spike_rows(seed, bh, w.Skv, w.spike_count)
            kk[bh, rows] = f64_to_bf16_bits(bf16_bits_to_f64(kk[bh, rows]) * w.spike_mult)
    return q, k, v


def make_dout(w: Workload, seed_offset: int = 0):
    """Upstream gradient dO [B,H,Sq,D] for the backward pass: N(0,1) rounded
    to bf16 (a synthetic stand-in for the loss gradient; no dataset here)."""
    return _normal_bf16(w.seed + seed_offset, STREAM_DOUT, (w.B, w.H, w.Sq, w.D), False)
