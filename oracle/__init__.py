"""fp64 CPU oracle for the DiT attention hot path -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package. The product library
(``dit_attention_b200``) never does, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows); this
module only builds it with gcc on first use and marshals numpy arrays.

Functions (each follows the definition written at its C counterpart):

* ``attention(q, k, v, scale, rows=None)`` -- exact softmax attention and
  natural-log LSE, inputs bf16 bit arrays [B, H, S, D] (or doubles).
* ``attention_bwd(q, k, v, dout, scale)`` -- dQ, dK, dV of exact attention;
  ``attention_bwd_rows`` -- the same for chosen query / key rows only.
* ``lse_merge(o_a, lse_a, o_b, lse_b)`` -- two-block (O, LSE) combination.
* ``rope3d(x, grid, theta)`` -- 3D RoPE, bf16 in/out (rounded to nearest even)
  or fp64 in/out; ``rope3d_bwd`` -- its gradient (the transposed rotation).
* ``f64_to_bf16`` / ``bf16_to_f64`` -- the oracle's own rounding and widening.
* ``qkv_proj`` / ``out_proj`` -- the DiT block's projections around the
  attention (linear layer, per-head RMSNorm and 3D RoPE on q and k).
* ``f64_to_e4m3`` / ``e4m3_to_f64`` / ``quantize_e4m3`` / ``dequantize_e4m3`` --
  OCP E4M3 rounding and the FP8 variant's blockwise quantisation.

Parity status: attention and the LSE merge are pinned by the tests against
brute force, closed forms, invariants and torch's CPU fp64 SDPA. The RoPE
*pairing convention* (interleaved pairs, axis order t/h/w, 44/42/42 split) is a
reading of the Wan2.1 architecture the pages name, not something the pages
print: "parity unpinned" for that convention; the rotation itself is pinned by
norm preservation, relative-offset invariance, the identity at position 0 and
reduction to 1D RoPE.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# Tests that check the pins against deliberately broken copies of oracle.c
# point this at such a copy (tests/test_oracle_mutants.py); nothing else sets it.
_LIB_OVERRIDE = os.environ.get("ORACLE_LIB")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def compile_library(src: str, out: str) -> str:
    """gcc -O2 -ffp-contract=off -fopenmp -shared: the oracle's one build recipe."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC", src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_library(_SRC, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE:
                lib = ctypes.CDLL(_LIB_OVERRIDE)
            else:
                build()
                lib = ctypes.CDLL(_LIB)
            lib.oracle_attention_f64.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64, _i64,
                                                 ctypes.c_double, _i64p, _i64, _dp, _dp]
            lib.oracle_attention_f64.restype = None
            lib.oracle_attention_bf16.argtypes = [_u16p, _u16p, _u16p, _i64, _i64, _i64, _i64,
                                                  ctypes.c_double, _i64p, _i64, _dp, _dp]
            lib.oracle_attention_bf16.restype = ctypes.c_int
            lib.oracle_attention_bwd_f64.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64,
                                                     ctypes.c_double, _dp, _dp, _dp]
            lib.oracle_attention_bwd_f64.restype = ctypes.c_int
            lib.oracle_attention_bwd_bf16.argtypes = [_u16p, _u16p, _u16p, _u16p, _i64, _i64, _i64, _i64,
                                                      ctypes.c_double, _dp, _dp, _dp]
            lib.oracle_attention_bwd_bf16.restype = ctypes.c_int
            lib.oracle_attention_bwd_block_f64.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64,
                                                           ctypes.c_double, _dp, _dp, _dp]
            lib.oracle_attention_bwd_block_f64.restype = None
            lib.oracle_attention_bwd_block_bf16.argtypes = [_u16p, _u16p, _u16p, _u16p, _dp, _u16p, _i64, _i64,
                                                            _i64, _i64, ctypes.c_double, _dp, _dp, _dp]
            lib.oracle_attention_bwd_block_bf16.restype = None
            lib.oracle_attention_bwd_rows_bf16.argtypes = [_u16p, _u16p, _u16p, _u16p, _i64, _i64, _i64, _i64,
                                                           ctypes.c_double, _i64p, _i64, _i64p, _i64, _dp, _dp,
                                                           _dp]
            lib.oracle_attention_bwd_rows_bf16.restype = ctypes.c_int
            lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_to_f64.restype = ctypes.c_double
            lib.oracle_f64_to_e4m3_array.argtypes = [_dp, ctypes.POINTER(ctypes.c_uint8), _i64]
            lib.oracle_f64_to_e4m3_array.restype = None
            lib.oracle_quantize_e4m3.argtypes = [_u16p, _i64, _i64, _i64, _i64, ctypes.POINTER(ctypes.c_uint8),
                                                 ctypes.POINTER(ctypes.c_float)]
            lib.oracle_quantize_e4m3.restype = ctypes.c_int
            lib.oracle_qkv_proj_rows.argtypes = [_u16p, _u16p, _dp, _dp, _dp] + [_i64] * 8 + [
                ctypes.c_double, ctypes.c_double, _i64p, _i64, _dp, _dp, _dp]
            lib.oracle_qkv_proj_rows.restype = ctypes.c_int
            lib.oracle_out_proj_rows.argtypes = [_u16p, _u16p, _dp] + [_i64] * 5 + [_i64p, _i64, _dp]
            lib.oracle_out_proj_rows.restype = ctypes.c_int
            lib.oracle_lse_merge_f64.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _dp, _dp]
            lib.oracle_lse_merge_f64.restype = None
            lib.oracle_rope3d_f64.argtypes = [_dp, _i64, _i64, _i64, _i64, _i64, ctypes.c_double]
            lib.oracle_rope3d_f64.restype = ctypes.c_int
            lib.oracle_rope3d_bf16.argtypes = [_u16p, _i64, _i64, _i64, _i64, _i64, ctypes.c_double]
            lib.oracle_rope3d_bf16.restype = ctypes.c_int
            lib.oracle_rope3d_bwd_f64.argtypes = [_dp, _i64, _i64, _i64, _i64, _i64, ctypes.c_double]
            lib.oracle_rope3d_bwd_f64.restype = ctypes.c_int
            lib.oracle_rope3d_bwd_bf16.argtypes = [_u16p, _i64, _i64, _i64, _i64, _i64, ctypes.c_double]
            lib.oracle_rope3d_bwd_bf16.restype = ctypes.c_int
            lib.oracle_f64_to_bf16_array.argtypes = [_dp, _u16p, _i64]
            lib.oracle_f64_to_bf16_array.restype = None
            lib.oracle_bf16_to_f64_array.argtypes = [_u16p, _dp, _i64]
            lib.oracle_bf16_to_f64_array.restype = None
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
            lib.oracle_set_num_threads.restype = None
            _lib = lib
    return _lib


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def f64_to_bf16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f64_to_bf16_array(_ptr(x, _dp), _ptr(out, _u16p), x.size)
    return out


def bf16_to_f64(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float64)
    _load().oracle_bf16_to_f64_array(_ptr(h, _u16p), _ptr(out, _dp), h.size)
    return out


def attention(q, k, v, scale: float, rows=None):
    """Exact attention. q [..., Sq, D], k/v [..., Skv, D] with equal leading dims.

    Arrays of dtype uint16 are bf16 bit patterns; float64 arrays are used as
    they are. Returns (out fp64, lse fp64): with rows=None, out has q's shape
    and lse q's shape without D; with rows (global indices bh*Sq + i) the
    results are [len(rows), D] and [len(rows)].
    """
    lib = _load()
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    Sq, D = q.shape[-2], q.shape[-1]
    Skv = k.shape[-2]
    lead = q.shape[:-2]
    if k.shape[:-2] != lead or v.shape != k.shape or k.shape[-1] != D:
        raise ValueError("q, k, v shapes do not agree")
    BH = int(np.prod(lead)) if lead else 1
    if rows is None:
        n = BH * Sq
        rp = None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        if rows.size and (rows.min() < 0 or rows.max() >= BH * Sq):
            raise ValueError("row index out of range")
        n = rows.size
        rp = _ptr(rows, _i64p)
    out = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    kinds = {q.dtype, k.dtype, v.dtype}
    if kinds == {np.dtype(np.uint16)}:
        rc = lib.oracle_attention_bf16(_ptr(q, _u16p), _ptr(k, _u16p), _ptr(v, _u16p),
                                       BH, Sq, Skv, D, float(scale), rp, n,
                                       _ptr(out, _dp), _ptr(lse, _dp))
        if rc != 0:
            raise MemoryError("oracle could not allocate its fp64 copies")
    elif kinds == {np.dtype(np.float64)}:
        lib.oracle_attention_f64(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp),
                                 BH, Sq, Skv, D, float(scale), rp, n,
                                 _ptr(out, _dp), _ptr(lse, _dp))
    else:
        raise TypeError("inputs must all be uint16 (bf16 bits) or all float64")
    if rows is None:
        return out.reshape(q.shape), lse.reshape(q.shape[:-1])
    return out, lse


def attention_bwd(q, k, v, dout, scale: float):
    """Gradients (dq, dk, dv) in fp64 of exact attention for upstream dout.

    q, dout [..., Sq, D]; k, v [..., Skv, D]; all uint16 (bf16 bits) or all float64.
    """
    lib = _load()
    q, k, v, dout = (np.ascontiguousarray(a) for a in (q, k, v, dout))
    Sq, D = q.shape[-2], q.shape[-1]
    Skv = k.shape[-2]
    lead = q.shape[:-2]
    if k.shape[:-2] != lead or v.shape != k.shape or dout.shape != q.shape or k.shape[-1] != D:
        raise ValueError("q, k, v, dout shapes do not agree")
    BH = int(np.prod(lead)) if lead else 1
    dq = np.empty(q.shape, dtype=np.float64)
    dk = np.empty(k.shape, dtype=np.float64)
    dv = np.empty(k.shape, dtype=np.float64)
    kinds = {a.dtype for a in (q, k, v, dout)}
    if kinds == {np.dtype(np.uint16)}:
        rc = lib.oracle_attention_bwd_bf16(*(_ptr(a, _u16p) for a in (q, k, v, dout)), BH, Sq, Skv, D,
                                           float(scale), _ptr(dq, _dp), _ptr(dk, _dp), _ptr(dv, _dp))
    elif kinds == {np.dtype(np.float64)}:
        rc = lib.oracle_attention_bwd_f64(*(_ptr(a, _dp) for a in (q, k, v, dout)), BH, Sq, Skv, D,
                                          float(scale), _ptr(dq, _dp), _ptr(dk, _dp), _ptr(dv, _dp))
    else:
        raise TypeError("inputs must all be uint16 (bf16 bits) or all float64")
    if rc != 0:
        raise MemoryError("oracle could not allocate its per-head P and dS")
    return dq, dk, dv


def attention_bwd_block(q, k, v, out, lse, dout, scale: float):
    """The gradients contributed by one block of keys, given the whole
    attention's out and lse: (dq share, dk, dv) in fp64.

    q, out, dout [..., Sq, D]; k, v [..., Skv, D] -- all uint16 (bf16 bits) or
    all float64; lse [..., Sq] (float64)."""
    lib = _load()
    q, k, v, out, dout = (np.ascontiguousarray(a) for a in (q, k, v, out, dout))
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    Sq, D = q.shape[-2], q.shape[-1]
    Skv = k.shape[-2]
    lead = q.shape[:-2]
    if (k.shape[:-2] != lead or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape
            or k.shape[-1] != D or lse.shape != q.shape[:-1]):
        raise ValueError("q, k, v, out, lse, dout shapes do not agree")
    BH = int(np.prod(lead)) if lead else 1
    dq = np.empty(q.shape, dtype=np.float64)
    dk = np.empty(k.shape, dtype=np.float64)
    dv = np.empty(k.shape, dtype=np.float64)
    kinds = {a.dtype for a in (q, k, v, out, dout)}
    if kinds == {np.dtype(np.uint16)}:
        lib.oracle_attention_bwd_block_bf16(*(_ptr(a, _u16p) for a in (q, k, v, out)), _ptr(lse, _dp),
                                            _ptr(dout, _u16p), BH, Sq, Skv, D, float(scale),
                                            _ptr(dq, _dp), _ptr(dk, _dp), _ptr(dv, _dp))
    elif kinds == {np.dtype(np.float64)}:
        lib.oracle_attention_bwd_block_f64(*(_ptr(a, _dp) for a in (q, k, v, out, lse, dout)), BH, Sq, Skv, D,
                                           float(scale), _ptr(dq, _dp), _ptr(dk, _dp), _ptr(dv, _dp))
    else:
        raise TypeError("q, k, v, out, dout must all be uint16 (bf16 bits) or all float64")
    return dq, dk, dv


def attention_bwd_rows(q, k, v, dout, scale: float, qrows, krows):
    """The gradients for chosen rows of every head: dq[..., len(qrows), D] for
    those query rows, dk, dv[..., len(krows), D] for those key rows (fp64).

    Inputs as ``attention_bwd`` but bf16 bits only; for sizes where the full
    gradient would take too long (every query row's statistics are still
    computed, once per head).
    """
    lib = _load()
    q, k, v, dout = (np.ascontiguousarray(a) for a in (q, k, v, dout))
    if {a.dtype for a in (q, k, v, dout)} != {np.dtype(np.uint16)}:
        raise TypeError("inputs must be uint16 (bf16 bits)")
    Sq, D = q.shape[-2], q.shape[-1]
    Skv = k.shape[-2]
    lead = q.shape[:-2]
    if k.shape[:-2] != lead or v.shape != k.shape or dout.shape != q.shape or k.shape[-1] != D:
        raise ValueError("q, k, v, dout shapes do not agree")
    BH = int(np.prod(lead)) if lead else 1
    qr = np.ascontiguousarray(qrows, dtype=np.int64)
    kr = np.ascontiguousarray(krows, dtype=np.int64)
    if qr.size and (qr.min() < 0 or qr.max() >= Sq) or kr.size and (kr.min() < 0 or kr.max() >= Skv):
        raise IndexError("row index out of range")
    dq = np.empty(lead + (qr.size, D), dtype=np.float64)
    dk = np.empty(lead + (kr.size, D), dtype=np.float64)
    dv = np.empty(lead + (kr.size, D), dtype=np.float64)
    rc = lib.oracle_attention_bwd_rows_bf16(*(_ptr(a, _u16p) for a in (q, k, v, dout)), BH, Sq, Skv, D,
                                            float(scale), _ptr(qr, _i64p), qr.size, _ptr(kr, _i64p), kr.size,
                                            _ptr(dq, _dp), _ptr(dk, _dp), _ptr(dv, _dp))
    if rc != 0:
        raise MemoryError("oracle could not allocate its row statistics")
    return dq, dk, dv


def e4m3_to_f64(codes):
    """Decode OCP E4M3 codes (uint8 array) to doubles (exact)."""
    lib = _load()
    table = np.array([lib.oracle_e4m3_to_f64(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def f64_to_e4m3(x):
    """Round doubles to E4M3 codes: nearest, ties to even, saturating at +-448."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint8)
    lib.oracle_f64_to_e4m3_array(_ptr(x, _dp), out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), x.size)
    return out


def quantize_e4m3(x, block_rows: int = 128):
    """Blockwise E4M3 quantisation of bf16 bits x [..., S, D] (see oracle.c):
    returns (codes uint8 [..., S, D], scales float32 [..., ceil(S/block_rows)])."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    S, D = x.shape[-2], x.shape[-1]
    lead = x.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1
    nb = -(-S // block_rows)
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty(lead + (nb,), dtype=np.float32)
    rc = lib.oracle_quantize_e4m3(_ptr(x, _u16p), BH, S, D, block_rows,
                                  codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                  scales.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    if rc != 0:
        raise ValueError("block_rows must be positive")
    return codes, scales


def dequantize_e4m3(codes, scales, block_rows: int = 128):
    """code * scale of its block, in fp64 (exact): the values the FP8 path represents."""
    v = e4m3_to_f64(codes)
    S = v.shape[-2]
    rep = np.repeat(np.asarray(scales, dtype=np.float64), block_rows, axis=-1)[..., :S]
    return v * rep[..., None]


def _opt_f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def qkv_proj(x, w, bias, gamma_q, gamma_k, heads: int, grid, theta: float = 10000.0, eps: float = 1e-6,
             rows=None):
    """QKV projection of the DiT block for token rows of x [B, S, C] (bf16 bits):
    y = x W^T + b, split into q | k | v of `heads` heads; per-head RMSNorm
    (weights gamma_q / gamma_k [H*D], None = 1) and 3D RoPE on q and k.
    w [3*H*D, C] bf16 bits; bias [3*H*D] float or None. rows: global token ids
    b*S + s (all if None). Returns q, k, v [len(rows), H, D] in fp64."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint16)
    B, S, C = x.shape
    N = w.shape[0]
    H = int(heads)
    D = N // (3 * H)
    if w.shape != (3 * H * D, C) or 3 * H * D != N:
        raise ValueError("w must be [3*H*D, C]")
    T, Hh, Ww = (int(g) for g in grid)
    r = np.arange(B * S, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    q = np.empty((r.size, H, D)); k = np.empty_like(q); v = np.empty_like(q)
    b, gq, gk = _opt_f64(bias), _opt_f64(gamma_q), _opt_f64(gamma_k)
    rc = lib.oracle_qkv_proj_rows(_ptr(x, _u16p), _ptr(w, _u16p), _ptr(b, _dp) if b is not None else None,
                                  _ptr(gq, _dp) if gq is not None else None, _ptr(gk, _dp) if gk is not None else None,
                                  B, S, C, H, D, T, Hh, Ww, float(theta), float(eps), _ptr(r, _i64p), r.size,
                                  _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp))
    if rc != 0:
        raise ValueError("bad sizes or row ids")
    return q, k, v


def out_proj(o, w, bias, rows=None):
    """Output projection y = o W^T + b for token rows, o the attention output
    [B, H, S, D] (bf16 bits) with heads concatenated per token; w [N, H*D].
    Returns y [len(rows), N] in fp64 (rows: global token ids, all if None)."""
    lib = _load()
    o = np.ascontiguousarray(o, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint16)
    B, H, S, D = o.shape
    N = w.shape[0]
    if w.shape[1] != H * D:
        raise ValueError("w must be [N, H*D]")
    r = np.arange(B * S, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((r.size, N))
    b = _opt_f64(bias)
    rc = lib.oracle_out_proj_rows(_ptr(o, _u16p), _ptr(w, _u16p), _ptr(b, _dp) if b is not None else None,
                                  B, S, H, D, N, _ptr(r, _i64p), r.size, _ptr(y, _dp))
    if rc != 0:
        raise ValueError("bad row ids")
    return y


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Two-block merge. o_* [..., D] (bf16 bits or float64), lse_* [...]."""
    lib = _load()

    def as64(a):
        a = np.ascontiguousarray(a)
        return bf16_to_f64(a) if a.dtype == np.uint16 else np.ascontiguousarray(a, dtype=np.float64)

    oa, ob = as64(o_a), as64(o_b)
    la = np.ascontiguousarray(lse_a, dtype=np.float64)
    lb = np.ascontiguousarray(lse_b, dtype=np.float64)
    D = oa.shape[-1]
    rows = oa.size // D if D else 0
    if ob.shape != oa.shape or la.size != rows or lb.size != rows:
        raise ValueError("merge shapes do not agree")
    out = np.empty(oa.shape, dtype=np.float64)
    lse = np.empty(la.shape, dtype=np.float64)
    lib.oracle_lse_merge_f64(_ptr(oa, _dp), _ptr(la, _dp), _ptr(ob, _dp), _ptr(lb, _dp),
                             rows, D, _ptr(out, _dp), _ptr(lse, _dp))
    return out, lse


def rope3d(x, grid, theta: float = 10000.0):
    """3D RoPE of x [..., S, D], S = T*Hh*Ww. Returns a new array.

    uint16 input (bf16 bits) -> uint16 output rounded to nearest even;
    float64 input -> float64 output (no rounding).
    """
    return _rope3d(x, grid, theta, False)


def rope3d_bwd(g, grid, theta: float = 10000.0):
    """Gradient of rope3d: R^T g, every pair turned back by its angle.

    Same dtypes and rounding as ``rope3d``.
    """
    return _rope3d(g, grid, theta, True)


def _rope3d(x, grid, theta, transpose):
    lib = _load()
    T, Hh, Ww = (int(g) for g in grid)
    x = np.array(x, copy=True, order="C")
    S, D = x.shape[-2], x.shape[-1]
    if S != T * Hh * Ww:
        raise ValueError("sequence length does not match the latent grid")
    BH = x.size // (S * D) if S * D else 0
    if x.dtype == np.uint16:
        fn = lib.oracle_rope3d_bwd_bf16 if transpose else lib.oracle_rope3d_bf16
        rc = fn(_ptr(x, _u16p), BH, T, Hh, Ww, D, float(theta))
    elif x.dtype == np.float64:
        fn = lib.oracle_rope3d_bwd_f64 if transpose else lib.oracle_rope3d_f64
        rc = fn(_ptr(x, _dp), BH, T, Hh, Ww, D, float(theta))
    else:
        raise TypeError("x must be uint16 (bf16 bits) or float64")
    if rc != 0:
        raise ValueError("rope3d needs an even head dim >= 6")
    return x
