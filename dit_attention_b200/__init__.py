"""DiT attention hot path for NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libregen_attn.so`` (C ABI in include/regen_attn.h).
Every computation runs in the library's CUDA kernels; this module only
marshals torch tensors (or raw integer device pointers) into the C calls and
raises ``RegenError`` on a non-zero status. There is no CPU fallback: if the
library is missing or fails to load, every entry point raises.

Entry points (same names as the C ABI):
    regen_attn_fwd(q, k, v, out, lse, B, H, Sq, Skv, D, scale, stream=None)
    regen_rope3d(q, k, T, Hh, Ww, theta, B, H, D, stream=None)
    regen_attn_fwd_rope3d(q, k, v, out, lse, B, H, Sq, Skv, D, scale, stream, T, Hh, Ww, theta,
                          workspace, workspace_bytes)
    regen_attn_fwd_rope3d_workspace_bytes(B, H, T, Hh, Ww, D)
    regen_lse_merge(o_a, lse_a, o_b, lse_b, out, lse_out, rows, D, stream=None)
    regen_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, Sq, Skv, D, scale, stream,
                   workspace, workspace_bytes, accumulate)   # REGEN_ACCUM_DQ | REGEN_ACCUM_DKDV
    regen_attn_bwd_workspace_bytes(B, H, Sq, D)
    regen_attn_bwd_kv2(q, k_a, v_a, k_b, v_b, out, lse, dout, dq, dk_a, dv_a, dk_b, dv_b, B, H, Sq,
                       Skv_a, Skv_b, D, scale, stream, workspace, workspace_bytes, accumulate)
    regen_rope3d_bwd(dq, dk, T, Hh, Ww, theta, B, H, D, stream=None)
    regen_rope3d_shard(q, k, T, Hh, Ww, theta, B, H, D, n0, S_local, inverse=0, stream=None)
    regen_quant_e4m3(x, codes, scales, B, H, S, D, stream=None)
    regen_attn_fwd_fp8(q8, q_scale, k8, k_scale, v8, v_scale, out, lse, B, H, Sq, Skv, D, scale, stream=None)
    regen_qkv_proj(x, w, bias, gamma_q, gamma_k, q, k, v, B, S, C, H, D, T, Hh, Ww, theta, eps, stream,
                   workspace, workspace_bytes);  regen_qkv_proj_workspace_bytes(T, Hh, Ww, D)
    regen_out_proj(o, w, bias, y, B, S, H, D, N, stream=None)
    regen_last_device_error() -> (status, site)
    regen_last_cuda_error() -> (code, name)   (behind this thread's last REGEN_ERR_CUDA)
    regen_set_wait_limit_ns(ns)
Convenience wrappers that allocate outputs with torch:
    attn_fwd(q, k, v, scale=None) -> (out, lse)
    attn_fwd_rope3d(q, k, v, grid, theta=10000.0) -> (out, lse)
    rope3d_(q, k, grid, theta=10000.0)
    lse_merge(o_a, lse_a, o_b, lse_b) -> (out, lse)
    attn_bwd(q, k, v, out, lse, dout, scale=None) -> (dq, dk, dv)
    attn_bwd_kv2(q, k_a, v_a, k_b, v_b, out, lse, dout, scale=None) -> (dq, dk_a, dv_a, dk_b, dv_b)
    rope3d_bwd_(dq, dk, grid, theta=10000.0)
    quant_e4m3(x) -> (codes, scales);  attn_fwd_fp8(q8, qs, k8, ks, v8, vs, scale=None) -> (out, lse)
    qkv_proj(x, w, heads, grid, bias=None, gamma_q=None, gamma_k=None) -> (q, k, v)
    out_proj(o, w, bias=None) -> y
Differentiable forms for training (torch.autograd over the same kernels):
    dit_attention_b200.autograd.dit_attention, dit_cross_attention
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

__all__ = [
    "RegenError", "library_path", "load", "regen_attn_fwd", "regen_rope3d", "regen_lse_merge",
    "regen_status_str", "regen_last_device_error", "regen_last_cuda_error", "regen_selftest_exp2", "regen_selftest_bounded_wait", "regen_set_wait_limit_ns", "regen_version",
    "regen_attn_fwd_rope3d", "regen_attn_fwd_rope3d_workspace_bytes", "regen_attn_fwd_rope3d_noalloc",
    "regen_noalloc_scratch_bytes",
    "regen_attn_bwd", "regen_attn_bwd_workspace_bytes", "regen_attn_bwd_kv2", "attn_bwd_kv2", "regen_rope3d_bwd", "regen_rope3d_shard", "regen_quant_e4m3",
    "regen_attn_fwd_fp8", "quant_e4m3", "attn_fwd_fp8", "regen_qkv_proj", "regen_qkv_proj_workspace_bytes",
    "regen_out_proj", "qkv_proj", "out_proj",
    "attn_fwd", "attn_fwd_kv2", "regen_attn_fwd_kv2", "attn_fwd_rope3d", "rope3d_", "lse_merge", "attn_bwd", "rope3d_bwd_", "STATUS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libregen_attn.so")
_lock = threading.Lock()
_lib = None

STATUS = {0: "REGEN_OK", -1: "REGEN_ERR_INVALID_ARG", -2: "REGEN_ERR_UNSUPPORTED",
          -3: "REGEN_ERR_MISALIGNED", -4: "REGEN_ERR_CUDA", -5: "REGEN_ERR_TIMEOUT"}


# regen_attn_bwd's accumulate bits (include/regen_attn.h)
REGEN_ACCUM_DQ = 1
REGEN_ACCUM_DKDV = 2

class RegenError(RuntimeError):
    def __init__(self, status: int, what: str, cuda_error=None):
        self.status = status
        self.cuda_error = cuda_error    # (code, name) behind a REGEN_ERR_CUDA, when known
        detail = f"; CUDA {cuda_error[1]} ({cuda_error[0]})" if cuda_error else ""
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_status_text(status)}){detail}")


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libregen_attn.so (raises if it is not built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is not built; run `python -m dit_attention_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        L.regen_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp]
        L.regen_attn_fwd.restype = i32
        L.regen_attn_fwd_kv2.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp]
        L.regen_attn_fwd_kv2.restype = i32
        L.regen_attn_fwd_rope3d.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp,
                                            i32, i32, i32, f32, vp, i64]
        L.regen_attn_fwd_rope3d.restype = i32
        L.regen_attn_fwd_rope3d_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp,
                                                    i32, i32, i32, f32]
        L.regen_attn_fwd_rope3d_noalloc.restype = i32
        L.regen_noalloc_scratch_bytes.argtypes = []
        L.regen_noalloc_scratch_bytes.restype = i64
        L.regen_attn_fwd_rope3d_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
        L.regen_attn_fwd_rope3d_workspace_bytes.restype = i64
        L.regen_rope3d.argtypes = [vp, vp, i32, i32, i32, f32, i32, i32, i32, vp]
        L.regen_rope3d.restype = i32
        L.regen_lse_merge.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, vp]
        L.regen_lse_merge.restype = i32
        L.regen_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp,
                                     vp, i64, i32]
        L.regen_attn_bwd.restype = i32
        L.regen_attn_bwd_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.regen_attn_bwd_workspace_bytes.restype = i64
        L.regen_attn_bwd_kv2.argtypes = [vp] * 13 + [i32] * 6 + [f32, vp, vp, i64, i32]
        L.regen_attn_bwd_kv2.restype = i32
        L.regen_rope3d_bwd.argtypes = [vp, vp, i32, i32, i32, f32, i32, i32, i32, vp]
        L.regen_rope3d_bwd.restype = i32
        L.regen_rope3d_shard.argtypes = [vp, vp, i32, i32, i32, f32, i32, i32, i32, i32, i32, i32, vp]
        L.regen_rope3d_shard.restype = i32
        L.regen_quant_e4m3.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
        L.regen_quant_e4m3.restype = i32
        L.regen_attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp]
        L.regen_attn_fwd_fp8.restype = i32
        L.regen_qkv_proj.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp] + [i32] * 8 + [f32, f32, vp, vp, i64]
        L.regen_qkv_proj.restype = i32
        L.regen_qkv_proj_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.regen_qkv_proj_workspace_bytes.restype = i64
        L.regen_out_proj.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]
        L.regen_out_proj.restype = i32
        L.regen_status_str.argtypes = [i32]
        L.regen_status_str.restype = ctypes.c_char_p
        L.regen_last_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
        L.regen_last_device_error.restype = i32
        L.regen_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.regen_set_wait_limit_ns.restype = i32
        L.regen_selftest_exp2.argtypes = [vp, vp, i64, vp]
        L.regen_selftest_exp2.restype = i32
        L.regen_selftest_bounded_wait.argtypes = [ctypes.c_uint64, vp, vp]
        L.regen_selftest_bounded_wait.restype = i32
        L.regen_last_cuda_error.argtypes = [ctypes.POINTER(ctypes.c_char_p)]
        L.regen_last_cuda_error.restype = i32
        L.regen_version.argtypes = []
        L.regen_version.restype = i32
        _lib = L
        return _lib


def _status_text(status: int) -> str:
    try:
        return load().regen_status_str(status).decode()
    except Exception:  # the library itself failed to load
        return "?"


def _ptr(x):
    """Device address of a tensor (or an integer address, or None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str) -> None:
    if rc != 0:
        cuda = regen_last_cuda_error() if rc == -4 else None   # REGEN_ERR_CUDA
        raise RegenError(rc, what, cuda)


# ------------------------------------------------------------- C names ---

def regen_attn_fwd(q, k, v, out, lse, B, H, Sq, Skv, D, scale, stream=None) -> None:
    _check(load().regen_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Sq, Skv, D,
                                 float(scale), _stream(stream)), "regen_attn_fwd")


def regen_attn_fwd_kv2(q, k_a, v_a, k_b, v_b, out, lse, B, H, Sq, Skv_a, Skv_b, D, scale, stream=None) -> None:
    _check(load().regen_attn_fwd_kv2(_ptr(q), _ptr(k_a), _ptr(v_a), _ptr(k_b), _ptr(v_b), _ptr(out), _ptr(lse),
                                     B, H, Sq, Skv_a, Skv_b, D, float(scale), _stream(stream)),
           "regen_attn_fwd_kv2")


def regen_attn_fwd_rope3d(q, k, v, out, lse, B, H, Sq, Skv, D, scale, stream, T, Hh, Ww, theta,
                          workspace, workspace_bytes) -> None:
    _check(load().regen_attn_fwd_rope3d(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Sq, Skv, D,
                                        float(scale), _stream(stream), T, Hh, Ww, float(theta), _ptr(workspace),
                                        int(workspace_bytes)), "regen_attn_fwd_rope3d")


def regen_noalloc_scratch_bytes() -> int:
    """Size of the fixed scratch array built into the library."""
    return int(load().regen_noalloc_scratch_bytes())


def regen_attn_fwd_rope3d_noalloc(q, k, v, out, lse, B, H, Sq, Skv, D, scale, stream, T, Hh, Ww, theta) -> None:
    """The RoPE-fused attention with the library's fixed scratch instead of a
    caller workspace: for callers that may not allocate device memory."""
    rc = load().regen_attn_fwd_rope3d_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Sq, Skv, D,
                                              float(scale), _stream(stream), T, Hh, Ww, float(theta))
    if rc == -2 and D in (64, 128) and T > 0 and Hh > 0 and Ww > 0:
        need = load().regen_attn_fwd_rope3d_workspace_bytes(B, H, T, Hh, Ww, D)
        have = regen_noalloc_scratch_bytes()
        if need > have:
            raise RegenError(rc, f"regen_attn_fwd_rope3d_noalloc: needs {need} bytes of scratch, "
                                 f"the fixed array holds {have}")
    _check(rc, "regen_attn_fwd_rope3d_noalloc")


def regen_attn_fwd_rope3d_workspace_bytes(B, H, T, Hh, Ww, D) -> int:
    n = load().regen_attn_fwd_rope3d_workspace_bytes(B, H, T, Hh, Ww, D)
    if n < 0:
        raise RegenError(int(n), "regen_attn_fwd_rope3d_workspace_bytes")
    return int(n)


def regen_rope3d(q, k, T, Hh, Ww, theta, B, H, D, stream=None) -> None:
    _check(load().regen_rope3d(_ptr(q), _ptr(k), T, Hh, Ww, float(theta), B, H, D, _stream(stream)),
           "regen_rope3d")


def regen_lse_merge(o_a, lse_a, o_b, lse_b, out, lse_out, rows, D, stream=None) -> None:
    _check(load().regen_lse_merge(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(out),
                                  _ptr(lse_out), int(rows), D, _stream(stream)), "regen_lse_merge")


def regen_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, Sq, Skv, D, scale, stream, workspace,
                   workspace_bytes, accumulate=0) -> None:
    _check(load().regen_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                                 _ptr(dv), B, H, Sq, Skv, D, float(scale), _stream(stream), _ptr(workspace),
                                 int(workspace_bytes), int(accumulate)), "regen_attn_bwd")


def regen_attn_bwd_kv2(q, k_a, v_a, k_b, v_b, out, lse, dout, dq, dk_a, dv_a, dk_b, dv_b, B, H, Sq, Skv_a, Skv_b,
                       D, scale, stream, workspace, workspace_bytes, accumulate=0) -> None:
    _check(load().regen_attn_bwd_kv2(_ptr(q), _ptr(k_a), _ptr(v_a), _ptr(k_b), _ptr(v_b), _ptr(out), _ptr(lse),
                                     _ptr(dout), _ptr(dq), _ptr(dk_a), _ptr(dv_a), _ptr(dk_b), _ptr(dv_b), B, H, Sq,
                                     Skv_a, Skv_b, D, float(scale), _stream(stream), _ptr(workspace),
                                     int(workspace_bytes), int(accumulate)), "regen_attn_bwd_kv2")


def regen_attn_bwd_workspace_bytes(B, H, Sq, D) -> int:
    n = load().regen_attn_bwd_workspace_bytes(B, H, Sq, D)
    if n < 0:
        raise RegenError(int(n), "regen_attn_bwd_workspace_bytes")
    return int(n)


def regen_rope3d_bwd(dq, dk, T, Hh, Ww, theta, B, H, D, stream=None) -> None:
    _check(load().regen_rope3d_bwd(_ptr(dq), _ptr(dk), T, Hh, Ww, float(theta), B, H, D, _stream(stream)),
           "regen_rope3d_bwd")


def regen_quant_e4m3(x, codes, scales, B, H, S, D, stream=None) -> None:
    _check(load().regen_quant_e4m3(_ptr(x), _ptr(codes), _ptr(scales), B, H, S, D, _stream(stream)),
           "regen_quant_e4m3")


def regen_attn_fwd_fp8(q8, q_scale, k8, k_scale, v8, v_scale, out, lse, B, H, Sq, Skv, D, scale,
                       stream=None) -> None:
    _check(load().regen_attn_fwd_fp8(_ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(v8), _ptr(v_scale),
                                     _ptr(out), _ptr(lse), B, H, Sq, Skv, D, float(scale), _stream(stream)),
           "regen_attn_fwd_fp8")


def regen_qkv_proj(x, w, bias, gamma_q, gamma_k, q, k, v, B, S, C, H, D, T, Hh, Ww, theta, eps, stream,
                   workspace, workspace_bytes) -> None:
    _check(load().regen_qkv_proj(_ptr(x), _ptr(w), _ptr(bias), _ptr(gamma_q), _ptr(gamma_k), _ptr(q), _ptr(k),
                                 _ptr(v), B, S, C, H, D, T, Hh, Ww, float(theta), float(eps), _stream(stream),
                                 _ptr(workspace), int(workspace_bytes)), "regen_qkv_proj")


def regen_qkv_proj_workspace_bytes(T, Hh, Ww, D) -> int:
    n = load().regen_qkv_proj_workspace_bytes(T, Hh, Ww, D)
    if n < 0:
        raise RegenError(int(n), "regen_qkv_proj_workspace_bytes")
    return int(n)


def regen_out_proj(o, w, bias, y, B, S, H, D, N, stream=None) -> None:
    _check(load().regen_out_proj(_ptr(o), _ptr(w), _ptr(bias), _ptr(y), B, S, H, D, N, _stream(stream)),
           "regen_out_proj")


def regen_rope3d_shard(q, k, T, Hh, Ww, theta, B, H, D, n0, S_local, inverse=0, stream=None) -> None:
    _check(load().regen_rope3d_shard(_ptr(q), _ptr(k), T, Hh, Ww, float(theta), B, H, D, int(n0), int(S_local),
                                     int(inverse), _stream(stream)), "regen_rope3d_shard")


def regen_selftest_exp2(x, y, n, stream=None) -> None:
    _check(load().regen_selftest_exp2(_ptr(x), _ptr(y), int(n), _stream(stream)), "regen_selftest_exp2")


def regen_selftest_bounded_wait(limit_ns, done, stream=None) -> None:
    _check(load().regen_selftest_bounded_wait(int(limit_ns), _ptr(done), _stream(stream)),
           "regen_selftest_bounded_wait")


def regen_status_str(status: int) -> str:
    return load().regen_status_str(status).decode()


def regen_last_device_error():
    """(status, site): synchronises the device, reads and clears the kernels' error record."""
    site = ctypes.c_uint32(0)
    rc = load().regen_last_device_error(ctypes.byref(site))
    return rc, site.value


def regen_last_cuda_error():
    """(code, name) of the CUDA result behind this thread's last REGEN_ERR_CUDA
    (0, "none" when there is none); reading clears it."""
    name = ctypes.c_char_p()
    code = load().regen_last_cuda_error(ctypes.byref(name))
    return code, (name.value or b"").decode()


def regen_set_wait_limit_ns(ns: int) -> None:
    _check(load().regen_set_wait_limit_ns(int(ns)), "regen_set_wait_limit_ns")


def regen_version() -> int:
    return load().regen_version()


# ------------------------------------------------------- torch helpers ---

def _bhsd(t, name):
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, H, S, D] tensor")
    return t.shape


def attn_fwd(q, k, v, scale=None, out=None, lse=None, stream=None):
    """Exact attention on bf16 [B, H, S, D] CUDA tensors -> (out bf16, lse fp32)."""
    import torch
    B, H, Sq, D = _bhsd(q, "q")
    Skv = _bhsd(k, "k")[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    regen_attn_fwd(q, k, v, out, lse, B, H, Sq, Skv, D, scale, stream)
    return out, lse


def attn_fwd_kv2(q, k_a, v_a, k_b, v_b, scale=None, out=None, lse=None, stream=None):
    """Attention of q over two key/value sources as one softmax over their
    concatenation [k_a; k_b] -> (out bf16, lse fp32)."""
    import torch
    B, H, Sq, D = _bhsd(q, "q")
    Skv_a, Skv_b = _bhsd(k_a, "k_a")[2], _bhsd(k_b, "k_b")[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    regen_attn_fwd_kv2(q, k_a, v_a, k_b, v_b, out, lse, B, H, Sq, Skv_a, Skv_b, D, scale, stream)
    return out, lse


def attn_fwd_rope3d(q, k, v, grid, theta=10000.0, scale=None, out=None, lse=None, workspace=None, stream=None):
    """Self-attention with 3D RoPE on Q and K (q, k not modified) -> (out, lse)."""
    import torch
    B, H, S, D = _bhsd(q, "q")
    T, Hh, Ww = grid
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    need = regen_attn_fwd_rope3d_workspace_bytes(B, H, T, Hh, Ww, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    regen_attn_fwd_rope3d(q, k, v, out, lse, B, H, S, S, D, scale, stream, T, Hh, Ww, theta, workspace,
                          workspace.numel() * workspace.element_size())
    return out, lse


def rope3d_(q, k, grid, theta=10000.0, stream=None):
    """3D RoPE in place on bf16 [B, H, T*Hh*Ww, D] CUDA tensors (either may be None)."""
    ref = q if q is not None else k
    B, H, S, D = _bhsd(ref, "q/k")
    T, Hh, Ww = grid
    if S != T * Hh * Ww:
        raise ValueError("sequence length does not match the latent grid")
    regen_rope3d(q, k, T, Hh, Ww, theta, B, H, D, stream)
    return q, k


def lse_merge(o_a, lse_a, o_b, lse_b, out=None, lse_out=None, stream=None):
    """Merge two partial attentions (bf16 [..., D], fp32 [...]) -> (out, lse)."""
    import torch
    D = o_a.shape[-1]
    rows = o_a.numel() // D
    if out is None:
        out = torch.empty_like(o_a)
    if lse_out is None:
        lse_out = torch.empty_like(lse_a)
    regen_lse_merge(o_a, lse_a, o_b, lse_b, out, lse_out, rows, D, stream)
    return out, lse_out


def attn_bwd(q, k, v, out, lse, dout, scale=None, dq=None, dk=None, dv=None, accumulate_dq=False,
             workspace=None, stream=None, accumulate_dkdv=False):
    """Gradients of attn_fwd -> (dq, dk, dv), bf16 like the inputs.

    out and lse are the forward's (or, for one key block of a merged
    attention, the merged ones). accumulate_dq adds into the given dq,
    accumulate_dkdv into the given dk and dv."""
    import torch
    B, H, Sq, D = _bhsd(q, "q")
    Skv = _bhsd(k, "k")[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if accumulate_dq and dq is None:
        raise ValueError("accumulate_dq needs the dq to add into")
    if accumulate_dkdv and (dk is None or dv is None):
        raise ValueError("accumulate_dkdv needs the dk and dv to add into")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = regen_attn_bwd_workspace_bytes(B, H, Sq, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    regen_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, Sq, Skv, D, scale, stream, workspace,
                   workspace.numel() * workspace.element_size(),
                   (REGEN_ACCUM_DQ if accumulate_dq else 0) | (REGEN_ACCUM_DKDV if accumulate_dkdv else 0))
    return dq, dk, dv


def attn_bwd_kv2(q, k_a, v_a, k_b, v_b, out, lse, dout, scale=None, dq=None, accumulate_dq=False, workspace=None,
                 stream=None, dkv=None, accumulate_dkdv=False):
    """Gradients of attn_fwd_kv2 -> (dq, dk_a, dv_a, dk_b, dv_b), bf16 like the
    inputs; out and lse are the two-source forward's. accumulate_dq adds into
    the given dq; accumulate_dkdv into the given dkv = (dk_a, dv_a, dk_b, dv_b)."""
    import torch
    B, H, Sq, D = _bhsd(q, "q")
    Skv_a, Skv_b = _bhsd(k_a, "k_a")[2], _bhsd(k_b, "k_b")[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if accumulate_dq and dq is None:
        raise ValueError("accumulate_dq needs the dq to add into")
    if accumulate_dkdv and dkv is None:
        raise ValueError("accumulate_dkdv needs the dk_a, dv_a, dk_b, dv_b to add into")
    dq = torch.empty_like(q) if dq is None else dq
    dk_a, dv_a, dk_b, dv_b = (torch.empty_like(t) for t in (k_a, v_a, k_b, v_b)) if dkv is None else dkv
    need = regen_attn_bwd_workspace_bytes(B, H, Sq, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    regen_attn_bwd_kv2(q, k_a, v_a, k_b, v_b, out, lse, dout, dq, dk_a, dv_a, dk_b, dv_b, B, H, Sq, Skv_a, Skv_b, D,
                       scale, stream, workspace, workspace.numel() * workspace.element_size(),
                       (REGEN_ACCUM_DQ if accumulate_dq else 0) | (REGEN_ACCUM_DKDV if accumulate_dkdv else 0))
    return dq, dk_a, dv_a, dk_b, dv_b


def rope3d_bwd_(dq, dk, grid, theta=10000.0, stream=None):
    """Gradient of rope3d_, in place on the gradients (either may be None)."""
    ref = dq if dq is not None else dk
    B, H, S, D = _bhsd(ref, "dq/dk")
    T, Hh, Ww = grid
    if S != T * Hh * Ww:
        raise ValueError("sequence length does not match the latent grid")
    regen_rope3d_bwd(dq, dk, T, Hh, Ww, theta, B, H, D, stream)
    return dq, dk


def quant_e4m3(x, codes=None, scales=None, stream=None):
    """Blockwise E4M3 codes (uint8, same shape) and fp32 scales [B, H, ceil(S/128)]
    of a bf16 [B, H, S, D] CUDA tensor."""
    import torch
    B, H, S, D = _bhsd(x, "x")
    if codes is None:
        codes = torch.empty((B, H, S, D), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((B, H, -(-S // 128)), dtype=torch.float32, device=x.device)
    regen_quant_e4m3(x, codes, scales, B, H, S, D, stream)
    return codes, scales


def attn_fwd_fp8(q8, q_scale, k8, k_scale, v8, v_scale, scale=None, out=None, lse=None, stream=None):
    """FP8 attention from quant_e4m3 outputs -> (out bf16, lse fp32)."""
    import torch
    B, H, Sq, D = _bhsd(q8, "q8")
    Skv = _bhsd(k8, "k8")[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, H, Sq, D), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q8.device)
    regen_attn_fwd_fp8(q8, q_scale, k8, k_scale, v8, v_scale, out, lse, B, H, Sq, Skv, D, scale, stream)
    return out, lse


def qkv_proj(x, w, heads, grid, bias=None, gamma_q=None, gamma_k=None, theta=10000.0, eps=1e-6, q=None, k=None,
             v=None, workspace=None, stream=None):
    """Fused QKV projection of bf16 token features x [B, S, C] with w [3*heads*128, C]
    -> q, k, v [B, heads, S, 128] (RMSNorm + 3D RoPE on q and k)."""
    import torch
    if x.dim() != 3 or not x.is_contiguous():
        raise ValueError("x must be a contiguous [B, S, C] tensor")
    B, S, C = x.shape
    T, Hh, Ww = grid
    H, D = int(heads), 128
    shape = (B, H, S, D)
    q = torch.empty(shape, dtype=torch.bfloat16, device=x.device) if q is None else q
    k = torch.empty(shape, dtype=torch.bfloat16, device=x.device) if k is None else k
    v = torch.empty(shape, dtype=torch.bfloat16, device=x.device) if v is None else v
    need = regen_qkv_proj_workspace_bytes(T, Hh, Ww, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    regen_qkv_proj(x, w, bias, gamma_q, gamma_k, q, k, v, B, S, C, H, D, T, Hh, Ww, theta, eps, stream, workspace,
                   workspace.numel() * workspace.element_size())
    return q, k, v


def out_proj(o, w, bias=None, y=None, stream=None):
    """Output projection of the attention output o [B, H, S, 128] with w [N, H*128]
    -> y [B, S, N] bf16."""
    import torch
    B, H, S, D = _bhsd(o, "o")
    N = w.shape[0]
    y = torch.empty((B, S, N), dtype=torch.bfloat16, device=o.device) if y is None else y
    regen_out_proj(o, w, bias, y, B, S, H, D, N, stream)
    return y
