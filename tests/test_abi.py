"""The C-ABI library: it builds, loads, exports exactly what include/regen_attn.h
declares, and answers invalid calls with the documented status before touching
the GPU (so these run without one)."""
import os
import re
import subprocess

import pytest

import dit_attention_b200 as rg
from dit_attention_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "regen_attn.h")


def declared_symbols():
    text = open(HEADER).read()
    return set(re.findall(r"REGEN_API\s+[\w\s\*]+?\b(regen_\w+)\s*\(", text))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return rg.load()


def test_exports_match_header(lib):
    declared = declared_symbols()
    assert {"regen_attn_fwd", "regen_rope3d", "regen_lse_merge"} <= declared
    out = subprocess.run(["nm", "-D", "--defined-only", rg.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.split()[-1].startswith("regen_")}
    assert exported == declared
    for name in declared:
        assert hasattr(lib, name)


def test_status_strings(lib):
    assert rg.regen_status_str(0) == "ok"
    assert "bounded wait" in rg.regen_status_str(-5)
    assert rg.regen_version() == 100


FAKE = 0x7F0000000000      # never dereferenced: every call below fails validation first
MB = 1 << 20


@pytest.mark.parametrize("args,status", [
    (dict(D=96), -2), (dict(D=0), -2), (dict(B=-1), -1), (dict(Sq=-3), -1), (dict(scale=float("inf")), -1),
    (dict(scale=float("nan")), -1), (dict(q=None), -1), (dict(k=None), -1), (dict(q=FAKE + 8), -3),
    (dict(lse=FAKE + 40 * MB + 4), -3), (dict(out=FAKE), -1), (dict(lse=FAKE + 1024), -1),
    (dict(B=0), 0), (dict(Sq=0), 0), (dict(H=0, q=None, out=None), 0),
])
def test_attn_fwd_validation(lib, args, status):
    a = dict(q=FAKE, k=FAKE + 10 * MB, v=FAKE + 20 * MB, out=FAKE + 30 * MB, lse=FAKE + 40 * MB,
             B=1, H=2, Sq=100, Skv=100, D=128, scale=0.125)
    a.update(args)
    rc = lib.regen_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"], a["Sq"], a["Skv"],
                            a["D"], a["scale"], None)
    assert rc == status


@pytest.mark.parametrize("args,status", [
    (dict(theta=0.0), -1), (dict(theta=float("inf")), -1), (dict(T=0), -1), (dict(D=12), -2),
    (dict(D=520), -2), (dict(q=None, k=None), -1), (dict(k=FAKE + 2), -3), (dict(k=FAKE + 16), -1),
    (dict(B=0), 0),
])
def test_rope3d_validation(lib, args, status):
    a = dict(q=FAKE, k=FAKE + 10 * MB, T=2, Hh=3, Ww=4, theta=10000.0, B=1, H=2, D=64)
    a.update(args)
    rc = lib.regen_rope3d(a["q"], a["k"], a["T"], a["Hh"], a["Ww"], a["theta"], a["B"], a["H"], a["D"], None)
    assert rc == status


@pytest.mark.parametrize("args,status", [
    (dict(rows=0), 0), (dict(rows=-1), -1), (dict(D=7), -2), (dict(o_a=None), -1), (dict(lse_b=FAKE + 3), -3),
    (dict(lse_out=FAKE + 20 * MB), -1), (dict(out=FAKE + 4096), -1),
])
def test_lse_merge_validation(lib, args, status):
    a = dict(o_a=FAKE, lse_a=FAKE + 20 * MB, o_b=FAKE + 10 * MB, lse_b=FAKE + 30 * MB, out=FAKE + 40 * MB,
             lse_out=FAKE + 50 * MB, rows=1000, D=128)
    a.update(args)
    rc = lib.regen_lse_merge(a["o_a"], a["lse_a"], a["o_b"], a["lse_b"], a["out"], a["lse_out"], a["rows"],
                             a["D"], None)
    assert rc == status


def test_python_binding_raises(lib):
    with pytest.raises(rg.RegenError) as e:
        rg.regen_attn_fwd(FAKE, FAKE + MB, FAKE + 2 * MB, FAKE + 3 * MB, None, 1, 1, 8, 8, 96, 0.1, stream=0)
    assert e.value.status == -2


def test_rope3d_fused_workspace_bytes(lib):
    # E = T*dt/2 + (Hh + Ww)*dh/2 table entries: 16 E bytes (fp64) and 8 E bytes (fp32),
    # each rounded up to 256; plus B*H*S*D*2 of rotated K
    T, Hh, Ww, D = 20, 30, 52, 128
    E = T * 22 + (Hh + Ww) * 21
    table = (16 * E + 255) // 256 * 256 + (8 * E + 255) // 256 * 256
    assert rg.regen_attn_fwd_rope3d_workspace_bytes(1, 40, T, Hh, Ww, D) == table + 40 * T * Hh * Ww * D * 2
    assert lib.regen_attn_fwd_rope3d_workspace_bytes(1, 1, 0, 1, 1, 128) == -1
    assert lib.regen_attn_fwd_rope3d_workspace_bytes(1, 1, 1, 1, 1, 96) == -2


@pytest.mark.parametrize("args,status", [
    (dict(Sq=99), -1), (dict(Skv=99), -1), (dict(D=96), -2), (dict(theta=0.0), -1), (dict(scale=float("nan")), -1),
    (dict(workspace=None), -1), (dict(workspace=FAKE + 100 * MB + 16), -3), (dict(workspace_bytes=1000), -1),
    (dict(workspace=FAKE), -1), (dict(B=0), 0),
])
def test_rope3d_fused_validation(lib, args, status):
    a = dict(q=FAKE, k=FAKE + 10 * MB, v=FAKE + 20 * MB, out=FAKE + 30 * MB, lse=FAKE + 40 * MB, B=1, H=2, Sq=60,
             Skv=60, D=128, scale=0.1, T=3, Hh=4, Ww=5, theta=1e4, workspace=FAKE + 100 * MB,
             workspace_bytes=64 * MB)
    a.update(args)
    rc = lib.regen_attn_fwd_rope3d(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"], a["Sq"], a["Skv"],
                                   a["D"], a["scale"], None, a["T"], a["Hh"], a["Ww"], a["theta"], a["workspace"],
                                   a["workspace_bytes"])
    assert rc == status


def test_attn_bwd_workspace_bytes(lib):
    # [B*H][ceil(Sq/128)][2][128] floats
    assert rg.regen_attn_bwd_workspace_bytes(1, 40, 31200, 128) == 40 * 244 * 1024
    assert rg.regen_attn_bwd_workspace_bytes(2, 3, 1, 64) == 6 * 1024
    assert rg.regen_attn_bwd_workspace_bytes(1, 1, 0, 128) == 0
    assert lib.regen_attn_bwd_workspace_bytes(1, 1, 128, 96) == -2
    assert lib.regen_attn_bwd_workspace_bytes(-1, 1, 128, 128) == -1


# inputs q, out, dout (Sq rows), k, v (Skv rows), lse; outputs dq, dk, dv; workspace
_BWD = dict(q=FAKE, k=FAKE + 10 * MB, v=FAKE + 20 * MB, out=FAKE + 30 * MB, lse=FAKE + 40 * MB,
            dout=FAKE + 50 * MB, dq=FAKE + 60 * MB, dk=FAKE + 70 * MB, dv=FAKE + 80 * MB, ws=FAKE + 90 * MB,
            B=1, H=2, Sq=100, Skv=100, D=128, scale=0.125, wsb=2048, acc=0)


@pytest.mark.parametrize("args,status", [
    (dict(D=96), -2), (dict(B=-1), -1), (dict(Skv=-1), -1), (dict(scale=float("nan")), -1), (dict(acc=4), -1), (dict(acc=-1), -1),
    (dict(wsb=-1), -1), (dict(wsb=2047), -1), (dict(ws=None), -1), (dict(lse=None), -1), (dict(dout=None), -1),
    (dict(dk=None), -1), (dict(ws=FAKE + 90 * MB + 16), -3), (dict(dq=FAKE + 60 * MB + 2), -3),
    (dict(dq=FAKE + 4096), -1),            # dq overlaps q
    (dict(dk=FAKE + 60 * MB + 4096), -1),  # dk overlaps dq
    (dict(ws=FAKE + 50 * MB), -1),         # workspace overlaps dout
    (dict(dv=FAKE + 40 * MB), -1),         # dv overlaps lse
    (dict(B=0), 0), (dict(H=0, q=None), 0), (dict(Sq=0, Skv=0), 0),
    (dict(Sq=0, dk=None), -1), (dict(Skv=0, dq=FAKE + 60 * MB + 8), -3),
    (dict(Skv=0, acc=1, dq=FAKE + 60 * MB), 0),   # accumulating nothing: dq unchanged, no launch
    (dict(Sq=0, acc=2), 0),                       # accumulating nothing: dk, dv unchanged, no launch
])
def test_attn_bwd_validation(lib, args, status):
    a = dict(_BWD)
    a.update(args)
    rc = lib.regen_attn_bwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], a["dq"], a["dk"], a["dv"],
                            a["B"], a["H"], a["Sq"], a["Skv"], a["D"], a["scale"], None, a["ws"], a["wsb"], a["acc"])
    assert rc == status


@pytest.mark.parametrize("args,status", [
    (dict(T=0), -1), (dict(theta=0.0), -1), (dict(D=12), -2), (dict(q=FAKE + 2), -3), (dict(q=None, k=None), -1),
    (dict(B=0), 0),
])
def test_rope3d_bwd_validation(lib, args, status):
    a = dict(q=FAKE, k=FAKE + 10 * MB, T=2, Hh=3, Ww=4, theta=1e4, B=1, H=2, D=128)
    a.update(args)
    rc = lib.regen_rope3d_bwd(a["q"], a["k"], a["T"], a["Hh"], a["Ww"], a["theta"], a["B"], a["H"], a["D"], None)
    assert rc == status


@pytest.mark.parametrize("args,status", [
    (dict(D=96), -2), (dict(B=-1), -1), (dict(x=None), -1), (dict(codes=FAKE + 20 * MB + 8), -3),
    (dict(scales=FAKE + 30 * MB + 2), -3), (dict(codes=FAKE + 4096), -1), (dict(S=0), 0), (dict(H=0, x=None), 0),
])
def test_quant_e4m3_validation(lib, args, status):
    a = dict(x=FAKE, codes=FAKE + 20 * MB, scales=FAKE + 30 * MB, B=1, H=2, S=300, D=128)
    a.update(args)
    assert lib.regen_quant_e4m3(a["x"], a["codes"], a["scales"], a["B"], a["H"], a["S"], a["D"], None) == status


@pytest.mark.parametrize("args,status", [
    (dict(D=64), -2), (dict(Sq=-1), -1), (dict(scale=float("inf")), -1), (dict(q8=None), -1), (dict(vs=None), -1),
    (dict(q8=FAKE + 4), -3), (dict(ks=FAKE + 50 * MB + 1), -3), (dict(out=FAKE + 1024), -1),
    (dict(lse=FAKE + 60 * MB + 16), -1), (dict(B=0), 0), (dict(Sq=0), 0),
])
def test_attn_fwd_fp8_validation(lib, args, status):
    a = dict(q8=FAKE, qs=FAKE + 10 * MB, k8=FAKE + 20 * MB, ks=FAKE + 30 * MB, v8=FAKE + 40 * MB, vs=FAKE + 50 * MB,
             out=FAKE + 60 * MB, lse=FAKE + 70 * MB, B=1, H=2, Sq=300, Skv=200, D=128, scale=0.1)
    a.update(args)
    rc = lib.regen_attn_fwd_fp8(a["q8"], a["qs"], a["k8"], a["ks"], a["v8"], a["vs"], a["out"], a["lse"], a["B"],
                                a["H"], a["Sq"], a["Skv"], a["D"], a["scale"], None)
    assert rc == status


@pytest.mark.parametrize("args,status", [
    (dict(D=64), -2), (dict(C=100), -2), (dict(S=61), -1), (dict(theta=0.0), -1), (dict(eps=-1.0), -1),
    (dict(x=None), -1), (dict(ws=None), -1), (dict(wsb=16), -1), (dict(bias=FAKE + 40 * MB + 4), -3),
    (dict(ws=FAKE + 90 * MB + 64), -3), (dict(q=FAKE + 4096), -1), (dict(k=FAKE + 50 * MB + 1024), -1),
    (dict(ws=FAKE + 10 * MB), -1), (dict(B=0), 0), (dict(H=0, x=None), 0),
])
def test_qkv_proj_validation(lib, args, status):
    # x [1, 60, 256]; w [3*2*128, 256]; grid 3x4x5
    a = dict(x=FAKE, w=FAKE + 10 * MB, bias=FAKE + 40 * MB, gq=None, gk=None, q=FAKE + 50 * MB, k=FAKE + 60 * MB,
             v=FAKE + 70 * MB, B=1, S=60, C=256, H=2, D=128, T=3, Hh=4, Ww=5, theta=1e4, eps=1e-6,
             ws=FAKE + 90 * MB, wsb=4096)
    a.update(args)
    rc = lib.regen_qkv_proj(a["x"], a["w"], a["bias"], a["gq"], a["gk"], a["q"], a["k"], a["v"], a["B"], a["S"],
                            a["C"], a["H"], a["D"], a["T"], a["Hh"], a["Ww"], a["theta"], a["eps"], None, a["ws"],
                            a["wsb"])
    assert rc == status


def test_qkv_proj_workspace_bytes(lib):
    # (20*22 + 30*21 + 52*21) entries of (cos, sin) fp32, rounded up to 256 bytes
    assert rg.regen_qkv_proj_workspace_bytes(20, 30, 52, 128) == -(-(440 + 630 + 1092) * 8 // 256) * 256
    assert lib.regen_qkv_proj_workspace_bytes(2, 3, 4, 64) == -2


@pytest.mark.parametrize("args,status", [
    (dict(D=64), -2), (dict(N=100), -2), (dict(H=0), -1), (dict(o=None), -1), (dict(y=FAKE + 8), -3),
    (dict(y=FAKE + 4096), -1), (dict(y=FAKE + 10 * MB), -1), (dict(B=0), 0), (dict(N=0), 0),
])
def test_out_proj_validation(lib, args, status):
    a = dict(o=FAKE, w=FAKE + 10 * MB, bias=None, y=FAKE + 30 * MB, B=1, S=60, H=2, D=128, N=256)
    a.update(args)
    rc = lib.regen_out_proj(a["o"], a["w"], a["bias"], a["y"], a["B"], a["S"], a["H"], a["D"], a["N"], None)
    assert rc == status


@pytest.mark.parametrize("args,status", [
    (dict(n0=-1), -1), (dict(n0=50, S=11), -1), (dict(S=-1), -1), (dict(inv=2), -1), (dict(D=12), -2),
    (dict(S=0), 0), (dict(q=FAKE + 2), -3), (dict(B=0), 0),
])
def test_rope3d_shard_validation(lib, args, status):
    # grid 3 x 4 x 5 = 60 tokens; the shard holds tokens n0 .. n0 + S - 1
    a = dict(q=FAKE, k=FAKE + 10 * MB, T=3, Hh=4, Ww=5, theta=1e4, B=1, H=2, D=128, n0=20, S=30, inv=0)
    a.update(args)
    rc = lib.regen_rope3d_shard(a["q"], a["k"], a["T"], a["Hh"], a["Ww"], a["theta"], a["B"], a["H"], a["D"], a["n0"],
                                a["S"], a["inv"], None)
    assert rc == status


def test_noalloc_scratch_size_matches_header(lib):
    text = open(HEADER).read()
    m = re.search(r"#define\s+REGEN_NOALLOC_SCRATCH_BYTES\s+\((\d+)LL\s*<<\s*(\d+)\)", text)
    assert m, "REGEN_NOALLOC_SCRATCH_BYTES not found in the header"
    assert rg.regen_noalloc_scratch_bytes() == int(m.group(1)) << int(m.group(2))


CTX_CACHE_TEST = r"""
#include <cstdio>
#include "ctx_cache.h"
int main() {
    regen::CtxCache<int, -4> cache;
    int calls = 0, v = 0;
    auto setup = [&](int value, int status) {
        return [&calls, value, status](int *out) { ++calls; *out = value; return status; };
    };
    // context 7: set up once, then served from the cache
    if (cache.get(7, setup(70, 0), &v) != 0 || v != 70 || calls != 1) return 1;
    if (cache.get(7, setup(71, 0), &v) != 0 || v != 70 || calls != 1) return 2;
    // a second context (another GPU, or a context the host created) gets its own set-up
    if (cache.get(9, setup(90, 0), &v) != 0 || v != 90 || calls != 2) return 3;
    if (cache.get(7, setup(72, 0), &v) != 0 || v != 70 || calls != 2) return 4;
    // a failing CUDA call (-4) is not cached: the next call retries
    if (cache.get(11, setup(0, -4), &v) != -4 || calls != 3) return 5;
    if (cache.get(11, setup(110, 0), &v) != 0 || v != 110 || calls != 4) return 6;
    // a refusal that a retry cannot change (-2) is cached like a success
    if (cache.get(13, setup(0, -2), &v) != -2 || calls != 5) return 7;
    if (cache.get(13, setup(130, 0), &v) != -2 || calls != 5) return 8;
    std::puts("ok");
    return 0;
}
"""


def test_per_context_setup_cache(tmp_path):
    """Kernel attributes and the fixed scratch's address are set up per CUDA
    context: each context runs the set-up once, failures of the CUDA call
    itself are retried, refusals are kept."""
    src = tmp_path / "ctx_cache_test.cpp"
    src.write_text(CTX_CACHE_TEST)
    exe = tmp_path / "ctx_cache_test"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "dit_attention_b200", "csrc"),
                    str(src), "-o", str(exe), "-pthread"], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True)
    assert res.returncode == 0 and res.stdout.strip() == "ok", (res.returncode, res.stdout)


@pytest.mark.parametrize("args,status", [
    (dict(D=96), -2), (dict(B=-1), -1), (dict(Skv_a=-1), -1), (dict(Skv_b=-2), -1), (dict(scale=float("nan")), -1),
    (dict(k_b=None), -1), (dict(v_a=None), -1), (dict(k_a=FAKE + 10 * MB + 8), -3), (dict(lse=FAKE + 60 * MB + 4), -3),
    (dict(out=FAKE + 20 * MB), -1), (dict(lse=FAKE + 40 * MB), -1), (dict(Skv_a=2**30, Skv_b=2**30), -2),
    (dict(B=0), 0), (dict(Sq=0), 0),
])
def test_attn_fwd_kv2_validation(lib, args, status):
    a = dict(q=FAKE, k_a=FAKE + 10 * MB, v_a=FAKE + 20 * MB, k_b=FAKE + 30 * MB, v_b=FAKE + 40 * MB,
             out=FAKE + 50 * MB, lse=FAKE + 60 * MB, B=1, H=2, Sq=100, Skv_a=60, Skv_b=40, D=128, scale=0.125)
    a.update(args)
    rc = lib.regen_attn_fwd_kv2(a["q"], a["k_a"], a["v_a"], a["k_b"], a["v_b"], a["out"], a["lse"], a["B"], a["H"],
                                a["Sq"], a["Skv_a"], a["Skv_b"], a["D"], a["scale"], None)
    assert rc == status


@pytest.mark.parametrize("args,status", [
    (dict(D=96), -2), (dict(B=-1), -1), (dict(Skv_b=-1), -1), (dict(scale=float("inf")), -1),
    (dict(accumulate=4), -1), (dict(B=0), 0), (dict(Skv_a=2**30, Skv_b=2**30), -2),
    (dict(k_b=None), -1), (dict(dv_b=None), -1), (dict(ws=None), -1), (dict(dk_b=FAKE + 110 * MB + 8), -3),
    (dict(ws=FAKE + 130 * MB + 16), -3), (dict(ws_bytes=2047), -1), (dict(dv_b=FAKE + 90 * MB), -1),
    (dict(dq=FAKE + 10 * MB), -1), (dict(ws=FAKE + 60 * MB), -1),
    # no queries: both sources' buffers are checked before anything is launched
    (dict(Sq=0, dv_b=FAKE + 120 * MB + 2), -3), (dict(Sq=0, dk_b=None), -1), (dict(Sq=0, dk_b=FAKE + 90 * MB), -1),
])
def test_attn_bwd_kv2_validation(lib, args, status):
    a = dict(q=FAKE, k_a=FAKE + 10 * MB, v_a=FAKE + 20 * MB, k_b=FAKE + 30 * MB, v_b=FAKE + 40 * MB,
             out=FAKE + 50 * MB, lse=FAKE + 60 * MB, dout=FAKE + 70 * MB, dq=FAKE + 80 * MB, dk_a=FAKE + 90 * MB,
             dv_a=FAKE + 100 * MB, dk_b=FAKE + 110 * MB, dv_b=FAKE + 120 * MB, ws=FAKE + 130 * MB, ws_bytes=2048,
             B=1, H=2, Sq=100, Skv_a=60, Skv_b=40, D=128, scale=0.125, accumulate=0)
    a.update(args)
    rc = lib.regen_attn_bwd_kv2(a["q"], a["k_a"], a["v_a"], a["k_b"], a["v_b"], a["out"], a["lse"], a["dout"],
                                a["dq"], a["dk_a"], a["dv_a"], a["dk_b"], a["dv_b"], a["B"], a["H"], a["Sq"],
                                a["Skv_a"], a["Skv_b"], a["D"], a["scale"], None, a["ws"], a["ws_bytes"],
                                a["accumulate"])
    assert rc == status
