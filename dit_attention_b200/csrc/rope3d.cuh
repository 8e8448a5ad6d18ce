// rope3d.cuh -- 3D rotary position embedding of Q and K (sm_100a).
//
// The ReGenVC decoder's DiT matches the Wan2.1-Fun-Control architecture (blog
// page, "Methodology -- deep read"), whose attention rotates Q and K by a 3D
// RoPE over the latent (t, h, w) grid. Reading used (the pages print no
// formula): token n = (t*Hh + y)*Ww + x; head-dim blocks t, h, w of widths
// D - 4*floor(D/6), 2*floor(D/6), 2*floor(D/6); pair (2j, 2j+1) of a block of
// width d turns by pos * theta^(-2j/d).
//
// Result contract: the angle's cosine and sine in fp64, the rotation in fp64,
// one rounding to bf16 (nearest even). The kernels reach that result with
// fp32 arithmetic on the fp32 roundings of the fp64 cosine and sine, and prove
// per element that the fp32 value rounds to the same bf16 as the fp64 one
// (rotate_pair_f32); the few pairs it cannot prove (about one in a thousand,
// near a bf16 rounding boundary) are redone in fp64 (rotate_pair).
//
// HBM-bound: every element is read and written once. One thread owns one
// 16-byte chunk (4 pairs) of one token's row and walks that chunk through
// every row of Q (or of K): its 4 angles are evaluated once and stay in
// registers in fp64 (for the rare fp64 redo) and fp32 (for the rotation), and
// the next four rows' loads are in flight while it rotates and stores the
// current four. Adjacent threads own adjacent chunks of a row: each warp
// access is two contiguous 256-byte rows.
#pragma once

#include <stdint.h>

#include "ptx.cuh"

namespace regen {

// bf16 -> double, exact (every bf16 is a double).
__device__ __forceinline__ double bf16_bits_to_double(uint32_t h16)
{
    double d;
    asm("cvt.f64.bf16 %0, %1;" : "=d"(d) : "h"(static_cast<unsigned short>(h16)));
    return d;
}

// Correctly rounded double -> bf16 (nearest, ties to even) in one conversion,
// no intermediate fp32 rounding; NaN becomes the canonical 0x7FC0.
__device__ __forceinline__ uint32_t double_to_bf16_bits(double x)
{
    unsigned short h;
    asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(h) : "d"(x));
    return x != x ? 0x7FC0u : static_cast<uint32_t>(h);
}

// Rotate one (even, odd) pair packed as two bf16 by the angle with cosine c
// and sine s, in fp64 with one explicit rounding order (so every kernel that
// rotates gives the same bits), then round each result once to bf16.
__device__ __forceinline__ uint32_t rotate_pair(uint32_t packed, double c, double s)
{
    const double x0 = bf16_bits_to_double(packed & 0xFFFFu);
    const double x1 = bf16_bits_to_double(packed >> 16);
    const double y0 = __fma_rn(x0, c, -__dmul_rn(x1, s));
    const double y1 = __fma_rn(x0, s, __dmul_rn(x1, c));
    return double_to_bf16_bits(y0) | (double_to_bf16_bits(y1) << 16);
}

// The same pair rotated in fp32 from c32 = fp32(c) and s32 = fp32(s), with a
// proof that it rounds like rotate_pair: returns true when both packed results
// in `out` equal rotate_pair(packed, c, s), false when it cannot tell.
// Bound: with X = |x0| + |x1|, the fp32 value differs from the fp64 one by at
// most 3.0001 * 2^-24 * X + 2^-148 (the fp32 roundings of c and s, of the
// product, of the fused result, and the fp64 path's own 2^-52 X; the last
// term covers results among the fp32 subnormals). If no bf16 rounding
// boundary -- the midpoint between two neighbouring bf16 values -- lies
// within that distance of the fp32 value, both round to the same bf16. The
// test uses fl(fl(X) * 2^-22 + 2^-146): fl(X) and the fused product each lose
// at most a factor (1 - 2^-24), and 4 (1 - 2^-24)^2 > 3.0001 (1 + 2^-24), so
// it is never below the bound. It measures the distance to the midpoint of the
// bf16 cell that holds y, which is exact in fp32 (same sign and binade). A
// NaN or infinite value fails the test and goes to fp64.
__device__ __forceinline__ bool rotate_pair_f32(uint32_t packed, float c32, float s32, uint32_t &out)
{
    const float x0 = __uint_as_float(packed << 16);
    const float x1 = __uint_as_float(packed & 0xFFFF0000u);
    const float y0 = __fmaf_rn(x0, c32, -__fmul_rn(x1, s32));
    const float y1 = __fmaf_rn(x0, s32, __fmul_rn(x1, c32));
    const float bound = __fmaf_rn(__fadd_rn(fabsf(x0), fabsf(x1)), 0x1p-22f, 0x1p-146f);
    const float g0 = fabsf(__fsub_rn(y0, __uint_as_float((__float_as_uint(y0) & 0xFFFF0000u) | 0x8000u)));
    const float g1 = fabsf(__fsub_rn(y1, __uint_as_float((__float_as_uint(y1) & 0xFFFF0000u) | 0x8000u)));
    out = pack_bf16x2(y0, y1);
    return g0 > bound && g1 > bound;
}

// Frequencies theta^(-local/width) of the pairs of a head dimension D <= 512,
// indexed by pair (d/2 for the pair starting at dimension d): they depend on
// D and theta only, so the host evaluates them once per call (fp64 pow) and
// passes them by value.
struct RopeFreqs {
    double f[256];
};

// cos and sin of pos * freq (fp64).
__device__ __forceinline__ void rope_angle(int pos, double freq, double &c, double &s)
{
    sincos(static_cast<double>(pos) * freq, &s, &c);
}

// Geometry of the 3D RoPE for a latent grid and head dim: axis blocks t, h, w
// of widths dt, dh, dh, and T*dt/2 + (Hh + Ww)*dh/2 (cos, sin) table entries.
// entry(n, d) indexes the position-major layout [T][dt/2], [Hh][dh/2],
// [Ww][dh/2] of the projection epilogue's table; the fused attention's table
// is pair-major (RopeRowEntries).
struct RopeGeom {
    int T, Hh, Ww, dt, dh;
    __host__ __device__ static RopeGeom make(int T, int Hh, int Ww, int D)
    {
        RopeGeom g;
        g.T = T; g.Hh = Hh; g.Ww = Ww;
        g.dh = 2 * (D / 6);
        g.dt = D - 2 * g.dh;
        return g;
    }
    __host__ __device__ int64_t entries() const
    {
        return static_cast<int64_t>(T) * (dt / 2) + static_cast<int64_t>(Hh) * (dh / 2) +
               static_cast<int64_t>(Ww) * (dh / 2);
    }
    // table entry of the pair whose first dimension is d, for token n
    __device__ __forceinline__ int64_t entry(int n, int d) const
    {
        if (d < dt) return static_cast<int64_t>(n / (Hh * Ww)) * (dt / 2) + d / 2;
        const int64_t base_h = static_cast<int64_t>(T) * (dt / 2);
        if (d < dt + dh) return base_h + static_cast<int64_t>((n / Ww) % Hh) * (dh / 2) + (d - dt) / 2;
        const int64_t base_w = base_h + static_cast<int64_t>(Hh) * (dh / 2);
        return base_w + static_cast<int64_t>(n % Ww) * (dh / 2) + (d - dt - dh) / 2;
    }
};

// The RoPE table of the fused attention, pair-major within each axis block:
// entries [dt/2][T], then [dh/2][Hh], then [dh/2][Ww] (pair j of position p of
// the t axis is entry j*T + p, and so on). Consecutive tokens differ mostly in
// their w position, so a warp's 32 rows read 32 consecutive entries of one
// pair (and broadcast entries for t and h): coalesced loads. t0, h0, w0: the
// token's entries of pair 0 in each block; a pair j further is j*T, j*Hh, j*Ww on.
struct RopeRowEntries {
    int64_t t0, h0, w0;
    int T, Hh, Ww;
    __device__ __forceinline__ static RopeRowEntries of(const RopeGeom &g, int n)
    {
        RopeRowEntries r;
        const int t = n / (g.Hh * g.Ww), y = (n / g.Ww) % g.Hh, x = n % g.Ww;
        const int64_t base_h = static_cast<int64_t>(g.T) * (g.dt / 2);
        const int64_t base_w = base_h + static_cast<int64_t>(g.Hh) * (g.dh / 2);
        r.t0 = t;
        r.h0 = base_h + y;
        r.w0 = base_w + x;
        r.T = g.T;
        r.Hh = g.Hh;
        r.Ww = g.Ww;
        return r;
    }
    __device__ __forceinline__ int64_t entry(int d, int dt, int dh) const
    {
        return d < dt ? t0 + static_cast<int64_t>(d / 2) * T
                      : (d < dt + dh ? h0 + static_cast<int64_t>((d - dt) / 2) * Hh
                                     : w0 + static_cast<int64_t>((d - dt - dh) / 2) * Ww);
    }
};

// The 3D RoPE table: (cos, sin) per (axis, position, pair) in fp64 (tab64,
// two doubles per entry) and their fp32 roundings (tab32, one float2 per
// entry), laid out as RopeGeom describes.
struct RopeTabs {
    const double *t64;
    const float2 *t32;
};

// tab64[2e], tab64[2e+1] = cos, sin of every table entry e, and tab32[e]
// their fp32 roundings (grid-stride; layout of RopeRowEntries).
__global__ void rope_table_kernel(double *__restrict__ tab64, float2 *__restrict__ tab32, RopeGeom g,
                                  const __grid_constant__ RopeFreqs fr)
{
    const int64_t n = g.entries();
    const int64_t base_h = static_cast<int64_t>(g.T) * (g.dt / 2);
    const int64_t base_w = base_h + static_cast<int64_t>(g.Hh) * (g.dh / 2);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n; e += stride) {
        int pos, pair;   // pair: index of the pair within the head dimension
        if (e < base_h) {
            pos = static_cast<int>(e % g.T); pair = static_cast<int>(e / g.T);
        } else if (e < base_w) {
            pos = static_cast<int>((e - base_h) % g.Hh);
            pair = g.dt / 2 + static_cast<int>((e - base_h) / g.Hh);
        } else {
            pos = static_cast<int>((e - base_w) % g.Ww);
            pair = (g.dt + g.dh) / 2 + static_cast<int>((e - base_w) / g.Ww);
        }
        double c, s;
        rope_angle(pos, fr.f[pair], c, s);
        tab64[2 * e] = c;
        tab64[2 * e + 1] = s;
        tab32[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
    }
}

// The four pairs of a 16-byte chunk: fp32 with one certificate for the whole
// chunk; if any pair is not certified (rare: the check fails near a bf16
// rounding boundary), the chunk is
// redone in fp64 from the fp64 cosines and sines.
__device__ __forceinline__ uint4 rotate_chunk_f32(uint4 v, const float2 (&cs)[4], const double (&c64)[4],
                                                  const double (&s64)[4])
{
    uint4 r;
    bool ok = rotate_pair_f32(v.x, cs[0].x, cs[0].y, r.x);
    ok &= rotate_pair_f32(v.y, cs[1].x, cs[1].y, r.y);
    ok &= rotate_pair_f32(v.z, cs[2].x, cs[2].y, r.z);
    ok &= rotate_pair_f32(v.w, cs[3].x, cs[3].y, r.w);
    if (__builtin_expect(!ok, 0))
        r = make_uint4(rotate_pair(v.x, c64[0], s64[0]), rotate_pair(v.y, c64[1], s64[1]),
                       rotate_pair(v.z, c64[2], s64[2]), rotate_pair(v.w, c64[3], s64[3]));
    return r;
}

// Walk rows [r0, r1) of one 16-byte chunk (element offset `off` in a row of
// `row_stride` elements): dst row r = rot(src row r), four rows at a time
// with the next four rows' loads issued before the current four are stored.
template <typename Rot>
__device__ __forceinline__ void rope_walk_rows(const uint16_t *src, uint16_t *dst, int64_t r0, int64_t r1,
                                               int64_t row_stride, int64_t off, Rot rot)
{
    auto ld = [&](int64_t r) { return *reinterpret_cast<const uint4 *>(src + r * row_stride + off); };
    uint4 cur[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (r0 + u < r1) cur[u] = ld(r0 + u);
    for (int64_t r = r0; r < r1; r += 4) {
        uint4 nxt[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (r + 4 + u < r1) nxt[u] = ld(r + 4 + u);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (r + u < r1) *reinterpret_cast<uint4 *>(dst + (r + u) * row_stride + off) = rot(cur[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u) cur[u] = nxt[u];
    }
}

// dst = RoPE(src) for `rows` rows of S x D (out of place), from the table.
// Thread = (token, 16-byte chunk) x one group of `rows_per_group` rows
// (blockIdx.y): the chunk's four table entries are read once per group.
__global__ void __launch_bounds__(128, 6) rope_apply_kernel(const uint16_t *__restrict__ src,
                                                            uint16_t *__restrict__ dst, int64_t rows, int S, int D,
                                                            RopeGeom g, RopeTabs tab, int rows_per_group)
{
    const int chunks = D >> 3;
    const int64_t per_row = static_cast<int64_t>(S) * chunks;
    const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (t >= per_row) return;
    const int n = static_cast<int>(t / chunks);
    const int c = static_cast<int>(t % chunks);
    const RopeRowEntries re = RopeRowEntries::of(g, n);
    int64_t e[4];
    float2 cs[4];
    double c64[4], s64[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        e[p] = re.entry(c * 8 + 2 * p, g.dt, g.dh);
        cs[p] = __ldg(tab.t32 + e[p]);
        c64[p] = __ldg(tab.t64 + 2 * e[p]);
        s64[p] = __ldg(tab.t64 + 2 * e[p] + 1);
    }
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_group;
    const int64_t r1 = r0 + rows_per_group < rows ? r0 + rows_per_group : rows;
    rope_walk_rows(src, dst, r0, r1, static_cast<int64_t>(S) * D, t * 8, [&](uint4 v) {
        return rotate_chunk_f32(v, cs, c64, s64);
    });
}

// In place on q and k: thread = (token, 16-byte chunk) x one group of rows
// (blockIdx.y in [0, 2*groups): groups of q's rows, then of k's). The four
// angles come from fp64 sincos once per thread. inverse: the transposed
// rotation (sine negated), the RoPE's gradient. n0: position of token 0 of
// this sequence shard on the latent grid.
__global__ void __launch_bounds__(128, 7) rope3d_kernel(uint16_t *__restrict__ q, uint16_t *__restrict__ k,
                                                        int64_t rows, int S, int Hh, int Ww, int D,
                                                        const __grid_constant__ RopeFreqs fr, bool inverse, int n0,
                                                        int rows_per_group, int groups)
{
    const int chunks = D >> 3;
    const int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (gid >= static_cast<int64_t>(S) * chunks) return;
    const int which = static_cast<int>(blockIdx.y) / groups;   // 0: q, 1: k
    uint16_t *x = which == 0 ? q : k;
    if (x == nullptr) return;
    const int n = static_cast<int>(gid / chunks);
    const int c = static_cast<int>(gid % chunks);
    const int tok = n0 + n;   // position on the latent grid
    const int pt = tok / (Hh * Ww), ph = (tok / Ww) % Hh, pw = tok % Ww;
    const int dh = 2 * (D / 6);
    const int dt = D - 2 * dh;
    double cs[4], sn[4];
    float2 cs2[4];   // their fp32 roundings
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int d = c * 8 + 2 * p;
        rope_angle(d < dt ? pt : (d < dt + dh ? ph : pw), fr.f[d / 2], cs[p], sn[p]);
        if (inverse) sn[p] = -sn[p];
        cs2[p] = make_float2(static_cast<float>(cs[p]), static_cast<float>(sn[p]));
    }
    const int64_t r0 = static_cast<int64_t>(blockIdx.y % groups) * rows_per_group;
    const int64_t r1 = r0 + rows_per_group < rows ? r0 + rows_per_group : rows;
    rope_walk_rows(x, x, r0, r1, static_cast<int64_t>(S) * D, static_cast<int64_t>(n) * D + c * 8, [&](uint4 v) {
        return rotate_chunk_f32(v, cs2, cs, sn);
    });
}

}  // namespace regen
