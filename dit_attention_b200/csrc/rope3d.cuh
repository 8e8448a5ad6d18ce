// rope3d.cuh -- 3D rotary position embedding of Q and K, in place (sm_100a).
//
// The ReGenVC decoder's DiT matches the Wan2.1-Fun-Control architecture (blog
// page, "Methodology -- deep read"), whose attention rotates Q and K by a 3D
// RoPE over the latent (t, h, w) grid. Reading used (the pages print no
// formula): token n = (t*Hh + y)*Ww + x; head-dim blocks t, h, w of widths
// D - 4*floor(D/6), 2*floor(D/6), 2*floor(D/6); pair (2j, 2j+1) of a block of
// width d turns by pos * theta^(-2j/d).
//
// HBM-bound: every element is read and written once. One thread owns one
// 16-byte chunk (4 pairs) of one token's row; it evaluates its 4 angles once
// (fp64 sincos) and then walks the same chunk through every (batch, head) row
// of Q and then of K, so the trigonometry is amortised over 2*B*H rows.
// Adjacent threads own adjacent chunks of a row: each warp access is two
// contiguous 256-byte rows. The rotation is done in fp64 and rounded once to
// bf16 (one direct fp64 -> bf16 conversion, nearest-even).
#pragma once

#include <stdint.h>

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

// cos and sin of pos * theta^(-local/width) for the pair starting at
// dimension `local` of an axis block of `width` dimensions (fp64).
__device__ __forceinline__ void rope_angle(int pos, int local, int width, double theta, double &c, double &s)
{
    const double freq = pow(theta, -static_cast<double>(local) / static_cast<double>(width));
    sincos(static_cast<double>(pos) * freq, &s, &c);
}

// Geometry of the 3D RoPE for a latent grid and head dim: axis blocks t, h, w
// of widths dt, dh, dh; table of (cos, sin) per (axis, position, pair) laid
// out as [T][dt/2] then [Hh][dh/2] then [Ww][dh/2] entries of two doubles.
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

// tab[2e], tab[2e+1] = cos, sin of every table entry e (grid-stride).
__global__ void rope_table_kernel(double *__restrict__ tab, RopeGeom g, double theta)
{
    const int64_t n = g.entries();
    const int64_t base_h = static_cast<int64_t>(g.T) * (g.dt / 2);
    const int64_t base_w = base_h + static_cast<int64_t>(g.Hh) * (g.dh / 2);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n; e += stride) {
        int pos, j, width;
        if (e < base_h) {
            pos = static_cast<int>(e / (g.dt / 2)); j = static_cast<int>(e % (g.dt / 2)); width = g.dt;
        } else if (e < base_w) {
            pos = static_cast<int>((e - base_h) / (g.dh / 2)); j = static_cast<int>((e - base_h) % (g.dh / 2));
            width = g.dh;
        } else {
            pos = static_cast<int>((e - base_w) / (g.dh / 2)); j = static_cast<int>((e - base_w) % (g.dh / 2));
            width = g.dh;
        }
        double c, s;
        rope_angle(pos, 2 * j, width, theta, c, s);
        tab[2 * e] = c;
        tab[2 * e + 1] = s;
    }
}

// Rotate the 16-byte chunk holding dimensions [8c, 8c + 8) of token n's row.
__device__ __forceinline__ uint4 rotate_chunk(uint4 v, int c, int n, const RopeGeom &g,
                                              const double *__restrict__ tab)
{
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int64_t e = g.entry(n, c * 8 + 2 * p);
        w[p] = rotate_pair(w[p], __ldg(tab + 2 * e), __ldg(tab + 2 * e + 1));
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// dst = RoPE(src) for `rows` rows of S x D (out of place), from the table.
__global__ void rope_apply_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int64_t rows, int S,
                                  int D, RopeGeom g, const double *__restrict__ tab)
{
    // One thread per (token, 16-byte chunk): the chunk's four (cos, sin) pairs
    // are read from the table once and applied to that chunk of every row
    // (consecutive threads, consecutive chunks of one row: coalesced).
    const int chunks = D >> 3;
    const int64_t per_row = static_cast<int64_t>(S) * chunks;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < per_row; t += stride) {
        const int n = static_cast<int>(t / chunks);
        const int c = static_cast<int>(t % chunks);
        double cs[4], sn[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int64_t e = g.entry(n, c * 8 + 2 * p);
            cs[p] = __ldg(tab + 2 * e);
            sn[p] = __ldg(tab + 2 * e + 1);
        }
        auto rot = [&](uint4 v) {
            return make_uint4(rotate_pair(v.x, cs[0], sn[0]), rotate_pair(v.y, cs[1], sn[1]),
                              rotate_pair(v.z, cs[2], sn[2]), rotate_pair(v.w, cs[3], sn[3]));
        };
        int64_t r = 0;
        for (; r + 4 <= rows; r += 4) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = src[(r + u) * per_row + t];
#pragma unroll
            for (int u = 0; u < 4; ++u) dst[(r + u) * per_row + t] = rot(v[u]);
        }
        for (; r < rows; ++r) dst[r * per_row + t] = rot(src[r * per_row + t]);
    }
}

__global__ void rope3d_kernel(uint16_t *__restrict__ q, uint16_t *__restrict__ k, int64_t rows,
                              int S, int Hh, int Ww, int D, double theta, bool inverse, int n0)
{
    const int chunks = D >> 3;
    const int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (gid >= static_cast<int64_t>(S) * chunks) return;
    const int n = static_cast<int>(gid / chunks);
    const int c = static_cast<int>(gid % chunks);
    const int tok = n0 + n;   // position on the latent grid
    const int pos[3] = {tok / (Hh * Ww), (tok / Ww) % Hh, tok % Ww};
    const int dh = 2 * (D / 6);
    const int dt = D - 2 * dh;
    double cs[4], sn[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int d = c * 8 + 2 * p;
        int axis, local, width;
        if (d < dt) {
            axis = 0; local = d; width = dt;
        } else if (d < dt + dh) {
            axis = 1; local = d - dt; width = dh;
        } else {
            axis = 2; local = d - dt - dh; width = dh;
        }
        rope_angle(pos[axis], local, width, theta, cs[p], sn[p]);
        if (inverse) sn[p] = -sn[p];
    }
    const int64_t row_stride = static_cast<int64_t>(S) * D;
    const int64_t off = static_cast<int64_t>(n) * D + c * 8;
    for (int which = 0; which < 2; ++which) {
        uint16_t *x = which == 0 ? q : k;
        if (x == nullptr) continue;
        int64_t r = 0;
        for (; r + 4 <= rows; r += 4) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const uint4 *>(x + (r + u) * row_stride + off);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                v[u].x = rotate_pair(v[u].x, cs[0], sn[0]);
                v[u].y = rotate_pair(v[u].y, cs[1], sn[1]);
                v[u].z = rotate_pair(v[u].z, cs[2], sn[2]);
                v[u].w = rotate_pair(v[u].w, cs[3], sn[3]);
                *reinterpret_cast<uint4 *>(x + (r + u) * row_stride + off) = v[u];
            }
        }
        for (; r < rows; ++r) {
            uint4 v = *reinterpret_cast<const uint4 *>(x + r * row_stride + off);
            v.x = rotate_pair(v.x, cs[0], sn[0]);
            v.y = rotate_pair(v.y, cs[1], sn[1]);
            v.z = rotate_pair(v.z, cs[2], sn[2]);
            v.w = rotate_pair(v.w, cs[3], sn[3]);
            *reinterpret_cast<uint4 *>(x + r * row_stride + off) = v;
        }
    }
}

}  // namespace regen
