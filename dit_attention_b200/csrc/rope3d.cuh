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
// bf16 (round to odd into fp32, then nearest-even into bf16, which equals one
// correct rounding).
#pragma once

#include <stdint.h>

namespace regen {

__device__ __forceinline__ double bf16_bits_to_double(uint32_t h16)
{
    return static_cast<double>(__uint_as_float(h16 << 16));
}

// Correctly rounded double -> bf16 (nearest, ties to even).
__device__ __forceinline__ uint32_t double_to_bf16_bits(double x)
{
    if (x != x) return 0x7FC0u;
    const float f = __double2float_rz(x);
    uint32_t b = __float_as_uint(f);
    if (static_cast<double>(f) != x) b |= 1u;  // sticky: round to odd
    b += 0x7FFFu + ((b >> 16) & 1u);
    return b >> 16;
}

__device__ __forceinline__ uint32_t rotate_pair(uint32_t packed, double c, double s)
{
    const double x0 = bf16_bits_to_double(packed & 0xFFFFu);
    const double x1 = bf16_bits_to_double(packed >> 16);
    const double y0 = x0 * c - x1 * s;
    const double y1 = x0 * s + x1 * c;
    return double_to_bf16_bits(y0) | (double_to_bf16_bits(y1) << 16);
}

// grid: ceil(S * D/8 / blockDim) blocks; x (q then k) has `rows` rows of S x D.
__global__ void rope3d_kernel(uint16_t *__restrict__ q, uint16_t *__restrict__ k, int64_t rows,
                              int S, int Hh, int Ww, int D, double theta)
{
    const int chunks = D >> 3;
    const int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (gid >= static_cast<int64_t>(S) * chunks) return;
    const int n = static_cast<int>(gid / chunks);
    const int c = static_cast<int>(gid % chunks);
    const int pos[3] = {n / (Hh * Ww), (n / Ww) % Hh, n % Ww};
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
        const double freq = pow(theta, -static_cast<double>(local) / static_cast<double>(width));
        sincos(static_cast<double>(pos[axis]) * freq, &sn[p], &cs[p]);
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
