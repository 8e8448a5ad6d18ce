// lse_merge.cuh -- combine two partial attentions over disjoint key blocks.
//
// Ring attention (blog page, "Methodology -- deep read": Ring streams KV
// blocks around the GPUs; "Technical innovations": the result stays exact)
// computes attention over each KV block separately and combines the partial
// outputs through their log-sum-exp values:
//   m = max(lse_a, lse_b), w_a = e^(lse_a - m), w_b = e^(lse_b - m)
//   out = (w_a o_a + w_b o_b) / (w_a + w_b),   lse = m + ln(w_a + w_b)
// HBM-bound elementwise kernel: one thread per 16-byte chunk (8 values) of a
// row, the row weights computed in fp32 by every thread of the row (the two
// LSE loads are shared through L1). Grid-stride over rows * D/8 chunks.
#pragma once

#include <stdint.h>

namespace regen {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t merge_pair(uint32_t a, uint32_t b, float ca, float cb)
{
    const float lo = fmaf(ca, bf16_lo(a), cb * bf16_lo(b));
    const float hi = fmaf(ca, bf16_hi(a), cb * bf16_hi(b));
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__global__ void lse_merge_kernel(const uint4 *oa, const float *__restrict__ la,
                                 const uint4 *ob, const float *__restrict__ lb,
                                 uint4 *out, float *__restrict__ lse_out, int64_t rows, int D)
{
    const int chunks = D >> 3;
    const int64_t total = rows * chunks;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total; g += stride) {
        const int64_t r = g / chunks;
        const int c = static_cast<int>(g - r * chunks);
        const float a = __ldg(la + r);
        const float b = __ldg(lb + r);
        const float m = fmaxf(a, b);
        if (m == -INFINITY) {
            out[g] = make_uint4(0, 0, 0, 0);
            if (c == 0 && lse_out) lse_out[r] = -INFINITY;
            continue;
        }
        const float wa = expf(a - m);
        const float wb = expf(b - m);
        const float inv = 1.0f / (wa + wb);
        const float ca = wa * inv, cb = wb * inv;
        const uint4 xa = oa[g];
        const uint4 xb = ob[g];
        uint4 y;
        y.x = merge_pair(xa.x, xb.x, ca, cb);
        y.y = merge_pair(xa.y, xb.y, ca, cb);
        y.z = merge_pair(xa.z, xb.z, ca, cb);
        y.w = merge_pair(xa.w, xb.w, ca, cb);
        out[g] = y;
        if (c == 0 && lse_out) lse_out[r] = m + logf(wa + wb);
    }
}

}  // namespace regen
