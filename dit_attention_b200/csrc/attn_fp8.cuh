// attn_fp8.cuh -- the FP8 (OCP E4M3) variant of the attention forward for sm_100a.
//
// Not on the pages: an accuracy-for-speed variant of the exact attention the
// DiT computes (ReGenVC, blog page, "Technical innovations"). Q, K and V are
// quantised per block of 128 rows of one (b, h): x ~ code * s_block, codes in
// E4M3, s = amax / 448. Then, per 128-key block j of the online softmax:
//   S    = Q8 K8_j^T                     (tcgen05 kind::f8f6f4, fp32 accumulate)
//   s_ij = S * scale * sq * sk_j          (the block scales fold into the softmax multiplier)
//   P'   = 2^(s*log2(e) - m + b_j + 4),  b_j = log2(sv_j / sv_max) <= 0
//   O   += P'8 V8_j                       (P' rounded to E4M3 in TMEM)
//   l   += rowsum(P') 2^(-b_j - 4)       (the row sum of the unrounded, unscaled P)
// and out = O * sv_max / (2^4 l): folding V's per-block scale into the exponent keeps
// one accumulator. m moves when a block's max exceeds it by more than 4 (log2
// units), so P <= 2^4 and P' <= 2^8 < 448; the bias of 4 keeps probabilities
// down to ~2^-10 of the row max in E4M3's normal range (3 significant bits)
// instead of its subnormals. D = 128 only: a row of codes is exactly one
// 128-byte swizzle row.
// Structure as in the bf16 kernel (attn_fwd.cuh): two 128-row Q tiles per CTA
// sharing one S buffer in tensor memory, each with its own P8 and O; K and V
// from two producer warps; S and PV MMAs from two issuing threads.
#pragma once

#include "attn_fwd.cuh"
#include "ptx.cuh"

// Pairs of every 8 whose 2^x runs on the FMA pipe. On the 77-frame window 1 is
// the fastest, by about 0.5 % over 2; 2 and 3 measured equal, and 0, 4 and 5 slower.
#ifndef REGEN_FP8_EXP2_EMU_PER8
#define REGEN_FP8_EXP2_EMU_PER8 1
#endif

namespace regen {

// Two floats -> two E4M3 codes (round to nearest even, saturating): lo in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d)
{
    return pack_e4m3x2(a, b) | (pack_e4m3x2(c, d) << 16);
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f8f6f4 (E4M3 in, fp32 accumulate).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Same with A (K-major) read from tensor memory: 4 codes per 32-bit column.
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor, kind::f8f6f4 with E4M3 A/B (format 0) and fp32 D.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool b_mn_major)
{
    return (1u << 4)                                   // D format: f32
           | ((b_mn_major ? 1u : 0u) << 16)            // B major-ness (A, B formats 0 = E4M3)
           | (static_cast<uint32_t>(N >> 3) << 17)
           | (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------ quantiser ---

// One CTA (256 threads) per (b*h, 128-row block): amax over the block's rows x
// D, scale = amax / 448 and inv = 448 / amax in fp32 (1 and 1 for an all-zero
// block), codes = E4M3(x * inv). Rows past S are neither read nor written.
// codes [BH][S][D] bytes; scales [BH][nb], nb = ceil(S / 128).
template <int D>
__global__ void __launch_bounds__(256) quant_e4m3_kernel(const uint4 *__restrict__ x, uint2 *__restrict__ codes,
                                                         float *__restrict__ scales, int S, int nb)
{
    constexpr int CPR = D / 8;                 // 16-byte chunks per row
    constexpr int PER = 128 * CPR / 256;       // chunks per thread
    __shared__ float warp_max[8];
    const int bh = blockIdx.x / nb, b = blockIdx.x % nb;
    const int r0 = b * 128;
    const int64_t base = (static_cast<int64_t>(bh) * S + r0) * CPR;
    uint4 v[PER];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = threadIdx.x + i * 256;
        const bool in = r0 + c / CPR < S;
        v[i] = in ? x[base + c] : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            amax = fmax3(amax, fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xFFFF0000u)));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, warp_max[i]);
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 1.0f;
    if (threadIdx.x == 0) scales[blockIdx.x] = scale;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = threadIdx.x + i * 256;
        if (r0 + c / CPR >= S) continue;
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        auto lo = [&](int e) { return __fmul_rn(__uint_as_float(w[e] << 16), inv); };
        auto hi = [&](int e) { return __fmul_rn(__uint_as_float(w[e] & 0xFFFF0000u), inv); };
        codes[base + c] = make_uint2(pack_e4m3x4(lo(0), hi(0), lo(1), hi(1)), pack_e4m3x4(lo(2), hi(2), lo(3), hi(3)));
    }
}

// ------------------------------------------------------------- attention ---

struct Fp8Cfg {
    static constexpr int HD = 128;
    static constexpr int BM = 128, BN = 128;
    static constexpr int TILE_BYTES = 128 * 128;          // 128 rows x 128 codes
    static constexpr int OUT_HALF = 128 * 128;            // bf16 output: 128 rows x 64 values
    static constexpr int NS = 4;                          // K ring and V ring depth
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + 2 * TILE_BYTES;
    static constexpr int V_OFF = K_OFF + NS * TILE_BYTES;
    static constexpr int BAR_OFF = V_OFF + NS * TILE_BYTES;
    // q, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2], s_free, p_full[2],
    // pv_done[2], drain
    static constexpr int NBARS = 1 + 4 * NS + 7 + 1;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;  // abort flag, TMEM base, 8 warp maxima
    static constexpr int SMEM_BYTES = MISC_OFF + 48 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 384;
    static constexpr uint32_t REGS_LOW = 64;
    static constexpr uint32_t REGS_HIGH = 208;
    static constexpr int MIN_LAUNCH_REGS = 160;
    static constexpr int EMU_PER8 = REGEN_FP8_EXP2_EMU_PER8;
    static constexpr float STALE = 4.0f;   // max growth (log2) before m and O are rescaled
    static constexpr float BIAS = 4.0f;    // exponent bias of P' (STALE + BIAS = 8: P' <= 256)
};

template <bool NEG_SCALE>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                        const float *__restrict__ q_scale, const float *__restrict__ k_scale,
                        const float *__restrict__ v_scale, float *__restrict__ lse, int Sq, int Skv,
                        float scale_log2, uint64_t wait_limit_ns)
{
    using C = Fp8Cfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = sbase + C::BAR_OFF;
    const uint32_t bar_q = bar0;
    auto bar_k_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto bar_k_empty = [&](int s) { return bar0 + 8u * (1 + C::NS + s); };
    auto bar_v_full = [&](int s) { return bar0 + 8u * (1 + 2 * C::NS + s); };
    auto bar_v_empty = [&](int s) { return bar0 + 8u * (1 + 3 * C::NS + s); };
    auto bar_s_full = [&](int t) { return bar0 + 8u * (1 + 4 * C::NS + t); };
    const uint32_t bar_s_free = bar0 + 8u * (3 + 4 * C::NS);  // S copied out by a softmax warpgroup
    auto bar_p_full = [&](int t) { return bar0 + 8u * (4 + 4 * C::NS + t); };
    auto bar_pv_done = [&](int t) { return bar0 + 8u * (6 + 4 * C::NS + t); };
    const uint32_t bar_drain = bar0 + 8u * (8 + 4 * C::NS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::MISC_OFF + 8);
    float *warp_max = reinterpret_cast<float *>(smem + C::MISC_OFF + 16);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(bar_k_full(s), 1);
            mbar_init(bar_k_empty(s), 1);
            mbar_init(bar_v_full(s), 1);
            mbar_init(bar_v_empty(s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_s_full(t), 1);
            mbar_init(bar_p_full(t), 128);
            mbar_init(bar_pv_done(t), 1);
        }
        mbar_init(bar_s_free, 128);
        mbar_init(bar_drain, 2);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const WaitCtl wc{abort_flag, wait_limit_ns};
    const int nkv = (Skv + C::BN - 1) / C::BN;
    const int nqb = (Sq + C::BM - 1) / C::BM;   // 128-row blocks of Q (its scale blocks)
    const int npairs = (Sq + 2 * C::BM - 1) / (2 * C::BM);
    const int bh = static_cast<int>(blockIdx.x / npairs);
    const int q0 = static_cast<int>(blockIdx.x % npairs) * (2 * C::BM);

    if (warp < 4) {
    setmaxnreg_dec<C::REGS_LOW>();
    // Aborting producers wait (bounded) for their copies still in flight; the
    // two MMA issuers each commit to bar_drain (count 2) and wait for both
    // before TMEM is freed (same protocol as the bf16 kernel).
    const uint64_t drain_ns = wait_limit_ns > kDrainFloorNs ? wait_limit_ns : kDrainFloorNs;
    auto drain_copies = [&](uint32_t bar, uint32_t parity) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < drain_ns) {
        }
    };
    auto drain_mmas = [&]() {
        tc_commit(bar_drain);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar_drain, 0)) {
            if (global_timer_ns() - t0 > drain_ns) {
                record_timeout(SITE_DRAIN);
                break;
            }
        }
    };
    // Tensor-memory columns: S at 0 (the two tiles in turn), P8_t at 128 + t*32
    // (128 codes per row, 4 per column), O_t at 256 + t*128.
    auto tm_p = [&](int t) { return tmem + 128u + static_cast<uint32_t>(t) * 32u; };
    auto tm_o = [&](int t) { return tmem + 256u + static_cast<uint32_t>(t) * 128u; };
    if (warp == 0) {
        // ------------------------------------------- producer: Q, then K ---
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            const uint64_t keep = l2_policy_evict_last();
            const uint64_t once = l2_policy_evict_first();
            mbar_arrive_expect_tx(bar_q, 2 * C::TILE_BYTES);
            for (int t = 0; t < 2; ++t)
                tma_load_3d(sbase + C::Q_OFF + t * C::TILE_BYTES, &tm_q, bar_q, 0, q0 + t * C::BM, bh, once);
            int nk = 0;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % C::NS;
                ok = wait_phase(bar_k_empty(s), ((j / C::NS) & 1) ^ 1, SITE_PROD_K_EMPTY, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_k_full(s), C::TILE_BYTES);
                tma_load_3d(sbase + C::K_OFF + s * C::TILE_BYTES, &tm_k, bar_k_full(s), 0, j * C::BN, bh, keep);
                ++nk;
            }
            if (!ok) {
                for (int j = (nk > C::NS ? nk - C::NS : 0); j < nk; ++j)
                    drain_copies(bar_k_full(j % C::NS), (j / C::NS) & 1);
                drain_copies(bar_q, 0);
            }
        }
    } else if (warp == 3) {
        // ------------------------------------------------- producer: V ---
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            const uint64_t keep = l2_policy_evict_last();
            int nv = 0;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % C::NS;
                ok = wait_phase(bar_v_empty(s), ((j / C::NS) & 1) ^ 1, SITE_PROD_V_EMPTY, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_v_full(s), C::TILE_BYTES);
                tma_load_3d(sbase + C::V_OFF + s * C::TILE_BYTES, &tm_v, bar_v_full(s), 0, j * C::BN, bh, keep);
                ++nv;
            }
            if (!ok)
                for (int j = (nv > C::NS ? nv - C::NS : 0); j < nv; ++j)
                    drain_copies(bar_v_full(j % C::NS), (j / C::NS) & 1);
        }
    } else if (warp == 1) {
        // ----------------------------------------- MMA issuer: S = Q8 K8^T ---
        // S_t = Q_t K_j^T: K = 128 codes = one 128-byte swizzle row, 32 codes
        // (32 bytes) per MMA. bar_s_free's phases complete in the order S0(0),
        // S1(0), S0(1), ...: S1(j) waits for parity 0, S0(j+1) for parity 1.
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_e4m3_f32(128, 128, false);  // Q8 K8^T, both K-major
            auto issue_s = [&](int t, int s) {
                const uint32_t qa = sbase + C::Q_OFF + t * C::TILE_BYTES;
                const uint32_t kb = sbase + C::K_OFF + s * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss_f8(tmem, smem_desc_sw128(qa + kk * 32, 16, 1024), smem_desc_sw128(kb + kk * 32, 16, 1024),
                              IDESC_S, kk > 0 ? 1u : 0u);
            };
            bool ok = wait_phase(bar_q, 0, SITE_MMA_Q, wc);
            for (int j = 0; j < nkv && ok; ++j) {
                const int s = j % C::NS;
                ok = wait_phase(bar_k_full(s), (j / C::NS) & 1, SITE_MMA_K_FULL, wc);
                if (!ok) break;
                if (j > 0) {
                    ok = wait_phase(bar_s_free, 1, SITE_MMA_S_FREE, wc);  // S1(j-1) copied out
                    if (!ok) break;
                }
                tc_fence_after_sync();
                issue_s(0, s);
                tc_commit(bar_s_full(0));
                ok = wait_phase(bar_s_free, 0, SITE_MMA_S_FREE, wc);      // S0(j) copied out
                if (!ok) break;
                tc_fence_after_sync();
                issue_s(1, s);
                tc_commit(bar_s_full(1));
                tc_commit(bar_k_empty(s));
            }
            drain_mmas();
        }
        __syncwarp();
    } else {
        // ----------------------------------------- MMA issuer: O += P8 V8 ---
        // O_t += P8_t V8_j: 32 keys per MMA = 8 TMEM columns of P8 and 32 rows
        // (4096 bytes) of V, whose 128 codes per row are the N extent.
        if (lane == 0) {
            constexpr uint32_t IDESC_O = idesc_e4m3_f32(128, 128, true);   // P8 V8, V MN-major
            auto issue_pv = [&](int t, int s, bool acc) {
                const uint32_t vb = sbase + C::V_OFF + s * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts_f8(tm_o(t), tm_p(t) + kk * 8, smem_desc_sw128(vb + kk * 4096, C::TILE_BYTES, 1024), IDESC_O,
                              (acc || kk > 0) ? 1u : 0u);
            };
            bool ok = true;
            for (int j = 0; j < nkv && ok; ++j) {
                const int s = j % C::NS;
                ok = wait_phase(bar_v_full(s), (j / C::NS) & 1, SITE_MMA_V_FULL, wc);
                if (!ok) break;
                ok = wait_phase(bar_p_full(0), j & 1, SITE_MMA_P_FULL, wc);
                if (!ok) break;
                tc_fence_after_sync();
                issue_pv(0, s, j > 0);
                tc_commit(bar_pv_done(0));
                ok = wait_phase(bar_p_full(1), j & 1, SITE_MMA_P_FULL, wc);
                if (!ok) break;
                tc_fence_after_sync();
                issue_pv(1, s, j > 0);
                tc_commit(bar_pv_done(1));
                tc_commit(bar_v_empty(s));
            }
            drain_mmas();
        }
        __syncwarp();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    } else {
        setmaxnreg_inc<C::REGS_HIGH>();
        // -------------------------------------------- softmax + epilogue ---
        const int t = (warp - 4) >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t ts = tmem + lane_bits;                 // the shared S buffer
        const uint32_t tp = tmem + lane_bits + 128u + t * 32u;  // this tile's P8
        const uint32_t to = tmem + lane_bits + 256u + t * 128u;
        const int kv_tail = Skv - (nkv - 1) * C::BN;
        const float *ksc = k_scale + static_cast<int64_t>(bh) * nkv;
        const float *vsc = v_scale + static_cast<int64_t>(bh) * nkv;
        // sv_max over the head's V blocks (both warpgroups: 256 threads)
        {
            const int tid = threadIdx.x - 128;
            float mx = 0.f;
            for (int j = tid; j < nkv; j += 256) mx = fmaxf(mx, vsc[j]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            if (lane == 0) warp_max[warp - 4] = mx;
            named_bar_sync(3, 256);
        }
        float sv_max = warp_max[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) sv_max = fmaxf(sv_max, warp_max[i]);
        const float lg_svmax = __log2f(sv_max);
        const int qb = q0 / C::BM + t;  // this tile's Q scale block
        const float cq = scale_log2 * (qb < nqb ? q_scale[static_cast<int64_t>(bh) * nqb + qb] : 1.0f);
        float m = 0.f, l = 0.f;
        bool ok = true;
        float sk_next = ksc[0], sv_next = vsc[0];
        for (int j = 0; ok && j < nkv; ++j) {
            const float c = cq * sk_next;                         // multiplier of this block's raw S (log2 units)
            const float bj = __log2f(sv_next) - lg_svmax;         // <= 0
            if (j + 1 < nkv) {
                sk_next = ksc[j + 1];
                sv_next = vsc[j + 1];
            }
            ok = __all_sync(0xffffffffu, wait_phase(bar_s_full(t), j & 1, SITE_SM_S_FULL, wc));
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t sr[4][32];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tmem_ld_32x32b_x32(ts + cc * 32, sr[cc]);
            tmem_ld_wait();
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) reg_fence(sr[cc]);
            // S is in registers: the buffer may take the other tile's next S.
            tc_fence_before_sync();
            mbar_arrive(bar_s_free);
            bool grow = false;
            float alpha = 1.0f;
            auto block = [&](auto masked_tag) {
                constexpr bool MASKED = decltype(masked_tag)::value;
                auto S = [&](int x) { return __uint_as_float(sr[x >> 5][x & 31]); };
                if constexpr (MASKED) {
#pragma unroll
                    for (int x = 0; x < 128; ++x)
                        if (x >= kv_tail) sr[x >> 5][x & 31] = __float_as_uint(NEG_SCALE ? INFINITY : -INFINITY);
                }
                float acc[8];
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    const int x0 = a * 16;
                    float r = NEG_SCALE ? fmin3(S(x0), S(x0 + 1), S(x0 + 2)) : fmax3(S(x0), S(x0 + 1), S(x0 + 2));
#pragma unroll
                    for (int x = x0 + 3; x + 1 < x0 + 16; x += 2)
                        r = NEG_SCALE ? fmin3(r, S(x), S(x + 1)) : fmax3(r, S(x), S(x + 1));
                    r = NEG_SCALE ? fminf(r, S(x0 + 15)) : fmaxf(r, S(x0 + 15));
                    acc[a] = r;
                }
                const float mx = NEG_SCALE
                    ? fmin3(fmin3(acc[0], acc[1], acc[2]), fmin3(acc[3], acc[4], acc[5]), fminf(acc[6], acc[7]))
                    : fmax3(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], acc[5]), fmaxf(acc[6], acc[7]));
                const float mnew = mx * c;
                if (j == 0) {
                    m = mnew;
                } else if (mnew > m + C::STALE) {
                    grow = true;
                    alpha = ex2_approx(m - mnew);
                    m = mnew;
                    l *= alpha;
                }
                // P' = 2^(S c - m + b_j + 4); row sum of P' in fp32 before rounding; 4 codes per column.
                const uint64_t c2 = f2_pack(c, c);
                const uint64_t nm2 = f2_pack(bj + C::BIAS - m, bj + C::BIAS - m);
                uint64_t rs2[4] = {0, 0, 0, 0};
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 128; i += 4) {
                    float p[4];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int x = i + 2 * h;
                        float y0, y1;
                        f2_unpack(f2_fma(f2_pack(S(x), S(x + 1)), c2, nm2), y0, y1);
                        if (((i >> 1) + h) % 8 < C::EMU_PER8) {
                            exp2_poly_pair(y0, y1, p[2 * h], p[2 * h + 1]);
                        } else {
                            p[2 * h] = ex2_approx(y0);
                            p[2 * h + 1] = ex2_approx(y1);
                        }
                        if constexpr (MASKED) {
                            if (x >= kv_tail) p[2 * h] = 0.f;
                            if (x + 1 >= kv_tail) p[2 * h + 1] = 0.f;
                        }
                        rs2[((i >> 1) + h) & 3] = f2_add(rs2[((i >> 1) + h) & 3], f2_pack(p[2 * h], p[2 * h + 1]));
                    }
                    pk[i >> 2] = pack_e4m3x4(p[0], p[1], p[2], p[3]);
                }
                // P8_t and O_t are free once PV_t(j-1) has completed.
                if (j > 0) {
                    ok = __all_sync(0xffffffffu, wait_phase(bar_pv_done(t), (j - 1) & 1, SITE_SM_PV_DONE, wc));
                    if (!ok) return;
                    tc_fence_after_sync();
                }
                tmem_st_32x32b_x32(tp, pk);
                float r0, r1;
                f2_unpack(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])), r0, r1);
                l += (r0 + r1) * ex2_approx(-bj - C::BIAS);
            };
            if (j == nkv - 1 && kv_tail < C::BN)
                block(std::true_type{});
            else
                block(std::false_type{});
            if (!ok) break;
            if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(to + cc * 32, o);
                    tmem_ld_wait();
                    reg_fence(o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st_32x32b_x32(to + cc * 32, o);
                }
            }
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(bar_p_full(t));
        }
        if (ok) ok = __all_sync(0xffffffffu, wait_phase(bar_pv_done(t), (nkv - 1) & 1, SITE_SM_O_FULL, wc));
        // The output is staged in the K ring, tile t in stages 2t and 2t+1. The S
        // MMAs come from the other issuing thread: tile 1 saw every one of them
        // complete (its last S is the last one issued), tile 0 waits for that too.
        if (ok && t == 0) ok = __all_sync(0xffffffffu, wait_phase(bar_s_full(1), (nkv - 1) & 1, SITE_SM_O_FULL, wc));
        if (ok) {
            tc_fence_after_sync();
            // Epilogue: O * sv_max / (2^BIAS l) -> bf16 (P' carried the factor
            // 2^(b_j + BIAS) = 2^BIAS sv_j / sv_max), staged in the (now free) K ring
            // in the 128-byte swizzled layout of the bf16 output map, then TMA-stored.
            const float f = sv_max / (l * (1 << static_cast<int>(C::BIAS)));
            uint8_t *stage = smem + C::K_OFF + t * 2 * C::OUT_HALF;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(to + cc * 32, o);
                tmem_ld_wait();
                reg_fence(o);
                const int half = cc >> 1;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int chunk = (cc & 1) * 4 + g;
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(o[g * 8 + 0]) * f, __uint_as_float(o[g * 8 + 1]) * f);
                    w.y = pack_bf16x2(__uint_as_float(o[g * 8 + 2]) * f, __uint_as_float(o[g * 8 + 3]) * f);
                    w.z = pack_bf16x2(__uint_as_float(o[g * 8 + 4]) * f, __uint_as_float(o[g * 8 + 5]) * f);
                    w.w = pack_bf16x2(__uint_as_float(o[g * 8 + 6]) * f, __uint_as_float(o[g * 8 + 7]) * f);
                    *reinterpret_cast<uint4 *>(stage + half * C::OUT_HALF + row * 128 + ((chunk ^ (row & 7)) << 4)) = w;
                }
            }
            const int qrow = q0 + t * C::BM + row;
            if (lse != nullptr && qrow < Sq)
                lse[static_cast<int64_t>(bh) * Sq + qrow] = (m + __log2f(l)) * 0.69314718055994531f;
            fence_proxy_async_smem();
        }
        named_bar_sync(1 + t, 128);
        if (ok && warp == 4 + 4 * t && lane == 0 && q0 + t * C::BM < Sq) {
            for (int h = 0; h < 2; ++h)
                tma_store_3d(&tm_o, sbase + C::K_OFF + t * 2 * C::OUT_HALF + h * C::OUT_HALF, h * 64,
                             q0 + t * C::BM, bh);
            tma_store_commit();
            tma_store_wait_read_all();   // only the shared-memory reads must finish before the CTA exits
        }
        tc_fence_before_sync();
        __syncthreads();
    }
}

}  // namespace regen
