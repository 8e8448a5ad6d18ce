// attn_bwd.cuh -- gradients of exact softmax attention for sm_100a.
//
// The decoder is distilled into a student DiT (ReGenVC, blog page, "Technical
// innovations": distillation of the diffusion decoder), so its attention is
// trained and needs dQ, dK, dV. With s_ij = scale <q_i, k_j>, P = softmax_j(s),
// O = P V, an upstream dO and the forward's natural-log LSE:
//   P_ij    = exp(s_ij - lse_i)               (recomputed, exact up to rounding)
//   dP_ij   = <dO_i, v_j>
//   delta_i = <dO_i, O_i>                     (= sum_j P_ij dP_ij)
//   dS_ij   = P_ij (dP_ij - delta_i)          (softmax Jacobian)
//   dV_j = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j
// When the keys are split into blocks whose partial outputs were combined by
// their log-sum-exp (the Ring attention merge), passing the MERGED O and LSE
// gives each block's exact share: P above is then the block's slice of the
// global softmax, so dK, dV of the block are exact and the dQ shares add up.
//
// Three launches, none with atomics (so results are deterministic):
//   bwd_prep    delta and lse*log2(e) per query row into a padded workspace
//               [B*H][ceil(Sq/128)][2][128] floats (rows >= Sq: lse = +inf, delta = 0,
//               which makes their P exactly 0);
//   bwd_dkdv    one CTA per (b*h, 128-key tile); loops over all 128-row query
//               tiles with transposed tiles S^T = K Q^T and dP^T = V dO^T, so
//               that the key is the TMEM lane and dV += P^T dO, dK += dS^T Q
//               accumulate in tensor memory for the whole loop;
//   bwd_dq      one CTA per (b*h, 128-row query tile); loops over the key tiles
//               with S = Q K^T, dP = dO V^T and dQ += dS K.
// S and dP are computed twice (once per kernel): 7 tile products instead of
// the 5 the gradient needs, traded for no dQ reduction across CTAs.
#pragma once

#include <type_traits>

#include "attn_fwd.cuh"
#include "ptx.cuh"

namespace regen {

enum BwdWaitSite : uint32_t {
    SITE_BWD_PROD = 12,   // a producer waiting for a free stage
    SITE_BWD_MMA = 13,    // the MMA issuer waiting for operands, P or dS
    SITE_BWD_SM = 14,     // the elementwise warps waiting for S or dP
    SITE_BWD_ACC = 15,    // the epilogue waiting for the accumulators
    SITE_BWD_SMEM = 16,   // the dynamic shared memory did not start 1024-byte aligned
};

template <int HD>
struct BwdCfg {
    static constexpr int BM = 128;                   // query rows per tile
    static constexpr int BN = 128;                   // keys per tile
    static constexpr int HALVES = HD / 64;           // 128-byte column groups per row
    static constexpr int TILE_BYTES = 128 * HD * 2;  // one 128-row bf16 tile
    static constexpr int HALF_BYTES = 128 * 128;     // 128 rows x 128 bytes
    static constexpr int STAT_BYTES = 1024;          // lse2[128] then delta[128] of one query tile
    static constexpr int THREADS = 384;
    static constexpr uint32_t TMEM_COLS = 512;
    // Register split after setmaxnreg: producer / MMA warpgroup at REGS_LOW,
    // the two elementwise warpgroups at REGS_HIGH. (REGS_HIGH - R) * 256 <=
    // (R - REGS_LOW) * 128 needs R registers per thread at launch (the build
    // uses 168). dK/dV: 64 / 208 (R >= 160). dQ: 56 / 216 (R >= 163): its
    // elementwise loop spilled at 208, and 216 took its cycles from 7.45 M to
    // 7.32 M on 8 heads, where the same split made the dK/dV kernel slower
    // (9.77 M to 9.90 M).
    static constexpr uint32_t REGS_LOW = 64;
    static constexpr uint32_t REGS_HIGH = 208;
    static constexpr int MIN_LAUNCH_REGS = 160;
    static constexpr uint32_t B_REGS_LOW = 56;
    static constexpr uint32_t B_REGS_HIGH = 216;
    static constexpr int B_MIN_LAUNCH_REGS = 163;
    static constexpr int EMU_PER8 = REGEN_EXP2_EMU_PER8;

    // dK/dV kernel: K and V tiles resident; Q through an NQ-stage ring and dO with
    // the per-row stats through an ND-stage ring, both released after dK.
    // barriers: kv, q_full[NQ], q_empty[NQ], do_full[ND], do_empty[ND], x_full, x_free,
    // p_full, ds_full, dv_done, dk_done, drain
    // At D = 128, 3 + 2 stages need 231.6 KB: that fits only without slack for
    // aligning the base, so the kernel checks that the dynamic shared memory
    // starts on a 1024-byte boundary (it does when, as here, no static shared
    // memory precedes it) and refuses to run otherwise.
    static constexpr int A_NQ = (HD == 128) ? 3 : 4;
    static constexpr int A_ND = (HD == 128) ? 2 : 4;
    static constexpr int A_K_OFF = 0;
    static constexpr int A_V_OFF = TILE_BYTES;
    static constexpr int A_Q_OFF = 2 * TILE_BYTES;
    static constexpr int A_DO_OFF = A_Q_OFF + A_NQ * TILE_BYTES;
    static constexpr int A_ST_OFF = A_DO_OFF + A_ND * TILE_BYTES;
    static constexpr int A_BAR_OFF = A_ST_OFF + A_ND * STAT_BYTES;
    static constexpr int A_NBARS = 1 + 2 * A_NQ + 2 * A_ND + 7;
    static constexpr int A_MISC_OFF = A_BAR_OFF + A_NBARS * 8;
    static constexpr int A_SMEM_BYTES = A_MISC_OFF + 16;

    // dQ kernel: Q and dO resident, K and V through rings of NK and NV stages.
    static constexpr int B_NK = (HD == 128) ? 3 : 4;
    static constexpr int B_NV = (HD == 128) ? 2 : 4;
    static constexpr int B_Q_OFF = 0;
    static constexpr int B_DO_OFF = TILE_BYTES;
    static constexpr int B_K_OFF = 2 * TILE_BYTES;
    static constexpr int B_V_OFF = B_K_OFF + B_NK * TILE_BYTES;
    static constexpr int B_BAR_OFF = B_V_OFF + B_NV * TILE_BYTES;
    // qdo, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2], dp_full, ds_full, acc_full,
    // drain, dp_free, s_free[2]
    static constexpr int B_NBARS = 1 + 2 * B_NK + 2 * B_NV + 2 + 7;
    static constexpr int B_MISC_OFF = B_BAR_OFF + B_NBARS * 8;
    static constexpr int B_SMEM_BYTES = B_MISC_OFF + 16 + 1024;
};

// ----------------------------------------------------------------- prep ---

// ws[((bh * nq + t) * 2 + 0) * 128 + r] = lse * log2(e) of query row t*128 + r,
// ws[((bh * nq + t) * 2 + 1) * 128 + r] = <dO, O> of that row (fp32 sum of the
// bf16 products); rows >= Sq get +inf and 0. D/8 threads share one row (one
// 16-byte chunk each) and combine their partial sums with shuffles.
__global__ void attn_bwd_prep_kernel(const uint4 *__restrict__ out, const uint4 *__restrict__ dout,
                                     const float *__restrict__ lse, float *__restrict__ ws, int64_t BH, int Sq,
                                     int D, int nq)
{
    const int chunks = D >> 3;  // 8 or 16 lanes per row, a power of two
    const int64_t padded = static_cast<int64_t>(nq) * 128;
    const int64_t total = BH * padded * chunks;  // a multiple of 32: whole warps stay in step
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total; i += stride) {
        const int64_t prow = i / chunks;
        const int c = static_cast<int>(i % chunks);
        const int64_t bh = prow / padded;
        const int r = static_cast<int>(prow % padded);
        float acc = 0.f;
        if (r < Sq) {
            const int64_t g = (bh * Sq + r) * chunks + c;
            const uint4 o = out[g], d = dout[g];
            const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc = fmaf(__uint_as_float(ow[u] << 16), __uint_as_float(dw[u] << 16), acc);
                acc = fmaf(__uint_as_float(ow[u] & 0xFFFF0000u), __uint_as_float(dw[u] & 0xFFFF0000u), acc);
            }
        }
        for (int off = chunks >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, chunks);
        if (c == 0) {
            float *blk = ws + (bh * nq + r / 128) * 256;
            blk[r % 128] = r < Sq ? lse[bh * Sq + r] * 1.4426950408889634f : INFINITY;
            blk[128 + r % 128] = r < Sq ? acc : 0.f;
        }
    }
}

// Elementwise helpers shared by the two gradient kernels. p holds 32 logits
// on entry (as fp32 bits) and P on exit; nl2 = (-lse2, -lse2) for one row or
// the per-column pairs.
template <int EMU>
__device__ __forceinline__ void probs_pair(uint32_t &s0, uint32_t &s1, uint64_t c2, uint64_t nl2, int pair_idx)
{
    float y0, y1;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(s0), __uint_as_float(s1)), c2, nl2), y0, y1);
    float p0, p1;
    if (pair_idx % 8 < EMU) {
        exp2_poly_pair(y0, y1, p0, p1);
    } else {
        p0 = ex2_approx(y0);
        p1 = ex2_approx(y1);
    }
    s0 = __float_as_uint(p0);
    s1 = __float_as_uint(p1);
}

// ------------------------------------------------------------- dK / dV ---

// One CTA = one (b*h, 128-key tile). Warp roles as in the forward kernel:
// warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps 4-7 and 8-11
// the elementwise warpgroups; warpgroup w owns query columns [64w, 64w + 64)
// of the transposed tiles, thread = key row (TMEM lane).
// TMEM columns: X [0,128) holds S^T(i), then dP^T(i) (fp32; warpgroup w reads
// [64w, 64w+64)); P^T [128,192) and dS^T [192,256) as bf16 (warpgroup w at
// +32w); dV [256, 256+HD), dK [256+HD, 256+2HD).
// The elementwise warps keep P in registers from the moment they copy S^T out,
// so S^T and dP^T never need tensor memory at the same time, and P^T, dS^T
// have columns of their own. Two MMA issuers:
//   warp 1:  S^T(i) = K Q(i)^T, then dP^T(i) = V dO(i)^T, each into X once the
//            elementwise warps have copied the previous product out;
//   warp 2:  dV += P^T(i) dO(i) once P^T(i) is stored, dK += dS^T(i) Q(i) once
//            dS^T(i) is stored.
// So S^T(i+1) need not wait for dV(i): the elementwise warps wait for dV(i-1)
// (dK(i-1)) only before storing P^T(i) (dS^T(i)).
// ACCUM: dK and dV are added to the bf16 values already in dk_old / dv_old
// (the output buffers themselves: each CTA reads its own key rows before its
// store), for gradients accumulated over several query blocks.
// Two key sources (the joint softmax over two key buffers): the grid covers
// the key tiles of the first source (Skv keys; tm_k, tm_v, tm_dk, tm_dv,
// dk_old, dv_old), then those of the second (Skv2 keys; the *2 arguments).
// Each CTA's work depends only on its own key tile and the per-row
// statistics, so the two sources' tiles are computed as in separate calls.
// Skv2 = 0: one source (the *2 maps are not read).
template <int HD, bool ACCUM>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                         const __grid_constant__ CUtensorMap tm_k2, const __grid_constant__ CUtensorMap tm_v2,
                         const __grid_constant__ CUtensorMap tm_dk2, const __grid_constant__ CUtensorMap tm_dv2,
                         const float *__restrict__ ws, int Sq, int Skv, int Skv2, float scale, float scale_log2,
                         uint64_t wait_limit_ns, const uint16_t *dk_old, const uint16_t *dv_old,
                         const uint16_t *dk_old2, const uint16_t *dv_old2)
{
    using C = BwdCfg<HD>;
    constexpr int NQ = C::A_NQ, ND = C::A_ND;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw;
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (sbase & 1023u) {  // uniform over the CTA: nothing has been initialised yet
        if (threadIdx.x == 0 && atomicCAS(&g_regen_err, 0, -2 /* REGEN_ERR_UNSUPPORTED */) == 0)
            g_regen_err_site = SITE_BWD_SMEM;
        return;
    }

    const uint32_t bar0 = sbase + C::A_BAR_OFF;
    const uint32_t bar_kv = bar0;
    auto bar_q_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto bar_q_empty = [&](int s) { return bar0 + 8u * (1 + NQ + s); };
    auto bar_do_full = [&](int s) { return bar0 + 8u * (1 + 2 * NQ + s); };
    auto bar_do_empty = [&](int s) { return bar0 + 8u * (1 + 2 * NQ + ND + s); };
    constexpr int NS = NQ + ND;  // barrier slots taken by the two rings
    // X's products complete bar_x_full in the order S^T(0), dP^T(0), S^T(1), ...
    // (parity 0 for S^T, 1 for dP^T) and their copy-outs complete bar_x_free in
    // the same order: no waiter can fall two phases behind, since the next
    // product is issued only after the copy-out of the previous one.
    const uint32_t bar_x_full = bar0 + 8u * (1 + 2 * NS);
    const uint32_t bar_x_free = bar0 + 8u * (2 + 2 * NS);
    const uint32_t bar_p_full = bar0 + 8u * (3 + 2 * NS);
    const uint32_t bar_ds_full = bar0 + 8u * (4 + 2 * NS);
    const uint32_t bar_dv_done = bar0 + 8u * (5 + 2 * NS);
    const uint32_t bar_dk_done = bar0 + 8u * (6 + 2 * NS);
    const uint32_t bar_drain = bar0 + 8u * (7 + 2 * NS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::A_MISC_OFF);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::A_MISC_OFF + 8);

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < NQ; ++s) {
            mbar_init(bar_q_full(s), 1);
            mbar_init(bar_q_empty(s), 1);
        }
        for (int s = 0; s < ND; ++s) {
            mbar_init(bar_do_full(s), 1);
            mbar_init(bar_do_empty(s), 1);
        }
        mbar_init(bar_x_full, 1);
        mbar_init(bar_x_free, 256);
        mbar_init(bar_p_full, 256);
        mbar_init(bar_ds_full, 256);
        mbar_init(bar_dv_done, 1);
        mbar_init(bar_dk_done, 1);
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
    const int nq = (Sq + C::BM - 1) / C::BM;
    const int nkv1 = (Skv + C::BN - 1) / C::BN;
    const int tiles = nkv1 + (Skv2 + C::BN - 1) / C::BN;   // key tiles of one (b, h), both sources
    const int bh = static_cast<int>(blockIdx.x / tiles);
    const int tile = static_cast<int>(blockIdx.x % tiles);
    const bool second = tile >= nkv1;                        // this CTA's key tile is the second source's
    const int key0 = (second ? tile - nkv1 : tile) * C::BN;  // first key of the tile within its source
    const int skv = second ? Skv2 : Skv;
    const CUtensorMap *map_k = second ? &tm_k2 : &tm_k;
    const CUtensorMap *map_v = second ? &tm_v2 : &tm_v;

    if (warp < 4) {
    setmaxnreg_dec<C::REGS_LOW>();
    const uint64_t drain_ns = wait_limit_ns > kDrainFloorNs ? wait_limit_ns : kDrainFloorNs;
    // Aborting: a producer waits (bounded) for its copies still in flight -- at
    // most the last stages of its ring -- before the CTA exits.
    auto drain_copies = [&](uint32_t bar, uint32_t parity) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < drain_ns) {
        }
    };
    if (warp == 0) {
        // -------------------------------------- producer: K, V, then Q ---
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(map_k);
            tma_prefetch_desc(map_v);
            const uint64_t keep = l2_policy_evict_last();   // Q: re-read by every key tile of the head
            const uint64_t once = l2_policy_evict_first();  // K, V: read by this CTA only
            mbar_arrive_expect_tx(bar_kv, 2 * C::TILE_BYTES);
            for (int h = 0; h < C::HALVES; ++h) {
                tma_load_3d(sbase + C::A_K_OFF + h * C::HALF_BYTES, map_k, bar_kv, h * 64, key0, bh, once);
                tma_load_3d(sbase + C::A_V_OFF + h * C::HALF_BYTES, map_v, bar_kv, h * 64, key0, bh, once);
            }
            int n = 0;  // query tiles issued
            bool ok = true;
            for (int i = 0; i < nq; ++i) {
                const int s = i % NQ;
                ok = wait_phase(bar_q_empty(s), ((i / NQ) & 1) ^ 1, SITE_BWD_PROD, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_q_full(s), C::TILE_BYTES);
                for (int h = 0; h < C::HALVES; ++h)
                    tma_load_3d(sbase + C::A_Q_OFF + s * C::TILE_BYTES + h * C::HALF_BYTES, &tm_q, bar_q_full(s),
                                h * 64, i * C::BM, bh, keep);
                ++n;
            }
            if (!ok) {
                for (int i = (n > NQ ? n - NQ : 0); i < n; ++i) drain_copies(bar_q_full(i % NQ), (i / NQ) & 1);
                drain_copies(bar_kv, 0);
            }
        }
    } else if (warp == 3) {
        // ------------------------------------- producer: dO and the stats ---
        if (lane == 0) {
            tma_prefetch_desc(&tm_do);
            const uint64_t keep = l2_policy_evict_last();   // dO: re-read by every key tile of the head
            int n = 0;
            bool ok = true;
            for (int i = 0; i < nq; ++i) {
                const int s = i % ND;
                ok = wait_phase(bar_do_empty(s), ((i / ND) & 1) ^ 1, SITE_BWD_PROD, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_do_full(s), C::TILE_BYTES + C::STAT_BYTES);
                for (int h = 0; h < C::HALVES; ++h)
                    tma_load_3d(sbase + C::A_DO_OFF + s * C::TILE_BYTES + h * C::HALF_BYTES, &tm_do, bar_do_full(s),
                                h * 64, i * C::BM, bh, keep);
                bulk_load_1d(sbase + C::A_ST_OFF + s * C::STAT_BYTES,
                             ws + (static_cast<int64_t>(bh) * nq + i) * 256, C::STAT_BYTES, bar_do_full(s));
                ++n;
            }
            if (!ok)
                for (int i = (n > ND ? n - ND : 0); i < n; ++i) drain_copies(bar_do_full(i % ND), (i / ND) & 1);
        }
    } else {
        // ------------------------------------------- MMA issuers (warps 1, 2) ---
        if (lane == 0) {
            constexpr uint32_t IDESC_T = idesc_bf16_f32(128, 128, false);  // K Q^T, V dO^T: both K-major
            constexpr uint32_t IDESC_G = idesc_bf16_f32(128, HD, true);    // P^T dO, dS^T Q: B MN-major
            const uint32_t tm_x = tmem, tm_pt = tmem + 128u, tm_dst = tmem + 192u;
            const uint32_t tm_dv = tmem + 256u, tm_dk = tmem + 256u + HD;
            const uint32_t k_s = sbase + C::A_K_OFF, v_s = sbase + C::A_V_OFF;
            auto q_s = [&](int i) { return sbase + C::A_Q_OFF + (i % NQ) * C::TILE_BYTES; };
            auto do_s = [&](int i) { return sbase + C::A_DO_OFF + (i % ND) * C::TILE_BYTES; };
            bool ok = true;
            if (warp == 1) {
                // D[128 x 128] = A[128 x HD] B[128 x HD]^T, both operands row-major
                // 128-byte-swizzled tiles: K steps of 16 (32 bytes) inside a swizzle row,
                // the second 64-column half HALF_BYTES on.
                auto issue_t = [&](uint32_t a, uint32_t b) {
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk) {
                        const uint32_t off = (kk / 4) * C::HALF_BYTES + (kk % 4) * 32;
                        mma_ss(tm_x, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024),
                               IDESC_T, kk > 0 ? 1u : 0u);
                    }
                };
                ok = wait_phase(bar_kv, 0, SITE_BWD_MMA, wc);
                for (int i = 0; i < nq && ok; ++i) {
                    ok = wait_phase(bar_q_full(i % NQ), (i / NQ) & 1, SITE_BWD_MMA, wc);
                    if (!ok) break;
                    if (i > 0) {
                        ok = wait_phase(bar_x_free, 1, SITE_BWD_MMA, wc);  // dP^T(i-1) copied out
                        if (!ok) break;
                    }
                    tc_fence_after_sync();
                    issue_t(k_s, q_s(i));
                    tc_commit(bar_x_full);
                    ok = wait_phase(bar_x_free, 0, SITE_BWD_MMA, wc);      // S^T(i) copied out
                    if (!ok) break;
                    ok = wait_phase(bar_do_full(i % ND), (i / ND) & 1, SITE_BWD_MMA, wc);
                    if (!ok) break;
                    tc_fence_after_sync();
                    issue_t(v_s, do_s(i));
                    tc_commit(bar_x_full);
                }
            } else {
                // D[128 x HD] += A[128 keys x 128 queries] (bf16 in TMEM) B[128 queries x HD]:
                // query steps of 16 = 8 TMEM columns; warpgroup w's 64 queries sit at
                // column 32w of the operand; B rows (queries) 128-byte swizzled, 16 rows
                // = 2048 bytes.
                auto issue_g = [&](uint32_t d, uint32_t a, uint32_t b, bool acc) {
#pragma unroll
                    for (int kk = 0; kk < C::BM / 16; ++kk)
                        mma_ts(d, a + 32u * (kk >> 2) + 8u * (kk & 3),
                               smem_desc_sw128(b + kk * 2048, C::HALF_BYTES, 1024), IDESC_G,
                               (acc || kk > 0) ? 1u : 0u);
                };
                for (int i = 0; i < nq && ok; ++i) {
                    // both stages are complete by now (S^T(i) and dP^T(i) read them)
                    ok = wait_phase(bar_do_full(i % ND), (i / ND) & 1, SITE_BWD_MMA, wc);
                    if (ok) ok = wait_phase(bar_q_full(i % NQ), (i / NQ) & 1, SITE_BWD_MMA, wc);
                    if (!ok) break;
                    ok = wait_phase(bar_p_full, i & 1, SITE_BWD_MMA, wc);
                    if (!ok) break;
                    tc_fence_after_sync();
                    issue_g(tm_dv, tm_pt, do_s(i), i > 0);
                    tc_commit(bar_dv_done);
                    ok = wait_phase(bar_ds_full, i & 1, SITE_BWD_MMA, wc);
                    if (!ok) break;
                    tc_fence_after_sync();
                    issue_g(tm_dk, tm_dst, q_s(i), i > 0);
                    tc_commit(bar_dk_done);
                    // every product that read the two stages has completed: S^T(i)
                    // and dP^T(i) before the elementwise warps could form dS^T(i),
                    // which also finished reading the stats in the dO stage
                    tc_commit(bar_q_empty(i % NQ));
                    tc_commit(bar_do_empty(i % ND));
                }
            }
            // Each issuer commits to bar_drain (count 2) and waits for both, so
            // that nothing runs on the tensor core when TMEM is freed.
            tc_commit(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0)) {
                if (global_timer_ns() - t0 > drain_ns) {
                    record_timeout(SITE_DRAIN);
                    break;
                }
            }
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
        // ------------------------------------------------- elementwise ---
        const int w = (warp - 4) >> 2;     // query columns [64w, 64w + 64)
        const int quad = warp & 3;
        const int krow = quad * 32 + lane;  // key row inside the tile
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tx = tmem + lane_bits + 64u * w;           // this warpgroup's columns of X
        const uint32_t tpt = tmem + lane_bits + 128u + 32u * w;   // its P^T
        const uint32_t tds = tmem + lane_bits + 192u + 32u * w;   // its dS^T
        const uint64_t c2 = f2_pack(scale_log2, scale_log2);
        bool ok = true;
        for (int i = 0; ok && i < nq; ++i) {
            const float *st = reinterpret_cast<const float *>(smem + C::A_ST_OFF + (i % ND) * C::STAT_BYTES);
            const float4 *lse4 = reinterpret_cast<const float4 *>(st + 64 * w);         // two column pairs each
            const float4 *dlt4 = reinterpret_cast<const float4 *>(st + 128 + 64 * w);
            ok = __all_sync(0xffffffffu, wait_phase(bar_x_full, 0, SITE_BWD_SM, wc));   // S^T(i)
            // the stats were written by the bulk copy: observe its barrier too
            // (complete by now; the stage is refilled only after dK(i))
            if (ok) ok = __all_sync(0xffffffffu, wait_phase(bar_do_full(i % ND), (i / ND) & 1, SITE_BWD_SM, wc));
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t pr[2][32];
            tmem_ld_32x32b_x32(tx, pr[0]);
            tmem_ld_32x32b_x32(tx + 32, pr[1]);
            tmem_ld_wait();
            reg_fence(pr[0]);
            reg_fence(pr[1]);
            tc_fence_before_sync();
            mbar_arrive(bar_x_free);
            // P^T = 2^(S^T * scale*log2(e) - lse2[column]); rows past Sq have lse2 = +inf.
            // Computed in quarters of 8 column pairs. dP^T(i) is copied out of X as
            // soon as a non-blocking test after a quarter finds it ready (a blocking
            // wait only after the last), so that X takes S^T(i+1) as early as possible.
            uint32_t pk[2][16];
            uint32_t dr[2][32];
            bool have_dp = false;
            auto probs_quarter = [&](int qtr) {
                const int hv = qtr >> 1;
#pragma unroll
                for (int c = (qtr & 1) * 8; c < (qtr & 1) * 8 + 8; c += 2) {
                    const float4 l = lse4[hv * 8 + c / 2];
                    probs_pair<C::EMU_PER8>(pr[hv][2 * c], pr[hv][2 * c + 1], c2, f2_pack(-l.x, -l.y), c);
                    probs_pair<C::EMU_PER8>(pr[hv][2 * c + 2], pr[hv][2 * c + 3], c2, f2_pack(-l.z, -l.w), c + 1);
                    pk[hv][c] = pack_bf16x2(__uint_as_float(pr[hv][2 * c]), __uint_as_float(pr[hv][2 * c + 1]));
                    pk[hv][c + 1] = pack_bf16x2(__uint_as_float(pr[hv][2 * c + 2]), __uint_as_float(pr[hv][2 * c + 3]));
                }
            };
            auto copy_dp = [&]() {
                tc_fence_after_sync();
                tmem_ld_32x32b_x32(tx, dr[0]);
                tmem_ld_32x32b_x32(tx + 32, dr[1]);
                tmem_ld_wait();
                reg_fence(dr[0]);
                reg_fence(dr[1]);
                tc_fence_before_sync();
                mbar_arrive(bar_x_free);
                have_dp = true;
            };
#pragma unroll
            for (int qtr = 0; qtr < 3; ++qtr) {
                probs_quarter(qtr);
                if (!have_dp && __all_sync(0xffffffffu, mbar_test_wait(bar_x_full, 1))) copy_dp();
            }
            probs_quarter(3);
            if (!have_dp) {
                ok = __all_sync(0xffffffffu, wait_phase(bar_x_full, 1, SITE_BWD_SM, wc));   // dP^T(i)
                if (!ok) break;
                copy_dp();
            }
            if (i > 0) {  // P^T is free once dV(i-1) has read it
                ok = __all_sync(0xffffffffu, wait_phase(bar_dv_done, (i - 1) & 1, SITE_BWD_SM, wc));
                if (!ok) break;
                tc_fence_after_sync();
            }
            tmem_st_32x32b_x16(tpt, pk[0]);
            tmem_st_32x32b_x16(tpt + 16u, pk[1]);
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(bar_p_full);
            // dS^T = P^T (dP^T - delta[column]), fp32, then bf16.
#pragma unroll
            for (int hv = 0; hv < 2; ++hv)
#pragma unroll
                for (int c = 0; c < 16; c += 2) {
                    const float4 d = dlt4[hv * 8 + c / 2];
                    const uint64_t ds0 = f2_mul(f2_pack(__uint_as_float(pr[hv][2 * c]), __uint_as_float(pr[hv][2 * c + 1])),
                                                f2_sub(f2_pack(__uint_as_float(dr[hv][2 * c]), __uint_as_float(dr[hv][2 * c + 1])),
                                                       f2_pack(d.x, d.y)));
                    const uint64_t ds1 = f2_mul(f2_pack(__uint_as_float(pr[hv][2 * c + 2]), __uint_as_float(pr[hv][2 * c + 3])),
                                                f2_sub(f2_pack(__uint_as_float(dr[hv][2 * c + 2]), __uint_as_float(dr[hv][2 * c + 3])),
                                                       f2_pack(d.z, d.w)));
                    float a0, b0, a1, b1;
                    f2_unpack(ds0, a0, b0);
                    f2_unpack(ds1, a1, b1);
                    pk[hv][c] = pack_bf16x2(a0, b0);
                    pk[hv][c + 1] = pack_bf16x2(a1, b1);
                }
            if (i > 0) {  // dS^T is free once dK(i-1) has read it
                ok = __all_sync(0xffffffffu, wait_phase(bar_dk_done, (i - 1) & 1, SITE_BWD_SM, wc));
                if (!ok) break;
                tc_fence_after_sync();
            }
            tmem_st_32x32b_x16(tds, pk[0]);
            tmem_st_32x32b_x16(tds + 16u, pk[1]);
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(bar_ds_full);
        }
        // dK(nq-1) is the last product; the commit after it covers dV(nq-1) too
        if (ok) ok = __all_sync(0xffffffffu, wait_phase(bar_dk_done, (nq - 1) & 1, SITE_BWD_ACC, wc));
        if (ok) {
            tc_fence_after_sync();
            // Epilogue: warpgroup 0 writes dV, warpgroup 1 writes scale * dK, each
            // as bf16 into a free stage of the Q / dO ring (every MMA has completed)
            // in the TMA's 128-byte swizzled layout; key rows past Skv fall outside
            // the tensor map and are not stored.
            const uint32_t tacc = tmem + lane_bits + 256u + (w ? HD : 0);
            const float mul = w ? scale : 1.0f;
            uint8_t *stage = smem + (w ? C::A_DO_OFF : C::A_Q_OFF);
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(tacc + c * 32, o);
                tmem_ld_wait();
                reg_fence(o);
                float add[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) add[x] = 0.f;
                if constexpr (ACCUM) {
                    if (key0 + krow < skv) {
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            (w ? (second ? dk_old2 : dk_old) : (second ? dv_old2 : dv_old)) +
                            (static_cast<int64_t>(bh) * skv + key0 + krow) * HD + c * 32);
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const uint4 u = src[g];
                            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                add[g * 8 + 2 * e] = __uint_as_float(uw[e] << 16);
                                add[g * 8 + 2 * e + 1] = __uint_as_float(uw[e] & 0xFFFF0000u);
                            }
                        }
                    }
                }
                auto val = [&](int x) { return fmaf(__uint_as_float(o[x]), mul, add[x]); };
                const int half = c >> 1;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int chunk = (c & 1) * 4 + g;
                    uint4 v;
                    v.x = pack_bf16x2(val(g * 8 + 0), val(g * 8 + 1));
                    v.y = pack_bf16x2(val(g * 8 + 2), val(g * 8 + 3));
                    v.z = pack_bf16x2(val(g * 8 + 4), val(g * 8 + 5));
                    v.w = pack_bf16x2(val(g * 8 + 6), val(g * 8 + 7));
                    *reinterpret_cast<uint4 *>(stage + half * C::HALF_BYTES + krow * 128 + ((chunk ^ (krow & 7)) << 4)) = v;
                }
            }
            fence_proxy_async_smem();
        }
        named_bar_sync(1 + w, 128);
        if (ok && warp == 4 + 4 * w && lane == 0) {
            const CUtensorMap *map = w ? (second ? &tm_dk2 : &tm_dk) : (second ? &tm_dv2 : &tm_dv);
            const uint32_t src = sbase + (w ? C::A_DO_OFF : C::A_Q_OFF);
            for (int h = 0; h < C::HALVES; ++h) tma_store_3d(map, src + h * C::HALF_BYTES, h * 64, key0, bh);
            tma_store_commit();
            tma_store_wait_read_all();   // only the shared-memory reads must finish before the CTA exits
        }
        tc_fence_before_sync();
        __syncthreads();
    }
}

// ------------------------------------------------------------------ dQ ---

// One CTA = one (b*h, 128-row query tile); thread = query row (TMEM lane),
// warpgroup w owns key columns [64w, 64w + 64) of each key tile.
// TMEM columns: S in two buffers [0,128) and [128,256) (dS as bf16 over
// [64w, 64w+32) of its buffer), dP [256,384), dQ [384, 384+HD).
// Two MMA issuers. Warp 1 issues S(j) = Q K(j)^T into buffer j & 1 once dQ(j-2)
// has released it, and dP(j) = dO V(j)^T once the elementwise warps have
// copied dP(j-1) out; neither waits for dS, so both run about a tile ahead.
// Warp 2 issues dQ += dS(j) K(j) as soon as dS(j) is stored. (With one issuing
// thread, in the order dQ(j) | dP(j+1) | S(j+2), a clock64 trace showed that
// thread busy for the whole tile and the elementwise warps idle ~45 % of it.)
// K and V come from two producer warps (0 and 3).
// ACCUM: dQ is added to the bf16 values already in dq.
// Two key sources: the key tiles of the first (Skv keys; tm_k, tm_v), then
// those of the second (Skv2 keys; tm_k2, tm_v2), one dQ accumulation over
// both; each source's last tile masks its own keys past its end. Skv2 = 0:
// one source.
template <int HD, bool ACCUM>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_k2,
                       const __grid_constant__ CUtensorMap tm_v2, const uint16_t *__restrict__ dq_old,
                       const float *__restrict__ ws, int Sq, int Skv, int Skv2, float scale, float scale_log2,
                       uint64_t wait_limit_ns)
{
    using C = BwdCfg<HD>;
    constexpr int NK = C::B_NK, NV = C::B_NV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = sbase + C::B_BAR_OFF;
    const uint32_t bar_qdo = bar0;
    auto bar_k_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto bar_k_empty = [&](int s) { return bar0 + 8u * (1 + NK + s); };
    auto bar_v_full = [&](int s) { return bar0 + 8u * (1 + 2 * NK + s); };
    auto bar_v_empty = [&](int s) { return bar0 + 8u * (1 + 2 * NK + NV + s); };
    auto bar_s_full = [&](int b) { return bar0 + 8u * (1 + 2 * NK + 2 * NV + b); };
    const uint32_t bar_dp_full = bar0 + 8u * (3 + 2 * NK + 2 * NV);
    const uint32_t bar_ds_full = bar0 + 8u * (4 + 2 * NK + 2 * NV);
    const uint32_t bar_acc_full = bar0 + 8u * (5 + 2 * NK + 2 * NV);
    const uint32_t bar_drain = bar0 + 8u * (6 + 2 * NK + 2 * NV);
    const uint32_t bar_dp_free = bar0 + 8u * (7 + 2 * NK + 2 * NV);                   // dP copied out
    auto bar_s_free = [&](int b) { return bar0 + 8u * (8 + 2 * NK + 2 * NV + b); };  // dQ read dS(b)
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::B_MISC_OFF);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::B_MISC_OFF + 8);

    if (threadIdx.x == 0) {
        mbar_init(bar_qdo, 1);
        for (int s = 0; s < NK; ++s) {
            mbar_init(bar_k_full(s), 1);
            mbar_init(bar_k_empty(s), 1);
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(bar_v_full(s), 1);
            mbar_init(bar_v_empty(s), 1);
        }
        mbar_init(bar_s_full(0), 1);
        mbar_init(bar_s_full(1), 1);
        mbar_init(bar_s_free(0), 1);
        mbar_init(bar_s_free(1), 1);
        mbar_init(bar_dp_full, 1);
        mbar_init(bar_dp_free, 256);
        mbar_init(bar_ds_full, 256);
        mbar_init(bar_acc_full, 1);
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
    const int nq = (Sq + C::BM - 1) / C::BM;
    const int nkv1 = (Skv + C::BN - 1) / C::BN;         // key tiles of the first source
    const int nkv = nkv1 + (Skv2 + C::BN - 1) / C::BN;  // of both
    const int bh = static_cast<int>(blockIdx.x / nq);
    const int qt = static_cast<int>(blockIdx.x % nq);
    const int q0 = qt * C::BM;
    // key tile j: its source's tensor maps, its first key row there, its valid keys
    auto tile_k = [&](int j) { return j < nkv1 ? &tm_k : &tm_k2; };
    auto tile_v = [&](int j) { return j < nkv1 ? &tm_v : &tm_v2; };
    auto tile_row = [&](int j) { return (j < nkv1 ? j : j - nkv1) * C::BN; };
    auto valid_keys = [&](int j) {
        const int rest = (j < nkv1 ? Skv : Skv2) - tile_row(j);
        return rest < C::BN ? rest : C::BN;
    };

    if (warp < 4) {
    setmaxnreg_dec<C::B_REGS_LOW>();
    const uint64_t drain_ns = wait_limit_ns > kDrainFloorNs ? wait_limit_ns : kDrainFloorNs;
    auto drain_copies = [&](uint32_t bar, uint32_t parity) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < drain_ns) {
        }
    };
    // Each MMA issuer commits to bar_drain (count 2) and waits for both before
    // TMEM is freed.
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
    auto tm_sb = [&](int b) { return tmem + 128u * static_cast<uint32_t>(b); };
    const uint32_t tm_dp = tmem + 256u, tm_dq = tmem + 384u;
    const uint32_t q_s = sbase + C::B_Q_OFF, do_s = sbase + C::B_DO_OFF;
    auto k_s = [&](int s) { return sbase + C::B_K_OFF + s * C::TILE_BYTES; };
    auto v_s = [&](int s) { return sbase + C::B_V_OFF + s * C::TILE_BYTES; };
    if (warp == 0) {
        // --------------------------------------- producer: Q, dO, then K ---
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            if (nkv > nkv1) tma_prefetch_desc(&tm_k2);
            tma_prefetch_desc(&tm_do);
            const uint64_t keep = l2_policy_evict_last();   // K: re-read by every query tile of the head
            const uint64_t once = l2_policy_evict_first();  // Q, dO: read by this CTA only
            mbar_arrive_expect_tx(bar_qdo, 2 * C::TILE_BYTES);
            for (int h = 0; h < C::HALVES; ++h) {
                tma_load_3d(sbase + C::B_Q_OFF + h * C::HALF_BYTES, &tm_q, bar_qdo, h * 64, q0, bh, once);
                tma_load_3d(sbase + C::B_DO_OFF + h * C::HALF_BYTES, &tm_do, bar_qdo, h * 64, q0, bh, once);
            }
            int nk = 0;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int sk = j % NK;
                ok = wait_phase(bar_k_empty(sk), ((j / NK) & 1) ^ 1, SITE_BWD_PROD, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_k_full(sk), C::TILE_BYTES);
                for (int h = 0; h < C::HALVES; ++h)
                    tma_load_3d(sbase + C::B_K_OFF + sk * C::TILE_BYTES + h * C::HALF_BYTES, tile_k(j), bar_k_full(sk),
                                h * 64, tile_row(j), bh, keep);
                ++nk;
            }
            if (!ok) {
                for (int j = (nk > NK ? nk - NK : 0); j < nk; ++j) drain_copies(bar_k_full(j % NK), (j / NK) & 1);
                drain_copies(bar_qdo, 0);
            }
        }
    } else if (warp == 3) {
        // ------------------------------------------------- producer: V ---
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            if (nkv > nkv1) tma_prefetch_desc(&tm_v2);
            const uint64_t keep = l2_policy_evict_last();   // V: re-read by every query tile of the head
            int nv = 0;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int sv = j % NV;
                ok = wait_phase(bar_v_empty(sv), ((j / NV) & 1) ^ 1, SITE_BWD_PROD, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_v_full(sv), C::TILE_BYTES);
                for (int h = 0; h < C::HALVES; ++h)
                    tma_load_3d(sbase + C::B_V_OFF + sv * C::TILE_BYTES + h * C::HALF_BYTES, tile_v(j), bar_v_full(sv),
                                h * 64, tile_row(j), bh, keep);
                ++nv;
            }
            if (!ok)
                for (int j = (nv > NV ? nv - NV : 0); j < nv; ++j) drain_copies(bar_v_full(j % NV), (j / NV) & 1);
        }
    } else if (warp == 1) {
        // ----------------------------- MMA issuer: S = Q K^T and dP = dO V^T ---
        // S(j) goes into buffer j & 1 once dQ(j-2) has read the dS written over
        // it; dP(j) into its buffer once the elementwise warps have copied dP(j-1)
        // out. Neither waits for dS, so both run ahead of the elementwise work.
        // This thread is the only waiter on bar_s_free(b) and bar_dp_free and
        // waits for each of their completions in turn.
        if (lane == 0) {
            constexpr uint32_t IDESC_T = idesc_bf16_f32(128, 128, false);  // Q K^T, dO V^T
            auto issue_t = [&](uint32_t d, uint32_t a, uint32_t b) {
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk / 4) * C::HALF_BYTES + (kk % 4) * 32;
                    mma_ss(d, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024), IDESC_T,
                           kk > 0 ? 1u : 0u);
                }
            };
            bool ok = wait_phase(bar_qdo, 0, SITE_BWD_MMA, wc);
            for (int j = 0; j < nkv && ok; ++j) {
                const int b = j & 1;
                if (j >= 2) {
                    ok = wait_phase(bar_s_free(b), ((j - 2) >> 1) & 1, SITE_BWD_MMA, wc);
                    if (!ok) break;
                }
                ok = wait_phase(bar_k_full(j % NK), (j / NK) & 1, SITE_BWD_MMA, wc);
                if (!ok) break;
                tc_fence_after_sync();
                issue_t(tm_sb(b), q_s, k_s(j % NK));
                tc_commit(bar_s_full(b));
                if (j >= 1) {
                    ok = wait_phase(bar_dp_free, (j - 1) & 1, SITE_BWD_MMA, wc);
                    if (!ok) break;
                }
                ok = wait_phase(bar_v_full(j % NV), (j / NV) & 1, SITE_BWD_MMA, wc);
                if (!ok) break;
                tc_fence_after_sync();
                issue_t(tm_dp, do_s, v_s(j % NV));
                tc_commit(bar_dp_full);
                tc_commit(bar_v_empty(j % NV));
            }
            drain_mmas();
        }
        __syncwarp();
    } else {
        // ---------------------------------------- MMA issuer: dQ += dS K ---
        if (lane == 0) {
            constexpr uint32_t IDESC_G = idesc_bf16_f32(128, HD, true);    // dS K: K tile MN-major
            auto issue_dq = [&](uint32_t a, uint32_t kb, bool acc) {
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ts(tm_dq, a + 64u * (kk >> 2) + 8u * (kk & 3),
                           smem_desc_sw128(kb + kk * 2048, C::HALF_BYTES, 1024), IDESC_G,
                           (acc || kk > 0) ? 1u : 0u);
            };
            bool ok = true;
            for (int j = 0; j < nkv && ok; ++j) {
                const int b = j & 1;
                ok = wait_phase(bar_k_full(j % NK), (j / NK) & 1, SITE_BWD_MMA, wc);  // complete by now
                if (ok) ok = wait_phase(bar_ds_full, j & 1, SITE_BWD_MMA, wc);
                if (!ok) break;
                tc_fence_after_sync();
                issue_dq(tm_sb(b), k_s(j % NK), j > 0);
                tc_commit(bar_s_free(b));
                // K(j) was read by S(j) too; that MMA completed before the
                // elementwise warps could form dS(j).
                tc_commit(bar_k_empty(j % NK));
                if (j + 1 == nkv) tc_commit(bar_acc_full);
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
        setmaxnreg_inc<C::B_REGS_HIGH>();
        // ------------------------------------------------- elementwise ---
        const int w = (warp - 4) >> 2;     // key columns [64w, 64w + 64)
        const int quad = warp & 3;
        const int row = quad * 32 + lane;  // query row inside the tile
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        const float *blk = ws + (static_cast<int64_t>(bh) * nq + qt) * 256;
        const float lse2 = blk[row];     // +inf past Sq: P = 0
        const float delta = blk[128 + row];
        const uint64_t c2 = f2_pack(scale_log2, scale_log2);
        const uint64_t nl2 = f2_pack(-lse2, -lse2);
        const uint64_t dl2 = f2_pack(delta, delta);
        bool ok = true;
        for (int j = 0; ok && j < nkv; ++j) {
            const int b = j & 1;
            const uint32_t ts = tmem + lane_bits + 128u * b + 64u * w;
            ok = __all_sync(0xffffffffu, wait_phase(bar_s_full(b), (j >> 1) & 1, SITE_BWD_SM, wc));
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t pr[2][32];
            tmem_ld_32x32b_x32(ts, pr[0]);
            tmem_ld_32x32b_x32(ts + 32, pr[1]);
            tmem_ld_wait();
            reg_fence(pr[0]);
            reg_fence(pr[1]);
#pragma unroll
            for (int hv = 0; hv < 2; ++hv)
#pragma unroll
                for (int c = 0; c < 16; ++c) probs_pair<C::EMU_PER8>(pr[hv][2 * c], pr[hv][2 * c + 1], c2, nl2, c);
            const int kv_tail = valid_keys(j);
            if (kv_tail < C::BN) {
                // keys past the source's end: their logits come from zero-filled rows; P = 0
#pragma unroll
                for (int x = 0; x < 64; ++x)
                    if (64 * w + x >= kv_tail) pr[x >> 5][x & 31] = 0u;
            }
            ok = __all_sync(0xffffffffu, wait_phase(bar_dp_full, j & 1, SITE_BWD_SM, wc));
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t dr[2][32];
            tmem_ld_32x32b_x32(tmem + lane_bits + 256u + 64u * w, dr[0]);
            tmem_ld_32x32b_x32(tmem + lane_bits + 256u + 64u * w + 32u, dr[1]);
            tmem_ld_wait();
            reg_fence(dr[0]);
            reg_fence(dr[1]);
            // dP is in registers: the buffer may take dP(j+1).
            tc_fence_before_sync();
            mbar_arrive(bar_dp_free);
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint64_t ds = f2_mul(f2_pack(__uint_as_float(pr[hv][2 * c]), __uint_as_float(pr[hv][2 * c + 1])),
                                               f2_sub(f2_pack(__uint_as_float(dr[hv][2 * c]), __uint_as_float(dr[hv][2 * c + 1])), dl2));
                    float a, bb;
                    f2_unpack(ds, a, bb);
                    pk[c] = pack_bf16x2(a, bb);
                }
                tmem_st_32x32b_x16(ts + 16u * hv, pk);
            }
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(bar_ds_full);
        }
        if (ok) ok = __all_sync(0xffffffffu, wait_phase(bar_acc_full, 0, SITE_BWD_ACC, wc));
        if (ok) {
            tc_fence_after_sync();
            // Epilogue: warpgroup w converts dQ columns [w*HD/2, (w+1)*HD/2) of
            // its rows (x scale, plus the previous dq when accumulating) into the
            // Q buffer, 128-byte swizzled, for one TMA store.
            const int qrow = q0 + row;
            uint8_t *stage = smem + C::B_Q_OFF;
#pragma unroll
            for (int cc = 0; cc < HD / 64; ++cc) {
                const int col0 = w * (HD / 2) + cc * 32;
                uint32_t o[32];
                tmem_ld_32x32b_x32(tmem + lane_bits + 384u + col0, o);
                tmem_ld_wait();
                reg_fence(o);
                float add[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) add[x] = 0.f;
                if constexpr (ACCUM) {
                    if (qrow < Sq) {
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            dq_old + (static_cast<int64_t>(bh) * Sq + qrow) * HD + col0);
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const uint4 u = src[g];
                            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                add[g * 8 + 2 * e] = __uint_as_float(uw[e] << 16);
                                add[g * 8 + 2 * e + 1] = __uint_as_float(uw[e] & 0xFFFF0000u);
                            }
                        }
                    }
                }
                const int half = col0 >> 6;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int chunk = ((col0 & 63) >> 3) + g;
                    auto val = [&](int x) { return fmaf(__uint_as_float(o[x]), scale, add[x]); };
                    uint4 v;
                    v.x = pack_bf16x2(val(g * 8 + 0), val(g * 8 + 1));
                    v.y = pack_bf16x2(val(g * 8 + 2), val(g * 8 + 3));
                    v.z = pack_bf16x2(val(g * 8 + 4), val(g * 8 + 5));
                    v.w = pack_bf16x2(val(g * 8 + 6), val(g * 8 + 7));
                    *reinterpret_cast<uint4 *>(stage + half * C::HALF_BYTES + row * 128 + ((chunk ^ (row & 7)) << 4)) = v;
                }
            }
            fence_proxy_async_smem();
        }
        // both warpgroups' halves must be staged before the one store
        named_bar_sync(1, 256);
        if (ok && warp == 4 && lane == 0) {
            for (int h = 0; h < C::HALVES; ++h)
                tma_store_3d(&tm_dq, sbase + C::B_Q_OFF + h * C::HALF_BYTES, h * 64, q0, bh);
            tma_store_commit();
            tma_store_wait_read_all();   // only the shared-memory reads must finish before the CTA exits
        }
        tc_fence_before_sync();
        __syncthreads();
    }
}

}  // namespace regen
