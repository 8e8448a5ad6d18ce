// proj_gemm.cuh -- the projections around the attention in a DiT block, on
// the tcgen05 tensor cores (sm_100a).
//
// The decoder's DiT matches the Wan2.1 architecture (ReGenVC blog page,
// "Methodology -- deep read"): each block's self-attention reads q, k, v from
// one linear layer of the token features and writes its heads back through
// another. Here:
//   QKV:  y = x W^T + b over the tokens x [B][S][C], W [3 H 128][C]; per head
//         of q and k an RMSNorm over its 128 values (weight g) and the 3D RoPE
//         of the token's latent grid position; q, k, v written straight into
//         the attention's [B][H][S][128] layout.
//   OUT:  y = o W^T + b with o the attention output [B][H][S][128] read as
//         token rows of H*128 features (one TMA box per (head, 64 values)), W
//         [N][H 128]; y [B][S][N].
//
// Pairs of SMs (clusters of 2 CTAs, tcgen05 cta_group::2) walk persistently
// over 256-token x 256-feature tiles, in groups of 8 token tiles (so the pairs
// in flight share A and W in L2). Each CTA holds its own 128 token rows of A
// and one 128-feature half of B per stage (6 stages, 32 KB each), loaded by
// its warp 0 with the pair form of the TMA load, all completing on the even
// CTA's stage barrier; the even CTA's warp 1 issues M256 N256 K16 MMAs over
// both CTAs' shared memory into one of two 256-column accumulators per CTA
// (each CTA's TMEM holds its own 128 rows), and releases stages and
// accumulators to both CTAs with multicast commits. Two epilogue warpgroups
// per CTA (warps 4-7, 8-11) each drain one accumulator, so a tile's epilogue
// overlaps the next tile's main loop; the odd CTA's epilogue reports to the
// even CTA's barrier. Per SM this halves the B operand bytes a 128 x 256 tile
// of one CTA would read. In the epilogue a thread owns one token row: the
// RMSNorm of a 128-value head needs no reduction across threads, and each
// thread stores its rows directly. No load multicasts.
#pragma once

#include "attn_fwd.cuh"
#include "ptx.cuh"
#include "rope3d.cuh"

namespace regen {

enum ProjMode : int { PROJ_QKV = 0, PROJ_OUT = 1 };

struct ProjShape {
    int B, S, K, N;     // tokens per batch S, input features K, output features N
    int H;              // heads: of q/k/v (QKV) or of the attention output read as A (OUT)
    int num_mt, num_nt; // pair tiles along tokens (per batch, ceil(S/256) each) and features (ceil(N/256))
};

struct ProjCfg {
    static constexpr int BM = 128, BN = 256, BK = 64;   // per CTA: 128 tokens; per pair: 256 x 256
    static constexpr int PAIR_M = 2 * BM;
    static constexpr int NS = 6;
    static constexpr int A_BYTES = BM * BK * 2;         // 16 KB: this CTA's 128 token rows
    static constexpr int B_BYTES = (BN / 2) * BK * 2;   // 16 KB: this CTA's 128-feature half
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = NS * A_BYTES;
    static constexpr int BAR_OFF = B_OFF + NS * B_BYTES;
    // full[NS], empty[NS], acc_full[2], acc_empty[2], drain
    static constexpr int NBARS = 2 * NS + 5;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 384;
    static constexpr uint32_t REGS_LOW = 64;
    static constexpr uint32_t REGS_HIGH = 208;
    static constexpr int MIN_LAUNCH_REGS = 160;
    static constexpr int GROUP_M = 8;
};

enum ProjWaitSite : uint32_t { SITE_PROJ_PROD = 20, SITE_PROJ_MMA = 21, SITE_PROJ_EPI = 22 };

// Tile t of the grouped order -> (token tile, feature tile).
__device__ __forceinline__ void proj_tile(int t, const ProjShape &p, int &mt, int &nt)
{
    const int per_group = ProjCfg::GROUP_M * p.num_nt;
    const int g = t / per_group;
    const int first = g * ProjCfg::GROUP_M;
    const int gm = min(ProjCfg::GROUP_M, p.num_mt - first);
    const int r = t - g * per_group;
    mt = first + r % gm;
    nt = r / gm;
}

// (cos, sin) in fp32 of every RoPE table entry (RopeGeom layout), from fp64.
__global__ void rope_table_f32_kernel(float2 *__restrict__ tab, RopeGeom g, const __grid_constant__ RopeFreqs fr)
{
    const int64_t n = g.entries();
    const int64_t base_h = static_cast<int64_t>(g.T) * (g.dt / 2);
    const int64_t base_w = base_h + static_cast<int64_t>(g.Hh) * (g.dh / 2);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n; e += stride) {
        int pos, pair;   // pair: index of the pair within the head dimension
        if (e < base_h) {
            pos = static_cast<int>(e / (g.dt / 2)); pair = static_cast<int>(e % (g.dt / 2));
        } else if (e < base_w) {
            pos = static_cast<int>((e - base_h) / (g.dh / 2));
            pair = g.dt / 2 + static_cast<int>((e - base_h) % (g.dh / 2));
        } else {
            pos = static_cast<int>((e - base_w) / (g.dh / 2));
            pair = (g.dt + g.dh) / 2 + static_cast<int>((e - base_w) % (g.dh / 2));
        }
        double c, s;
        rope_angle(pos, fr.f[pair], c, s);
        tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
    }
}

struct ProjEpi {
    const float *bias;       // [N] or null
    const float *gamma_q;    // [H 128] or null (QKV)
    const float *gamma_k;    // [H 128] or null (QKV)
    uint16_t *out0, *out1, *out2;   // QKV: q, k, v [B][H][S][128]; OUT: y [B][S][N] in out0
    const float2 *rope_tab;  // QKV: (cos, sin) per RopeGeom entry
    RopeGeom geom;
    float eps;
};

template <int MODE>
__global__ void __launch_bounds__(384, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     ProjShape p, ProjEpi ep, uint64_t wait_limit_ns)
{
    using C = ProjCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = sbase + C::BAR_OFF;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (C::NS + s); };
    auto bar_acc_full = [&](int e) { return bar0 + 8u * (2 * C::NS + e); };
    auto bar_acc_empty = [&](int e) { return bar0 + 8u * (2 * C::NS + 2 + e); };
    const uint32_t bar_drain = bar0 + 8u * (2 * C::NS + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::MISC_OFF + 8);

    const uint32_t rank = cluster_ctarank();   // 0: the pair's MMA issuer
    const bool leader = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(bar_full(s), 1);         // the leader's: both CTAs' loads complete on it
            mbar_init(bar_empty(s), 1);        // each CTA's: the leader's multicast commit
        }
        for (int e = 0; e < 2; ++e) {
            mbar_init(bar_acc_full(e), 1);     // each CTA's: multicast commit
            mbar_init(bar_acc_empty(e), 256);  // the leader's: both CTAs' epilogue threads
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();    // both CTAs' barriers exist before any remote use
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const WaitCtl wc{abort_flag, wait_limit_ns};
    const int total = p.num_mt * p.num_nt;
    const int kblocks = (p.K + C::BK - 1) / C::BK;
    const int mpb = (p.S + C::PAIR_M - 1) / C::PAIR_M;   // pair tiles per batch along tokens
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (warp < 4) {
    setmaxnreg_dec<C::REGS_LOW>();
    if (warp == 0) {
        // ------------------------------------------------------ producer ---
        // Each CTA loads its own A rows and B half; both complete on the
        // leader's stage barrier, where the leader posts both CTAs' bytes.
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            const uint64_t keep = l2_policy_evict_last();
            int it = 0;
            bool ok = true;
            for (int t = pair; ok && t < total; t += npairs) {
                int mt, nt;
                proj_tile(t, p, mt, nt);
                const int b = mt / mpb, s0 = (mt % mpb) * C::PAIR_M + static_cast<int>(rank) * C::BM;
                const int nb0 = nt * C::BN + static_cast<int>(rank) * (C::BN / 2);
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % C::NS;
                    ok = wait_phase(bar_empty(s), ((it / C::NS) & 1) ^ 1, SITE_PROJ_PROD, wc);
                    if (!ok) break;
                    const uint32_t full_leader = mapa_shared(bar_full(s), 0);
                    if (leader) mbar_arrive_expect_tx(bar_full(s), 2 * (C::A_BYTES + C::B_BYTES));
                    if constexpr (MODE == PROJ_QKV)
                        tma_load_3d_pair(sbase + C::A_OFF + s * C::A_BYTES, &tm_a, full_leader, kb * C::BK, s0, b, keep);
                    else  // the attention output: k block kb = (head kb/2, values 64 (kb%2) ..)
                        tma_load_3d_pair(sbase + C::A_OFF + s * C::A_BYTES, &tm_a, full_leader, (kb & 1) * 64, s0,
                                         b * p.H + (kb >> 1), keep);
                    tma_load_3d_pair(sbase + C::B_OFF + s * C::B_BYTES, &tm_b, full_leader, kb * C::BK, nb0, 0, keep);
                }
            }
            if (!ok) {
                // Aborting: the copies in flight land in this CTA's memory within
                // microseconds; give them a bounded moment before the CTA leaves.
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 1000000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------ MMA issuer (leader only) ---
        if (lane == 0 && leader) {
            constexpr uint32_t IDESC = idesc_bf16_f32(256, 256, false);   // M over the pair; both K-major
            int it = 0, local = 0;
            bool ok = true;
            for (int t = pair; ok && t < total; t += npairs, ++local) {
                const int e = local & 1;
                ok = wait_phase(bar_acc_empty(e), ((local >> 1) & 1) ^ 1, SITE_PROJ_MMA, wc);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t acc = tmem + 256u * e;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % C::NS;
                    ok = wait_phase(bar_full(s), (it / C::NS) & 1, SITE_PROJ_MMA, wc);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t a = sbase + C::A_OFF + s * C::A_BYTES;
                    const uint32_t bb = sbase + C::B_OFF + s * C::B_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::BK / 16; ++kk)
                        mma_ss_pair(acc, smem_desc_sw128(a + kk * 32, 16, 1024), smem_desc_sw128(bb + kk * 32, 16, 1024),
                                    IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
                    tc_commit_pair(bar_empty(s), 0x3);
                }
                if (ok) tc_commit_pair(bar_acc_full(e), 0x3);
            }
            tc_commit_pair(bar_drain, 0x1);
            const uint64_t drain_ns = wait_limit_ns > kDrainFloorNs ? wait_limit_ns : kDrainFloorNs;
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
    cluster_sync_all();    // the pair's MMAs, commits and remote arrivals are over
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
    } else {
        setmaxnreg_inc<C::REGS_HIGH>();
        // ------------------------------------------------------- epilogue ---
        const int e = (warp - 4) >> 2;      // the accumulator this warpgroup drains
        const int quad = warp & 3;
        const int row = quad * 32 + lane;   // token row inside the tile
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t acc = tmem + lane_bits + 256u * e;
        const uint32_t acc_empty_leader = mapa_shared(bar_acc_empty(e), 0);
        bool ok = true;
        int local = 0;
        for (int t = pair; ok && t < total; t += npairs, ++local) {
            if ((local & 1) != e) continue;
            int mt, nt;
            proj_tile(t, p, mt, nt);
            const int b = mt / mpb, n0 = nt * C::BN;
            const int s = (mt % mpb) * C::PAIR_M + static_cast<int>(rank) * C::BM + row;
            ok = __all_sync(0xffffffffu, wait_phase(bar_acc_full(e), (local >> 1) & 1, SITE_PROJ_EPI, wc));
            if (!ok) break;
            tc_fence_after_sync();
            if constexpr (MODE == PROJ_QKV) {
                const int HD = p.H * 128;
#pragma unroll 1
                for (int hc = 0; hc < 2; ++hc) {
                    const int n = n0 + hc * 128;   // first feature of this head
                    const int which = n / HD, h = (n % HD) / 128;
                    const bool live = n < p.N && s < p.S;
                    const bool norm = which < 2;
                    // pass 1 (q, k): sum of squares of the head's 128 biased values
                    float inv = 1.0f;
                    if (norm) {
                        float ss = 0.f;
#pragma unroll 1
                        for (int c = 0; c < 4; ++c) {
                            uint32_t r[32];
                            tmem_ld_32x32b_x32(acc + hc * 128 + c * 32, r);
                            tmem_ld_wait();
                            reg_fence(r);
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const float yv = __uint_as_float(r[i]) + (ep.bias && live ? __ldg(ep.bias + n + c * 32 + i) : 0.f);
                                ss = fmaf(yv, yv, ss);
                            }
                        }
                        inv = rsqrtf(ss * (1.0f / 128.0f) + ep.eps);
                    }
                    // table rows of this token's t, h, w positions (D = 128: axis blocks
                    // of 44, 42, 42 dims, i.e. 22, 21, 21 pairs)
                    const RopeGeom &gm = ep.geom;
                    const int64_t et = static_cast<int64_t>(s / (gm.Hh * gm.Ww)) * 22;
                    const int64_t eh = static_cast<int64_t>(gm.T) * 22 + static_cast<int64_t>((s / gm.Ww) % gm.Hh) * 21;
                    const int64_t ew = static_cast<int64_t>(gm.T) * 22 + static_cast<int64_t>(gm.Hh) * 21 +
                                       static_cast<int64_t>(s % gm.Ww) * 21;
                    const float *g = which == 0 ? ep.gamma_q : ep.gamma_k;
                    uint16_t *dst = which == 0 ? ep.out0 : which == 1 ? ep.out1 : ep.out2;
                    uint4 *o = reinterpret_cast<uint4 *>(dst + ((static_cast<int64_t>(b) * p.H + h) * p.S + s) * 128);
                    // pass 2: bias, RMSNorm and RoPE (q, k), bf16, 32 values at a time
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(acc + hc * 128 + c * 32, r);
                        tmem_ld_wait();
                        reg_fence(r);
                        if (!live) continue;
                        float y[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            y[i] = __uint_as_float(r[i]) + (ep.bias ? __ldg(ep.bias + n + c * 32 + i) : 0.f);
                        if (norm) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) y[i] *= inv * (g ? __ldg(g + h * 128 + c * 32 + i) : 1.0f);
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) {
                                const int j = c * 16 + jj;   // pair index in the head
                                const int64_t ent = j < 22 ? et + j : j < 43 ? eh + (j - 22) : ew + (j - 43);
                                const float2 cs = __ldg(ep.rope_tab + ent);
                                const float x0 = y[2 * jj], x1 = y[2 * jj + 1];
                                y[2 * jj] = fmaf(x0, cs.x, -x1 * cs.y);
                                y[2 * jj + 1] = fmaf(x0, cs.y, x1 * cs.x);
                            }
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            o[c * 4 + i] = make_uint4(pack_bf16x2(y[8 * i], y[8 * i + 1]),
                                                      pack_bf16x2(y[8 * i + 2], y[8 * i + 3]),
                                                      pack_bf16x2(y[8 * i + 4], y[8 * i + 5]),
                                                      pack_bf16x2(y[8 * i + 6], y[8 * i + 7]));
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < C::BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(acc + c * 32, r);
                    tmem_ld_wait();
                    reg_fence(r);
                    const int n = n0 + c * 32;
                    if (s >= p.S || n >= p.N) continue;
                    float y[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(r[i]) + (ep.bias ? __ldg(ep.bias + n + i) : 0.f);
                    uint4 *o = reinterpret_cast<uint4 *>(ep.out0 + (static_cast<int64_t>(b) * p.S + s) * p.N + n);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (n + 8 * i < p.N)
                            o[i] = make_uint4(pack_bf16x2(y[8 * i], y[8 * i + 1]), pack_bf16x2(y[8 * i + 2], y[8 * i + 3]),
                                              pack_bf16x2(y[8 * i + 4], y[8 * i + 5]),
                                              pack_bf16x2(y[8 * i + 6], y[8 * i + 7]));
                }
            }
            // every TMEM read of this accumulator is complete (waited above)
            tc_fence_before_sync();
            if (leader)
                mbar_arrive(bar_acc_empty(e));
            else
                mbar_arrive_remote(acc_empty_leader);
        }
        tc_fence_before_sync();
        __syncthreads();
        cluster_sync_all();
    }
}

}  // namespace regen
