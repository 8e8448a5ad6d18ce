// attn_fwd.cuh -- exact softmax attention forward for sm_100a.
//
// What it computes (ReGenVC, blog.captcha.la page, "Technical innovations":
// the DiT's attention stays exact under Ulysses x Ring sharding; Ring
// attention streams KV blocks and combines them by their log-sum-exp):
//   out_i = sum_j softmax_j(scale * <q_i, k_j>) v_j,  lse_i = ln sum_j exp(scale * <q_i, k_j>)
// One pass over 128-key blocks with an online softmax, i.e. the same
// blockwise LSE combination Ring attention applies between GPUs, applied
// here between key blocks of one GPU.
//
// Work unit = one CTA = one (batch*head, 256 query rows) = two 128-row Q tiles;
// grid = B*H*ceil(Sq/256) CTAs.
// Warp roles (384 threads):
//   warp 0      TMA producer: Q tiles once, then K tiles through an NS-stage ring
//   warp 3      TMA producer: V tiles through an NS-stage ring
//   warp 1      TMEM allocator; lane 0 issues the S = QK^T MMAs and their commits
//   warp 2      lane 0 issues the O += PV MMAs and their commits
//   warps 4-7   softmax + correction + epilogue for Q tile 0 (one thread per row)
//   warps 8-11  the same for Q tile 1
// Tensor memory (512 columns, fp32): one S buffer [0,128) shared by the two
// tiles, P0 [128,192) and P1 [192,256) (bf16, two per column), then O0 and O1
// (HD columns each). P feeds the PV MMA straight from TMEM. Because P has
// columns of its own, the next S of a tile need not wait for that tile's PV:
// S is free as soon as the softmax warps have copied it into registers.
// The S MMAs (S0(0) S1(0) S0(1) S1(1) ..., the S buffer alternating between
// the tiles) and the PV MMAs (PV0(0) PV1(0) PV0(1) ...) come from two issuing
// threads: the tensor core queues only a few MMAs, so one thread that stops to
// wait on a barrier between groups lets it run dry, while two keep it fed.
// Each tile's softmax of block j+1 runs while its PV of block j does; it
// waits for that PV only before it stores P (and rescales O, when it must).
// Softmax keeps a per-row running max m (log2 units, scale folded in) and
// sum l in fp32; O is rescaled only when the max grows by more than 8
// (log2), which stays exact because P = 2^(s - m) is then at most 2^8 and
// the final O/l and LSE use the same m.
#pragma once

#include <type_traits>

#include "ptx.cuh"
#include "rope3d.cuh"

// Pairs of every 8 probabilities whose 2^x runs on the FMA pipe (exp2_poly_pair)
// instead of MUFU. Gradient kernels: on the 77-frame window 1 measured ~2 %
// faster than 2, and 3 slower. Forward: with its two MMA issuers the kernel
// runs at the 1 kW power cap, where the polynomial's FMA-pipe work costs more
// than the MUFU time it frees: 0 measured 15.2-15.3 ms, 1 16.1-16.2 ms and 2
// 17.4-17.6 ms on the 77-frame window, so the forward uses MUFU alone.
#ifndef REGEN_EXP2_EMU_PER8
#define REGEN_EXP2_EMU_PER8 1
#endif
#ifndef REGEN_FWD_EXP2_EMU_PER8
#define REGEN_FWD_EXP2_EMU_PER8 0
#endif

namespace regen {

__device__ int g_regen_err;            // first error code recorded by a kernel
__device__ unsigned int g_regen_err_site;  // which wait gave up

enum WaitSite : uint32_t {
    SITE_PROD_K_EMPTY = 1,
    SITE_PROD_V_EMPTY = 2,
    SITE_MMA_Q = 3,
    SITE_MMA_K_FULL = 4,
    SITE_MMA_V_FULL = 5,
    SITE_MMA_P_FULL = 6,
    SITE_SM_S_FULL = 7,
    SITE_SM_O_FULL = 8,
    SITE_DRAIN = 9,
    SITE_SM_Q = 11,
    SITE_SELFTEST = 10,
    SITE_MMA_S_FREE = 12,
    SITE_SM_PV_DONE = 13,
};

__device__ __forceinline__ void record_timeout(uint32_t site)
{
    if (atomicCAS(&g_regen_err, 0, -5 /* REGEN_ERR_TIMEOUT */) == 0) g_regen_err_site = site;
}

// Lower bound on the waits that drain a CTA's own copies and MMAs before it
// exits after an abort (they complete in microseconds; 100 ms).
constexpr uint64_t kDrainFloorNs = 100000000ull;

struct WaitCtl {
    volatile int *abort;   // CTA-wide flag in shared memory
    uint64_t limit_ns;
};

// Bounded wait on an mbarrier phase. Returns false when the CTA is aborting
// (another role gave up) or when this wait exceeded the limit (then it
// records the site and raises the abort flag).
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, uint32_t site,
                                           const WaitCtl &w)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 31) == 0) {
            if (*w.abort) return false;
            if (global_timer_ns() - t0 > w.limit_ns) {
                record_timeout(site);
                *w.abort = 1;
                return false;
            }
        }
    }
}

template <int HD>
struct AttnCfg {
    static constexpr int BM = 128;                        // query rows per tile
    static constexpr int BN = 128;                        // keys per block
    static constexpr int HALVES = HD / 64;                // 128-byte column groups per row
    static constexpr int TILE_BYTES = 128 * HD * 2;       // one 128-row bf16 tile
    static constexpr int HALF_BYTES = 128 * 128;          // 128 rows x 128 bytes
#ifndef REGEN_FWD_K_STAGES
#define REGEN_FWD_K_STAGES 2
#endif
#ifndef REGEN_FWD_V_STAGES
#define REGEN_FWD_V_STAGES 2
#endif
    static constexpr int NSK = (HD == 128) ? REGEN_FWD_K_STAGES : 4;  // K ring depth
    static constexpr int NSV = (HD == 128) ? REGEN_FWD_V_STAGES : 4;  // V ring depth
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + 2 * TILE_BYTES;
    static constexpr int V_OFF = K_OFF + NSK * TILE_BYTES;
    static constexpr int BAR_OFF = V_OFF + NSV * TILE_BYTES;
    // barriers: q, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV], s_full[2], s_free,
    // p_full[2], pv_done[2], drain, q_rotated[2]
    static constexpr int NBARS = 1 + 2 * NSK + 2 * NSV + 7 + 1 + 2;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;  // abort flag, TMEM base
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 384;
    static constexpr uint32_t REGS_LOW = 64;    // producer / MMA / idle warpgroup
    static constexpr uint32_t REGS_HIGH = 208;  // the two softmax warpgroups
    // need (REGS_HIGH - R) * 256 <= (R - REGS_LOW) * 128, i.e. R >= 160
    static constexpr int MIN_LAUNCH_REGS = 160;
    // Of every 8 pairs of probabilities, this many are evaluated on the FMA
    // pipe (exp2_poly_pair) instead of MUFU (ex2 throughput, 16/clk/SM, alone
    // equals the tensor time of a key block; the power cap decides the split).
    static constexpr int EMU_PER8 = REGEN_FWD_EXP2_EMU_PER8;
};

// The RoPE of one row of a Q tile in shared memory (128-byte swizzled rows:
// 16-byte chunk cw of row r sits at chunk cw ^ (r & 7)), for token n (rows
// past Sq are left alone). The row's 64 fp32 (cos, sin) pairs depend only on
// its token, so they are loaded before the wait for the tile's TMA load. Two
// passes: every pair in fp32, stored where its certificate holds (the others
// keep their input and a bit in `redo`); then the few uncertified pairs in
// fp64 from the fp64 table. The fp32 pass has no branch, and the fp64 one
// runs only as often as the warp's most unlucky lane needs it.
// Returns the wait's outcome, made warp-uniform.
template <int HD>
__device__ __forceinline__ bool rope_q_tile_row(uint8_t *tile, int row, int n, int Sq, uint32_t bar_q, WaitCtl wc,
                                                RopeTabs rope_tab, RopeGeom rope_geom)
{
    constexpr int DH = 2 * (HD / 6), DT = HD - 2 * DH;   // axis widths t, h, w = DT, DH, DH
    constexpr int NP = HD / 2;                           // pairs per row
    constexpr int HALF_BYTES = 128 * 128;
    const bool live = n < Sq;
    const RopeRowEntries re = RopeRowEntries::of(rope_geom, live ? n : 0);
    float2 cs[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) cs[p] = __ldg(rope_tab.t32 + re.entry(2 * p, DT, DH));
    const bool ok = __all_sync(0xffffffffu, wait_phase(bar_q, 0, SITE_SM_Q, wc));
    if (ok && live) {
        uint8_t *rowp = tile + row * 128;
        auto chunk = [&](int c) {
            return reinterpret_cast<uint4 *>(rowp + (c >> 3) * HALF_BYTES + (((c & 7) ^ (row & 7)) << 4));
        };
        uint64_t redo = 0;   // bit p: pair p was not certified
#pragma unroll
        for (int c = 0; c < HD / 8; ++c) {
            const uint4 v = *chunk(c);
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                uint32_t r;
                const bool certified = rotate_pair_f32(w[p], cs[4 * c + p].x, cs[4 * c + p].y, r);
                redo |= static_cast<uint64_t>(!certified) << (4 * c + p);
                w[p] = certified ? r : w[p];
            }
            *chunk(c) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        while (redo) {
            const int p = __ffsll(static_cast<long long>(redo)) - 1;
            redo &= redo - 1;
            uint32_t *pair = reinterpret_cast<uint32_t *>(chunk(p >> 2)) + (p & 3);
            const int64_t e = re.entry(2 * p, DT, DH);
            *pair = rotate_pair(*pair, __ldg(rope_tab.t64 + 2 * e), __ldg(rope_tab.t64 + 2 * e + 1));
        }
    }
    return ok;
}

// ROPE_Q: the Q tiles are rotated by the 3D RoPE in shared memory right after
// their TMA load (each softmax thread rotates its own row, from the (cos, sin)
// table `rope_tab`), before the first S MMA of that tile reads them; the
// rotation gives the same bits as rope_stream_kernel (fp32 with a per-pair
// certificate, else fp64), so the result equals rotating Q in HBM first.
// KV2: the keys come from two sources, tm_k/tm_v (the first Skv1 keys) and
// tm_k2/tm_v2 (the other Skv - Skv1), under one online softmax: the result is
// the attention over the two sources concatenated. The blocks of source 1 come
// first, then those of source 2; each source's last block is masked past its
// own end. (Other instantiations ignore tm_k2, tm_v2 and Skv1.)
// The plain instantiation holds no RoPE code at all (a run-time flag, or the
// prologue in one instantiation, measurably changed the main loop's code).
template <int HD, bool NEG_SCALE, bool ROPE_Q, bool KV2 = false>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const __grid_constant__ CUtensorMap tm_k2, const __grid_constant__ CUtensorMap tm_v2,
                    float *__restrict__ lse, int Sq, int Skv, int Skv1, float scale_log2,
                    uint64_t wait_limit_ns, RopeTabs rope_tab, RopeGeom rope_geom)
{
    static_assert(!(ROPE_Q && KV2), "the RoPE-fused attention has one key source");
    constexpr bool rope_q = ROPE_Q;
    using C = AttnCfg<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = sbase + C::BAR_OFF;
    const uint32_t bar_q = bar0;
    auto bar_k_full = [&](int s) { return bar0 + 8u * (1 + s); };
    constexpr int NB = 2 * C::NSK + 2 * C::NSV;  // slots of the two rings' barriers
    auto bar_k_empty = [&](int s) { return bar0 + 8u * (1 + C::NSK + s); };
    auto bar_v_full = [&](int s) { return bar0 + 8u * (1 + 2 * C::NSK + s); };
    auto bar_v_empty = [&](int s) { return bar0 + 8u * (1 + 2 * C::NSK + C::NSV + s); };
    auto bar_s_full = [&](int t) { return bar0 + 8u * (1 + NB + t); };
    const uint32_t bar_s_free = bar0 + 8u * (3 + NB);  // S copied out by a softmax warpgroup
    auto bar_p_full = [&](int t) { return bar0 + 8u * (4 + NB + t); };
    auto bar_pv_done = [&](int t) { return bar0 + 8u * (6 + NB + t); };
    const uint32_t bar_drain = bar0 + 8u * (8 + NB);
    auto bar_qrot = [&](int t) { return bar0 + 8u * (9 + NB + t); };  // Q tile t rotated (rope_q)
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::MISC_OFF + 8);

    // 1-D grid, query-tile pairs of one head adjacent so that the CTAs resident
    // at any time share the K/V of one or two heads in L2.
    const int npairs = (Sq + 2 * C::BM - 1) / (2 * C::BM);
    const int bh = static_cast<int>(blockIdx.x / npairs);
    const int q0 = static_cast<int>(blockIdx.x % npairs) * (2 * C::BM);
    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < C::NSK; ++s) {
            mbar_init(bar_k_full(s), 1);
            mbar_init(bar_k_empty(s), 1);
        }
        for (int s = 0; s < C::NSV; ++s) {
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
        mbar_init(bar_qrot(0), 128);
        mbar_init(bar_qrot(1), 128);
        *abort_flag = 0;
        fence_mbarrier_init();
        // The Q tiles' loads (this thread is also the Q/K producer) leave now,
        // ahead of the TMEM allocation and the block-wide barrier.
        tma_prefetch_desc(&tm_q);
        mbar_arrive_expect_tx(bar_q, 2 * C::TILE_BYTES);
        for (int t = 0; t < 2; ++t)
            for (int h = 0; h < C::HALVES; ++h)
                tma_load_3d(sbase + C::Q_OFF + t * C::TILE_BYTES + h * C::HALF_BYTES, &tm_q, bar_q, h * 64,
                            q0 + t * C::BM, bh, l2_policy_evict_first());
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
    // key blocks: source 1's, then (KV2) source 2's
    const int nkv1 = KV2 ? (Skv1 + C::BN - 1) / C::BN : 0;
    const int nkv = KV2 ? nkv1 + (Skv - Skv1 + C::BN - 1) / C::BN : (Skv + C::BN - 1) / C::BN;
    // the map and first key row of key block j
    auto kv_src = [&](int j, const CUtensorMap *m1, const CUtensorMap *m2, const CUtensorMap *&m, int &row) {
        if (KV2 && j >= nkv1) {
            m = m2;
            row = (j - nkv1) * C::BN;
        } else {
            m = m1;
            row = j * C::BN;
        }
    };

    // Registers: the producer/MMA warpgroup gives (R - REGS_LOW) per thread back,
    // the two softmax warpgroups take (REGS_HIGH - R) each; the host launches
    // only builds with R >= MIN_LAUNCH_REGS, for which the release covers it.
    // Each register region runs to its own final barrier (no shared tail).
    if (warp < 4) {
    setmaxnreg_dec<C::REGS_LOW>();
    // Aborting: wait (bounded) for the copies a producer may still have in
    // flight -- at most the last NS of its ring (and the Q tiles) -- so that
    // none lands in shared memory after the CTA has exited. (copies complete
    // in microseconds; the drain never uses less than kDrainFloorNs even when
    // the caller's wait limit is tiny)
    const uint64_t drain_ns = wait_limit_ns > kDrainFloorNs ? wait_limit_ns : kDrainFloorNs;
    auto drain_copies = [&](uint32_t bar, uint32_t parity) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < drain_ns) {
        }
    };
    // Before TMEM is freed nothing may still run on the tensor core: each MMA
    // issuer commits to bar_drain (count 2) and waits for both commits.
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
    // Tensor-memory columns: S at 0 (the two tiles in turn), P_t at 128 + t*64,
    // O_t at 256 + t*HD (computed, not indexed, so nothing lands in local memory)
    auto tm_p = [&](int t) { return tmem + 128u + static_cast<uint32_t>(t) * 64u; };
    auto tm_o = [&](int t) { return tmem + 256u + static_cast<uint32_t>(t) * HD; };
    if (warp == 0) {
        // ------------------------------------------- producer: Q, then K ---
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            if (KV2) tma_prefetch_desc(&tm_k2);
            const uint64_t keep = l2_policy_evict_last();   // K: re-read by every Q tile of the head
            int nk = 0;   // (the Q tiles' loads were issued at set-up, evict-first: read once)  // K block loads issued so far
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % C::NSK;
                ok = wait_phase(bar_k_empty(s), ((j / C::NSK) & 1) ^ 1, SITE_PROD_K_EMPTY, wc);
                if (!ok) break;
                const CUtensorMap *mk;
                int krow;
                kv_src(j, &tm_k, &tm_k2, mk, krow);
                mbar_arrive_expect_tx(bar_k_full(s), C::TILE_BYTES);
                for (int h = 0; h < C::HALVES; ++h)
                    tma_load_3d(sbase + C::K_OFF + s * C::TILE_BYTES + h * C::HALF_BYTES, mk,
                                bar_k_full(s), h * 64, krow, bh, keep);
                ++nk;
            }
            if (!ok) {
                for (int j = (nk > C::NSK ? nk - C::NSK : 0); j < nk; ++j)
                    drain_copies(bar_k_full(j % C::NSK), (j / C::NSK) & 1);
                drain_copies(bar_q, 0);
            }
        }
    } else if (warp == 3) {
        // ------------------------------------------------- producer: V ---
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            if (KV2) tma_prefetch_desc(&tm_v2);
            const uint64_t keep = l2_policy_evict_last();   // V: re-read by every Q tile of the head
            int nv = 0;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % C::NSV;
                ok = wait_phase(bar_v_empty(s), ((j / C::NSV) & 1) ^ 1, SITE_PROD_V_EMPTY, wc);
                if (!ok) break;
                const CUtensorMap *mv;
                int vrow;
                kv_src(j, &tm_v, &tm_v2, mv, vrow);
                mbar_arrive_expect_tx(bar_v_full(s), C::TILE_BYTES);
                for (int h = 0; h < C::HALVES; ++h)
                    tma_load_3d(sbase + C::V_OFF + s * C::TILE_BYTES + h * C::HALF_BYTES, mv,
                                bar_v_full(s), h * 64, vrow, bh, keep);
                ++nv;
            }
            if (!ok)
                for (int j = (nv > C::NSV ? nv - C::NSV : 0); j < nv; ++j)
                    drain_copies(bar_v_full(j % C::NSV), (j / C::NSV) & 1);
        }
    } else if (warp == 1) {
        // -------------------------------------------- MMA issuer: S = QK^T ---
        // S = Q_t K_j^T : M=128, N=128, K=HD in steps of 16 (32 bytes) inside
        // each 128-byte swizzle row; the second 64-column half starts HALF_BYTES on.
        // The S buffer's copy-outs complete bar_s_free's phases in a fixed
        // order: S0(0), S1(0), S0(1), S1(1), ... So S1(j) waits for the phase
        // of S0(j) (even, parity 0) and S0(j+1) for that of S1(j) (odd,
        // parity 1); this thread is the only waiter and waits for every
        // phase in turn, so no wait can be two phases behind.
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false);  // Q.K^T, both K-major
            auto issue_s = [&](int t, int s) {
                const uint32_t qa = sbase + C::Q_OFF + t * C::TILE_BYTES;
                const uint32_t kb = sbase + C::K_OFF + s * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk / 4) * C::HALF_BYTES + (kk % 4) * 32;
                    mma_ss(tmem, smem_desc_sw128(qa + off, 16, 1024),
                           smem_desc_sw128(kb + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
                }
            };
            // Q tile t is ready when its TMA load landed (rope_q: when its rows
            // have been rotated); S_t(0) waits for that tile alone.
            bool ok = rope_q ? true : wait_phase(bar_q, 0, SITE_MMA_Q, wc);
            for (int j = 0; j < nkv && ok; ++j) {
                const int s = j % C::NSK;
                ok = wait_phase(bar_k_full(s), (j / C::NSK) & 1, SITE_MMA_K_FULL, wc);
                if (!ok) break;
                if (j > 0) {
                    ok = wait_phase(bar_s_free, 1, SITE_MMA_S_FREE, wc);  // S1(j-1) copied out
                    if (!ok) break;
                }
                if (rope_q && j == 0) {
                    ok = wait_phase(bar_qrot(0), 0, SITE_MMA_Q, wc);
                    if (!ok) break;
                }
                tc_fence_after_sync();
                issue_s(0, s);
                tc_commit(bar_s_full(0));
                ok = wait_phase(bar_s_free, 0, SITE_MMA_S_FREE, wc);      // S0(j) copied out
                if (!ok) break;
                if (rope_q && j == 0) {
                    ok = wait_phase(bar_qrot(1), 0, SITE_MMA_Q, wc);
                    if (!ok) break;
                }
                tc_fence_after_sync();
                issue_s(1, s);
                tc_commit(bar_s_full(1));
                tc_commit(bar_k_empty(s));
            }
            drain_mmas();
        }
        __syncwarp();
    } else {
        // ------------------------------------------ MMA issuer: O += P V ---
        // O_t += P_t V_j : M=128, N=HD, K=128 keys in steps of 16. P comes from
        // TMEM (16 keys = 8 columns); V rows are 128-byte swizzled, 16 keys =
        // 2048 bytes, the two 64-wide D halves are HALF_BYTES apart (LBO).
        // Its MMAs touch none of the S issuer's columns (P_t and O_t only), so
        // the two streams need no order between them beyond the softmax's
        // barriers; each issuer's commits track its own MMAs.
        if (lane == 0) {
            constexpr uint32_t IDESC_O = idesc_bf16_f32(128, HD, true);  // P.V, V is MN-major
            auto issue_pv = [&](int t, int s, bool acc) {
                const uint32_t vb = sbase + C::V_OFF + s * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    mma_ts(tm_o(t), tm_p(t) + kk * 8, smem_desc_sw128(vb + kk * 2048, C::HALF_BYTES, 1024),
                           IDESC_O, (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = true;
            for (int j = 0; j < nkv && ok; ++j) {
                const int s = j % C::NSV;
                ok = wait_phase(bar_v_full(s), (j / C::NSV) & 1, SITE_MMA_V_FULL, wc);
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
        const int t = (warp - 4) >> 2;     // Q tile of this warpgroup
        const int quad = warp & 3;         // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;  // row inside the tile
        const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t ts = tmem + lane_bits;                 // the shared S buffer
        const uint32_t tp = tmem + lane_bits + 128u + t * 64u;  // this tile's P
        const uint32_t to = tmem + lane_bits + 256u + t * HD;
        // valid keys of block j (1..128): fewer only in the last block of a source
        auto valid_keys = [&](int j) -> int {
            if constexpr (KV2) {
                if (j == nkv1 - 1) return Skv1 - (nkv1 - 1) * C::BN;
                if (j == nkv - 1) return Skv - Skv1 - (nkv - 1 - nkv1) * C::BN;
                return C::BN;
            } else {
                return j == nkv - 1 ? Skv - (nkv - 1) * C::BN : C::BN;
            }
        };
        float m = 0.f;   // running max of scaled logits (log2 units); set by block 0
        float l = 0.f;   // running sum of 2^(s - m)
        bool ok = true;
        if constexpr (rope_q) {
            ok = rope_q_tile_row<HD>(smem + C::Q_OFF + t * C::TILE_BYTES, row, q0 + t * C::BM + row, Sq, bar_q, wc,
                                     rope_tab, rope_geom);
            fence_proxy_async_smem();
            mbar_arrive(bar_qrot(t));
        }
        for (int j = 0; ok && j < nkv; ++j) {
            // every lane waits; the outcome is made warp-uniform so that the
            // warp-collective tcgen05 ops below never run on a partial warp
            ok = __all_sync(0xffffffffu, wait_phase(bar_s_full(t), j & 1, SITE_SM_S_FULL, wc));
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t sr[2][64];
#pragma unroll
            for (int c = 0; c < 2; ++c) tmem_ld_32x32b_x64(ts + c * 64, sr[c]);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 2; ++c) reg_fence(sr[c]);
            // S is in registers: the buffer may take the other tile's next S.
            tc_fence_before_sync();
            mbar_arrive(bar_s_free);
            // One block of the online softmax. MASKED: the last block of a key
            // source, whose columns >= kv_tail lie past that source's end (their
            // logits are zero-filled loads) and get probability 0.
            const int kv_tail = valid_keys(j);
            bool grow = false;
            float alpha = 1.0f;
            auto block = [&](auto masked_tag) {
                constexpr bool MASKED = decltype(masked_tag)::value;
                auto S = [&](int x) { return __uint_as_float(sr[x >> 6][x & 63]); };
                if constexpr (MASKED) {
#pragma unroll
                    for (int x = 0; x < 128; ++x)
                        if (x >= kv_tail) sr[x >> 6][x & 63] = __float_as_uint(NEG_SCALE ? INFINITY : -INFINITY);
                }
                // Row extreme of the raw logits: 8 independent 3-input chains.
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
                const float mnew = mx * scale_log2;
                // Stale-max rule: move m (and rescale O, l) only when the block
                // max exceeds it by more than 8 in log2 units.
                if (j == 0) {
                    m = mnew;
                } else if (mnew > m + 8.0f) {
                    grow = true;
                    alpha = ex2_approx(m - mnew);
                    m = mnew;
                    l *= alpha;
                }
                // P = 2^(s*scale_log2 - m): packed FMA for the affine step, MUFU
                // ex2, fp32 row sum (4 packed accumulators) before rounding to bf16.
                // All 64 packed columns are formed in registers first: only
                // their stores need PV_t(j-1) to have finished reading P_t.
                const uint64_t c2 = f2_pack(scale_log2, scale_log2);
                const uint64_t nm2 = f2_pack(-m, -m);
                uint64_t rs2[4] = {0, 0, 0, 0};
                uint32_t pk[64];
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {   // 64 keys -> 32 packed columns per half
#pragma unroll
                    for (int i = 0; i < 64; i += 2) {
                        const int x = hv * 64 + i;
                        float y0, y1;
                        f2_unpack(f2_fma(f2_pack(S(x), S(x + 1)), c2, nm2), y0, y1);
                        float p0, p1;
                        if ((i >> 1) % 8 < C::EMU_PER8) {
                            exp2_poly_pair(y0, y1, p0, p1);     // FMA pipe
                        } else {
                            p0 = ex2_approx(y0);                // MUFU
                            p1 = ex2_approx(y1);
                        }
                        if constexpr (MASKED) {
                            if (x >= kv_tail) p0 = 0.f;
                            if (x + 1 >= kv_tail) p1 = 0.f;
                        }
                        rs2[(i >> 1) & 3] = f2_add(rs2[(i >> 1) & 3], f2_pack(p0, p1));
                        pk[hv * 32 + (i >> 1)] = pack_bf16x2(p0, p1);
                    }
                }
                // P_t and O_t are free once PV_t(j-1) has completed.
                if (j > 0) {
                    ok = __all_sync(0xffffffffu, wait_phase(bar_pv_done(t), (j - 1) & 1, SITE_SM_PV_DONE, wc));
                    if (!ok) return;
                    tc_fence_after_sync();
                }
                tmem_st_32x32b_x64(tp, pk);
                float r0, r1, r2, r3;
                f2_unpack(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])), r0, r1);
                (void)r2;
                (void)r3;
                l += r0 + r1;
            };
            if (kv_tail < C::BN)
                block(std::true_type{});
            else
                block(std::false_type{});
            if (!ok) break;
            // O_t holds exactly PV_t(0..j-1) here: block() waited for PV_t(j-1)
            // before writing P, and PV_t(j) waits for this warpgroup's arrive.
            if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(to + c * 32, o);
                    tmem_ld_wait();
                    reg_fence(o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st_32x32b_x32(to + c * 32, o);
                }
            }
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(bar_p_full(t));
        }
        if (ok) ok = __all_sync(0xffffffffu, wait_phase(bar_pv_done(t), (nkv - 1) & 1, SITE_SM_O_FULL, wc));
        if (ok) {
            tc_fence_after_sync();
            // Epilogue: O / l -> bf16 into this tile's Q buffer (free now: every
            // MMA that read it has completed), in the same 128-byte swizzled
            // layout TMA uses, then one TMA store per 64-column half. Rows past
            // Sq fall outside the tensor map and are not written.
            const float inv_l = 1.0f / l;
            uint8_t *stage = smem + C::Q_OFF + t * C::TILE_BYTES;
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(to + c * 32, o);
                tmem_ld_wait();
                reg_fence(o);
                const int half = c >> 1;
#pragma unroll
                for (int g = 0; g < 4; ++g) {  // four 16-byte chunks of 8 values
                    const int chunk = (c & 1) * 4 + g;
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(o[g * 8 + 0]) * inv_l, __uint_as_float(o[g * 8 + 1]) * inv_l);
                    w.y = pack_bf16x2(__uint_as_float(o[g * 8 + 2]) * inv_l, __uint_as_float(o[g * 8 + 3]) * inv_l);
                    w.z = pack_bf16x2(__uint_as_float(o[g * 8 + 4]) * inv_l, __uint_as_float(o[g * 8 + 5]) * inv_l);
                    w.w = pack_bf16x2(__uint_as_float(o[g * 8 + 6]) * inv_l, __uint_as_float(o[g * 8 + 7]) * inv_l);
                    uint8_t *dst = stage + half * C::HALF_BYTES + row * 128 + ((chunk ^ (row & 7)) << 4);
                    *reinterpret_cast<uint4 *>(dst) = w;
                }
            }
            const int qrow = q0 + t * C::BM + row;
            if (lse != nullptr && qrow < Sq)
                lse[static_cast<int64_t>(bh) * Sq + qrow] = (m + __log2f(l)) * 0.69314718055994531f;
            fence_proxy_async_smem();
        }
        // Reached by all 128 threads of the warpgroup on every path.
        named_bar_sync(1 + t, 128);
        if (ok && warp == 4 + 4 * t && lane == 0 && q0 + t * C::BM < Sq) {
            for (int h = 0; h < C::HALVES; ++h)
                tma_store_3d(&tm_o, sbase + C::Q_OFF + t * C::TILE_BYTES + h * C::HALF_BYTES, h * 64,
                             q0 + t * C::BM, bh);
            tma_store_commit();
            tma_store_wait_read_all();   // only the shared-memory reads must finish before the CTA exits
        }
        tc_fence_before_sync();
        __syncthreads();
    }
}

// Self-test of the bounded wait: one warp waits on an mbarrier that nothing
// arrives on; after limit_ns it records REGEN_ERR_TIMEOUT (site SITE_SELFTEST)
// and returns. *done is set to 1 when the kernel has returned from the wait.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int *done)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    const WaitCtl wc{&abort_flag, limit_ns};
    const bool ok = __all_sync(0xffffffffu, wait_phase(smem_u32(&bar), 0, SITE_SELFTEST, wc));
    __syncthreads();
    if (threadIdx.x == 0) *done = ok ? 2 : 1;
}

// Self-test of the kernel's FMA-pipe exp2 (n even): y[i] = 2^x[i].
__global__ void exp2_poly_selftest_kernel(const float *__restrict__ x, float *__restrict__ y, int64_t npairs)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < npairs; i += stride) {
        float a, b;
        exp2_poly_pair(x[2 * i], x[2 * i + 1], a, b);
        y[2 * i] = a;
        y[2 * i + 1] = b;
    }
}

// Skv == 0: the empty softmax. out = 0, lse = -inf.
__global__ void attn_empty_kernel(uint4 *__restrict__ out, int64_t n16, float *__restrict__ lse,
                                  int64_t nrows)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n16; i += stride)
        out[i] = make_uint4(0, 0, 0, 0);
    if (lse)
        for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nrows; i += stride)
            lse[i] = -INFINITY;
}

}  // namespace regen
