/*
 * regen_attn.h -- C ABI of the DiT attention hot path on NVIDIA B200 (sm_100a).
 *
 * The operations are those of the ReGenVC decoder's diffusion transformer
 * (arXiv 2607.28144): exact softmax attention over the flattened latent
 * token sequence (blog.captcha.la page, "Technical innovations": the
 * Ulysses x Ring sequence parallelism keeps attention exact), its 3D rotary
 * embedding (the decoder matches the Wan2.1-Fun-Control architecture, blog
 * page "Methodology -- deep read"), and the log-sum-exp merge of partial
 * results over key blocks that Ring attention performs while it streams KV
 * blocks around the GPUs (same section).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major, in [B, H, S, D] order ("BHSD"): element
 *    (b, h, s, d) sits at ((b*H + h)*S + s)*D + d. No strides.
 *  - regen_bf16 is the bit pattern of a bfloat16 value; LSE values are fp32
 *    natural logarithms in units of the scaled logits.
 *  - Every pointer is a DEVICE pointer owned by the caller; the library keeps
 *    no reference after the call returns and allocates no device memory per
 *    call. Pointers must be 16-byte aligned.
 *  - Calls are asynchronous and stream-ordered on `stream` (NULL = the legacy
 *    default stream). The return value reports argument and launch errors
 *    only. A kernel that gives up on a bounded wait records a code that
 *    regen_last_device_error() reports after the caller synchronises.
 *  - Inputs and outputs must not overlap, except where "in place" is stated.
 */
#ifndef REGEN_ATTN_H
#define REGEN_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define REGEN_API __declspec(dllexport)
#else
#define REGEN_API __attribute__((visibility("default")))
#endif

typedef uint16_t regen_bf16;
typedef struct CUstream_st *regen_stream_t; /* same type as cudaStream_t */

typedef enum {
    REGEN_OK = 0,
    REGEN_ERR_INVALID_ARG = -1,  /* NULL pointer, negative size, non-finite scale */
    REGEN_ERR_UNSUPPORTED = -2,  /* head dim or size outside the supported set */
    REGEN_ERR_MISALIGNED = -3,   /* a pointer is not 16-byte aligned */
    REGEN_ERR_CUDA = -4,         /* the CUDA runtime or driver reported an error */
    REGEN_ERR_TIMEOUT = -5       /* a kernel gave up on a bounded wait */
} regen_status;

/*
 * regen_attn_fwd -- exact bidirectional multi-head softmax attention.
 *
 * For every (b, h) and query i < Sq, with s_j = scale * <q_i, k_j>, j < Skv:
 *     out_i = sum_j softmax(s)_j v_j        lse_i = ln sum_j exp(s_j)
 * (self-attention: Sq == Skv over the same latent tokens; cross-attention:
 * Skv conditioning / reference-frame tokens). Computed in one pass over key
 * blocks with an fp32 online softmax; QK^T and PV run on the tensor cores in
 * bf16 with fp32 accumulation; out is rounded to bf16 (nearest even).
 *
 *   q    [B, H, Sq,  D] bf16        k, v [B, H, Skv, D] bf16
 *   out  [B, H, Sq,  D] bf16        lse  [B, H, Sq] fp32, or NULL to skip it
 *   D    64 or 128 (else REGEN_ERR_UNSUPPORTED)
 *   scale  any finite float (1/sqrt(D) is the usual one)
 * B, H or Sq == 0: nothing to do, REGEN_OK. Skv == 0: out = 0, lse = -inf.
 * Sizes: B*H < 2^31, Sq and Skv < 2^31 with B*H*S*D < 2^62.
 */
REGEN_API int regen_attn_fwd(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v,
                             regen_bf16 *out, float *lse,
                             int B, int H, int Sq, int Skv, int D, float scale,
                             regen_stream_t stream);

/*
 * regen_attn_fwd_kv2 -- regen_attn_fwd over keys held in two separate
 * buffers: the cross-attention of the video tokens to the reference-frame
 * latent tokens and to the conditioning tokens (mlsanity.com abstract; blog
 * page, "Methodology -- deep read"), as one softmax over the two key sets
 * concatenated, [k_a ; k_b] with their values [v_a ; v_b]:
 *     out_i = sum_j softmax(s)_j v_j,  lse_i = ln sum_j exp(s_j),  j over Skv_a + Skv_b keys
 * In one launch: the kernel takes key blocks from source a, then from source
 * b, and masks each source's last block past that source's end, so nothing is
 * copied and no partial results are merged. Same arithmetic and rounding as
 * regen_attn_fwd on the concatenated keys (bit for bit when Skv_a is a
 * multiple of 128).
 *
 *   q    [B, H, Sq, D] bf16;  k_a, v_a [B, H, Skv_a, D];  k_b, v_b [B, H, Skv_b, D] bf16
 *   out  [B, H, Sq, D] bf16;  lse [B, H, Sq] fp32 or NULL
 *   D, scale and edge cases as regen_attn_fwd; Skv_a + Skv_b < 2^31. One
 *   source empty: the same as regen_attn_fwd over the other (its pointers
 *   may then be NULL). out and lse must not overlap any input.
 */
REGEN_API int regen_attn_fwd_kv2(const regen_bf16 *q, const regen_bf16 *k_a, const regen_bf16 *v_a,
                                 const regen_bf16 *k_b, const regen_bf16 *v_b,
                                 regen_bf16 *out, float *lse,
                                 int B, int H, int Sq, int Skv_a, int Skv_b, int D, float scale,
                                 regen_stream_t stream);

/*
 * regen_attn_fwd_rope3d -- self-attention with the 3D RoPE applied on the
 * way in: the same result, bit for bit, as regen_rope3d(q, k, ...) followed
 * by regen_attn_fwd(...), but q and k are left unmodified.
 *  - Q is rotated inside the attention kernel, on its 128-row tiles in
 *    shared memory right after they are loaded (fused into the Q load).
 *  - K is rotated once into the workspace: every query tile of a head reads
 *    every key tile, so rotating K per load would repeat the work for each of
 *    the ceil(S/256) query-tile pairs.
 *  - The (cos, sin) of every (axis, position, pair) are computed once, in fp64,
 *    into a small table at the start of the workspace, with its fp32 copy.
 *
 *   q, k, v, out, lse, B, H, D, scale, stream: as regen_attn_fwd
 *   Sq == Skv == T*Hh*Ww (else REGEN_ERR_INVALID_ARG); T, Hh, Ww, theta: as regen_rope3d
 *   workspace        device scratch owned by the caller, 256-byte aligned, at least
 *                    regen_attn_fwd_rope3d_workspace_bytes(B, H, T, Hh, Ww, D) bytes;
 *                    it must not overlap any other argument; its contents are
 *                    overwritten and need not be initialised
 *   workspace_bytes  its size (a smaller size is REGEN_ERR_INVALID_ARG)
 * Three launches on `stream`: the table, the rotated K, the attention.
 */
REGEN_API int regen_attn_fwd_rope3d(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v,
                                    regen_bf16 *out, float *lse,
                                    int B, int H, int Sq, int Skv, int D, float scale,
                                    regen_stream_t stream,
                                    int T, int Hh, int Ww, float theta,
                                    void *workspace, int64_t workspace_bytes);

/*
 * Bytes of workspace regen_attn_fwd_rope3d needs: with E = T*(D - 4*floor(D/6))/2
 * + (Hh + Ww)*floor(D/6) table entries, 16*E bytes of fp64 table and 8*E bytes
 * of fp32 table (each rounded up to a multiple of 256) plus B*H*S*D*2 bytes of
 * rotated K. Negative (a regen_status) for invalid sizes.
 */
REGEN_API int64_t regen_attn_fwd_rope3d_workspace_bytes(int B, int H, int T, int Hh, int Ww, int D);

/*
 * regen_attn_fwd_rope3d_noalloc -- regen_attn_fwd_rope3d without a workspace
 * argument, for callers that cannot allocate device memory: for example a
 * plug-in running inside a host application that owns every device
 * allocation, or a serving loop in which cudaMalloc/cudaFree (which may
 * synchronise the device and stall other work) are not permitted. It takes
 * the same arguments and gives the same results, but calls no allocator at
 * all (no cudaMalloc, no cudaFree, no allocating library routine).
 * The pages have no counterpart: this is a deployment convenience.
 *
 *  - Scratch: a fixed array of REGEN_NOALLOC_SCRATCH_BYTES (64 MiB) inside
 *    this library, kept by every device that loads the library until the
 *    process exits. A call whose scratch -- the same size
 *    regen_attn_fwd_rope3d_workspace_bytes reports -- exceeds it is rejected
 *    with REGEN_ERR_UNSUPPORTED before anything is launched (that admits e.g.
 *    12 heads of 10920 tokens at D = 128, not 40 heads of 31200).
 *  - Set-up: the first call made in a CUDA context (the one current when the
 *    call binds the data's device: normally that device's primary context)
 *    looks up the array's device address there (cudaGetSymbolAddress) and
 *    caches it for that context. Make that first call before any stream
 *    capture: a first call whose stream is capturing is refused with
 *    REGEN_ERR_INVALID_ARG, since the lookup may load the module.
 *  - Sharing: all calls use the same array, which keeps whatever the last
 *    call left in it. Nothing there needs clearing, since each call writes
 *    every byte it later reads. Calls whose work overlaps on the GPU (for
 *    example on two unordered streams) race on the array: order them.
 */
#define REGEN_NOALLOC_SCRATCH_BYTES (64LL << 20)
/* Size in bytes of that fixed array, as built into this library. */
REGEN_API int64_t regen_noalloc_scratch_bytes(void);
REGEN_API int regen_attn_fwd_rope3d_noalloc(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v,
                                            regen_bf16 *out, float *lse,
                                            int B, int H, int Sq, int Skv, int D, float scale,
                                            regen_stream_t stream,
                                            int T, int Hh, int Ww, float theta);

/*
 * regen_rope3d -- 3D rotary position embedding of Q and K, in place.
 *
 * The sequence is the flattened latent grid: token n = (t*Hh + y)*Ww + x,
 * S = T*Hh*Ww. The head dim splits into axis blocks t, h, w of widths
 * D - 4*floor(D/6), 2*floor(D/6), 2*floor(D/6) (44/42/42 at D = 128); in a
 * block of width d_a the pair (2j, 2j+1) turns by pos_a * theta^(-2j/d_a):
 *     x'_{2j} = x_{2j} cos - x_{2j+1} sin,   x'_{2j+1} = x_{2j} sin + x_{2j+1} cos
 * The result is that of fp64 angles and an fp64 rotation rounded once to
 * bf16 (nearest even). The kernel computes it in fp32 and proves, pair by
 * pair, that the fp32 value rounds to the same bf16; the pairs it cannot
 * prove (near a bf16 rounding boundary) are redone in fp64.
 *
 *   q, k   [B, H, S, D] bf16, rotated in place; either may be NULL (skipped),
 *          not both. q and k must not overlap.
 *   T, Hh, Ww > 0 (their product < 2^31); theta > 0 and finite
 *   D      even, multiple of 8, 8 <= D <= 512
 * B or H == 0: REGEN_OK, nothing done.
 */
REGEN_API int regen_rope3d(regen_bf16 *q, regen_bf16 *k, int T, int Hh, int Ww, float theta,
                           int B, int H, int D, regen_stream_t stream);

/*
 * regen_rope3d_shard -- regen_rope3d (inverse = 0) or regen_rope3d_bwd
 * (inverse = 1) on a sequence shard: q, k [B, H, S_local, D] hold the latent
 * tokens n0 .. n0 + S_local - 1 of the T x Hh x Ww grid, which set their
 * positions. Needs 0 <= n0 and n0 + S_local <= T*Hh*Ww (else
 * REGEN_ERR_INVALID_ARG); S_local == 0: REGEN_OK, nothing done. Same
 * arithmetic, rounding and other arguments as regen_rope3d, so a sharded
 * rotation equals the matching rows of the whole-grid one bit for bit.
 */
REGEN_API int regen_rope3d_shard(regen_bf16 *q, regen_bf16 *k, int T, int Hh, int Ww, float theta,
                                 int B, int H, int D, int n0, int S_local, int inverse, regen_stream_t stream);

/*
 * regen_lse_merge -- combine two partial attentions of the same queries
 * over disjoint key blocks a and b:
 *     m = max(lse_a, lse_b), w_a = exp(lse_a - m), w_b = exp(lse_b - m)
 *     out = (w_a o_a + w_b o_b) / (w_a + w_b),   lse_out = m + ln(w_a + w_b)
 * in fp32 per row; out rounded to bf16. Rows whose two LSEs are both -inf
 * (two empty key blocks) give out = 0 and lse_out = -inf.
 *
 *   o_a, o_b, out  [rows, D] bf16;  lse_a, lse_b  [rows] fp32
 *   lse_out        [rows] fp32 or NULL (skipped); must not overlap any other array
 *   rows = B*H*Sq >= 0;  D multiple of 8, 8 <= D <= 512
 * out may be exactly o_a or o_b (each element is read before the same thread
 * writes it); any other overlap is REGEN_ERR_INVALID_ARG.
 */
REGEN_API int regen_lse_merge(const regen_bf16 *o_a, const float *lse_a,
                              const regen_bf16 *o_b, const float *lse_b,
                              regen_bf16 *out, float *lse_out,
                              int64_t rows, int D, regen_stream_t stream);

/*
 * regen_attn_bwd -- gradients of regen_attn_fwd (the decoder's student DiT is
 * trained by distillation: arXiv 2607.28144, blog page "Technical
 * innovations"). With s_ij = scale <q_i, k_j>, the forward's out and lse,
 * and an upstream gradient dout:
 *     P_ij = exp(s_ij - lse_i),  dP_ij = <dout_i, v_j>,  delta_i = <dout_i, out_i>
 *     dS_ij = P_ij (dP_ij - delta_i)
 *     dv_j = sum_i P_ij dout_i,  dk_j = scale sum_i dS_ij q_i,  dq_i = scale sum_j dS_ij k_j
 * Products of bf16 tiles on the tensor cores with fp32 accumulation; P and dS
 * are rounded to bf16 before their products; results rounded once to bf16.
 * No atomics: the same inputs give the same bits on every run.
 *
 * Key blocks: when the keys were split into blocks whose partial results were
 * combined by regen_lse_merge, passing the MERGED out and lse with one
 * block's k, v gives that block's exact dk, dv and its share of dq; call once
 * per block with REGEN_ACCUM_DQ after the first to sum the dq shares.
 * Query blocks (Ring attention's backward, where a key shard meets every
 * rank's queries): REGEN_ACCUM_DKDV sums the dk, dv shares in the same way.
 *
 *   q, out, dout, dq  [B, H, Sq, D] bf16;  k, v, dk, dv  [B, H, Skv, D] bf16
 *   lse       [B, H, Sq] fp32 (the forward's, natural log)
 *   D         64 or 128 (else REGEN_ERR_UNSUPPORTED); scale finite
 *   workspace device scratch of at least regen_attn_bwd_workspace_bytes(B, H, Sq, D)
 *             bytes, 256-byte aligned, owned by the caller; overwritten.
 *   accumulate  a bit set, each bit one output: 0 writes every result;
 *             REGEN_ACCUM_DQ (1): dq = bf16(dq + result) (dq read first);
 *             REGEN_ACCUM_DKDV (2): dk, dv = bf16(dk + result), bf16(dv + result);
 *             any other value: REGEN_ERR_INVALID_ARG.
 * dq, dk, dv must not overlap each other, an input or the workspace.
 * Sq == 0: dk = dv = 0; Skv == 0: dq = 0 (each unchanged when it accumulates).
 * B or H == 0: REGEN_OK, nothing done.
 */
REGEN_API int regen_attn_bwd(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v,
                             const regen_bf16 *out, const float *lse, const regen_bf16 *dout,
                             regen_bf16 *dq, regen_bf16 *dk, regen_bf16 *dv,
                             int B, int H, int Sq, int Skv, int D, float scale,
                             regen_stream_t stream, void *workspace, int64_t workspace_bytes,
                             int accumulate);
enum { REGEN_ACCUM_DQ = 1, REGEN_ACCUM_DKDV = 2 };

/* Bytes of workspace regen_attn_bwd needs (B*H*ceil(Sq/128)*1024), or a
 * negative status for invalid sizes. */
REGEN_API int64_t regen_attn_bwd_workspace_bytes(int B, int H, int Sq, int D);

/*
 * regen_attn_bwd_kv2 -- gradients of regen_attn_fwd_kv2: the cross-attention
 * of the video tokens to the reference-frame and conditioning tokens (blog
 * page, "Methodology -- deep read") as one softmax over the two key sets
 * [k_a ; k_b], with that softmax's out and lse. The formulas of
 * regen_attn_bwd over the concatenated keys; dk, dv of each key go to its
 * source's buffer. Three launches for both sources:
 *  - one prep;
 *  - one dK/dV grid over the key tiles of a and then of b;
 *  - one dQ pass over all key tiles, accumulating dq in fp32 across both
 *    sources before its one rounding to bf16.
 * dk and dv equal regen_attn_bwd's for each source's keys, bit for bit. dq
 * has the same formula, rounded once instead of once per source.
 *
 *   q, out, dout, dq  [B, H, Sq, D] bf16;  lse [B, H, Sq] fp32
 *   k_a, v_a, dk_a, dv_a  [B, H, Skv_a, D];  k_b, v_b, dk_b, dv_b  [B, H, Skv_b, D] bf16
 *   D, scale, workspace (regen_attn_bwd_workspace_bytes(B, H, Sq, D) bytes) and
 *   accumulate as regen_attn_bwd (REGEN_ACCUM_DKDV applies to both sources).
 * The outputs must not overlap each other, an input or the workspace. One
 * source empty: the same as regen_attn_bwd over the other (the empty
 * source's pointers may then be NULL). Sq == 0: every dk, dv = 0 (unchanged
 * when accumulating). B or H == 0: REGEN_OK, nothing done.
 */
REGEN_API int regen_attn_bwd_kv2(const regen_bf16 *q, const regen_bf16 *k_a, const regen_bf16 *v_a,
                                 const regen_bf16 *k_b, const regen_bf16 *v_b, const regen_bf16 *out,
                                 const float *lse, const regen_bf16 *dout, regen_bf16 *dq, regen_bf16 *dk_a,
                                 regen_bf16 *dv_a, regen_bf16 *dk_b, regen_bf16 *dv_b, int B, int H, int Sq,
                                 int Skv_a, int Skv_b, int D, float scale, regen_stream_t stream,
                                 void *workspace, int64_t workspace_bytes, int accumulate);

/*
 * regen_rope3d_bwd -- gradient of regen_rope3d, in place: every pair of the
 * gradients dq, dk is turned back by its angle (the transposed rotation),
 *     g'_{2j} = g_{2j} cos + g_{2j+1} sin,   g'_{2j+1} = g_{2j+1} cos - g_{2j} sin
 * with the same angles, fp64 arithmetic, rounding and arguments as regen_rope3d.
 */
REGEN_API int regen_rope3d_bwd(regen_bf16 *dq, regen_bf16 *dk, int T, int Hh, int Ww, float theta,
                               int B, int H, int D, regen_stream_t stream);

/*
 * regen_quant_e4m3 -- blockwise FP8 quantisation for regen_attn_fwd_fp8 (a
 * speed/accuracy variant of the attention; the pages do not describe one).
 * For each (b, h) and each block of 128 consecutive rows (the last ragged):
 *     amax = max |x|,  scale = amax / 448,  inv = 448 / amax   (fp32; 1 and 1 if amax == 0)
 *     codes = E4M3(x * inv)   (OCP E4M3, round to nearest even, saturating at +-448)
 * so that x ~ codes * scale.
 *
 *   x       [B, H, S, D] bf16;  D = 64 or 128 (else REGEN_ERR_UNSUPPORTED)
 *   codes   [B, H, S, D] bytes, 16-byte aligned
 *   scales  [B, H, ceil(S/128)] fp32, 4-byte aligned
 * No overlaps. B, H or S == 0: REGEN_OK, nothing done.
 */
REGEN_API int regen_quant_e4m3(const regen_bf16 *x, uint8_t *codes, float *scales, int B, int H, int S, int D,
                               regen_stream_t stream);

/*
 * regen_attn_fwd_fp8 -- attention of the dequantised inputs (codes * block
 * scale, from regen_quant_e4m3) with E4M3 tensor-core products:
 *     S = Q8 K8^T (fp32 accumulate) times scale * sq * sk,  online softmax in fp32,
 *     O = sum_j P_j V_j with P rounded to E4M3 (in units of 2^-4 of the running
 *     row max, so at most 2^8) and V's block scales folded into P's exponent,
 *     out = O / l in bf16,  lse = m + ln l (fp32)
 * The row sum l uses P before rounding. Arguments and edge cases as
 * regen_attn_fwd, with the codes and scales in place of bf16 q, k, v:
 *   q8 [B,H,Sq,128], k8, v8 [B,H,Skv,128] bytes (16-byte aligned);
 *   q_scale [B,H,ceil(Sq/128)], k_scale, v_scale [B,H,ceil(Skv/128)] fp32.
 *   D must be 128 (else REGEN_ERR_UNSUPPORTED).
 */
REGEN_API int regen_attn_fwd_fp8(const uint8_t *q8, const float *q_scale, const uint8_t *k8, const float *k_scale,
                                 const uint8_t *v8, const float *v_scale, regen_bf16 *out, float *lse,
                                 int B, int H, int Sq, int Skv, int D, float scale, regen_stream_t stream);

/*
 * regen_qkv_proj -- the QKV projection that feeds the self-attention of a DiT
 * block (the decoder's DiT matches the Wan2.1 architecture: blog page,
 * "Methodology -- deep read"), fused with the per-head QK RMSNorm and the 3D
 * RoPE, writing q, k, v in the attention's [B, H, S, 128] layout:
 *     y = x W^T + b                     (bf16 tensor-core products, fp32 accumulate)
 *     [q | k | v] = y, head h of q at features h*128 .. h*128+127
 *     q_h <- RoPE( q_h / sqrt(mean(q_h^2) + eps) * gamma_q[h*128 ..] ), likewise k; v as is
 * with RoPE as in regen_rope3d (here in fp32 from an fp64-computed table) and
 * one rounding of each result to bf16.
 *
 *   x        [B, S, C] bf16 token features, S = T*Hh*Ww (else REGEN_ERR_INVALID_ARG)
 *   w        [3*H*128, C] bf16 (row n = output feature n);  C multiple of 8
 *   bias     [3*H*128] fp32 or NULL;  gamma_q, gamma_k  [H*128] fp32 or NULL (= 1)
 *   q, k, v  [B, H, S, 128] bf16 outputs (must not overlap anything else)
 *   D        must be 128 (else REGEN_ERR_UNSUPPORTED);  eps >= 0;  theta > 0
 *   workspace  >= regen_qkv_proj_workspace_bytes(T, Hh, Ww, D) bytes, 256-byte
 *            aligned, caller-owned (the RoPE table); overwritten
 * All pointers 16-byte aligned. B, S or H == 0: REGEN_OK, nothing done.
 */
REGEN_API int regen_qkv_proj(const regen_bf16 *x, const regen_bf16 *w, const float *bias, const float *gamma_q,
                             const float *gamma_k, regen_bf16 *q, regen_bf16 *k, regen_bf16 *v,
                             int B, int S, int C, int H, int D, int T, int Hh, int Ww, float theta, float eps,
                             regen_stream_t stream, void *workspace, int64_t workspace_bytes);

/* Bytes of workspace regen_qkv_proj needs, or a negative status. */
REGEN_API int64_t regen_qkv_proj_workspace_bytes(int T, int Hh, int Ww, int D);

/*
 * regen_out_proj -- the output projection after the attention, reading its
 * output in place: y[b, s, :] = o_tok W^T + b where o_tok[h*128 + d] =
 * o[b, h, s, d] (the heads of one token concatenated).
 *
 *   o     [B, H, S, 128] bf16 (the attention output);  D must be 128
 *   w     [N, H*128] bf16;  bias [N] fp32 or NULL;  N multiple of 8
 *   y     [B, S, N] bf16 output (must not overlap o, w, bias)
 * All pointers 16-byte aligned. B, S or N == 0: REGEN_OK, nothing done.
 */
REGEN_API int regen_out_proj(const regen_bf16 *o, const regen_bf16 *w, const float *bias, regen_bf16 *y,
                             int B, int S, int H, int D, int N, regen_stream_t stream);

/*
 * regen_selftest_exp2 -- diagnostic: evaluates, for each x[i], the FMA-pipe
 * 2^x that the attention kernel uses for part of its softmax probabilities
 * (degree-4 polynomial after Cody-Waite range reduction; inputs below -127
 * are clamped to -127, whose result is 0). x, y: device fp32 arrays of n
 * elements, n even. No counterpart on the pages: it exists so that tests can
 * check the kernel's exponential against CUDA's exp2f and its error bound.
 */
REGEN_API int regen_selftest_exp2(const float *x, float *y, int64_t n, regen_stream_t stream);

/*
 * regen_selftest_bounded_wait -- diagnostic of the failure-detection path: a
 * single-warp kernel waits, with the same bounded wait the attention kernel
 * uses, on a barrier that nothing ever completes. After limit_ns (1 ns .. 5 s)
 * it records REGEN_ERR_TIMEOUT with site code 10, writes 1 to *done (device
 * int; 2 would mean the wait unexpectedly succeeded) and returns, leaving the
 * context usable. No counterpart on the pages.
 */
REGEN_API int regen_selftest_bounded_wait(uint64_t limit_ns, int *done, regen_stream_t stream);

/* Human-readable text of a status code (static storage). */
REGEN_API const char *regen_status_str(int status);

/*
 * regen_last_cuda_error -- the CUDA result behind the last REGEN_ERR_CUDA that
 * a call on THIS host thread returned: a cudaError_t (its name in *name when
 * name is not NULL), or 100000 + a driver CUresult when a driver call failed
 * (a TMA descriptor could not be encoded, or the current context could not be
 * queried); 0 (name "none") when there is none. Reading clears it.
 * The string is static; the caller does not free it.
 */
REGEN_API int regen_last_cuda_error(const char **name);

/*
 * regen_last_device_error -- REGEN_OK, or the first error a kernel of this
 * library recorded since the previous call; clears the record:
 *   REGEN_ERR_TIMEOUT      a kernel gave up on a bounded wait;
 *   REGEN_ERR_UNSUPPORTED  the gradient's dK/dV kernel found its dynamic shared
 *                          memory not 1024-byte aligned and did nothing (detail 16;
 *                          it needs all 227 KB, with no room to realign).
 * It synchronises the device first (cudaDeviceSynchronize) and returns
 * REGEN_ERR_CUDA if that fails. *detail (may be NULL) receives a code naming
 * the wait or check that failed (0 if none).
 */
REGEN_API int regen_last_device_error(uint32_t *detail);

/*
 * regen_set_wait_limit_ns -- upper bound, in nanoseconds, on any single wait
 * inside the attention kernel (default 2e9 = 2 s; 0 restores the default).
 * A wait that exceeds it makes the kernel stop, record REGEN_ERR_TIMEOUT and
 * return; no wait in a correct run comes near the default.
 */
REGEN_API int regen_set_wait_limit_ns(uint64_t ns);

/* Version of this ABI (major*10000 + minor*100 + patch). */
REGEN_API int regen_version(void);

#ifdef __cplusplus
}
#endif

#endif /* REGEN_ATTN_H */
