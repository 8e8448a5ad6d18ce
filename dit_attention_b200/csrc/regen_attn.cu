// regen_attn.cu -- C ABI of the DiT attention hot path (declared in
// include/regen_attn.h): argument checks, TMA descriptor encoding, launches.
//
// Every argument check runs before the first CUDA call, so invalid calls are
// answered on machines without a GPU as well. Launches are asynchronous on
// the caller's stream; nothing here synchronises except
// regen_last_device_error().
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "regen_attn.h"

#include "ctx_cache.h"

#include "attn_bwd.cuh"
#include "attn_fp8.cuh"
#include "attn_fwd.cuh"
#include "lse_merge.cuh"
#include "proj_gemm.cuh"
#include "rope3d.cuh"

namespace {

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};

// The CUDA result behind this thread's last REGEN_ERR_CUDA: a cudaError_t, or a
// driver CUresult + kDriverErrorBase (descriptor encoding); 0 when none.
constexpr int kDriverErrorBase = 100000;
thread_local int g_last_cuda_error = 0;

int cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return REGEN_OK;
    g_last_cuda_error = static_cast<int>(e);
    return REGEN_ERR_CUDA;
}

// Status of the launches issued so far on this thread (and clears the runtime's record).
int launched() { return cuda_status(cudaGetLastError()); }

bool encoded(CUresult r)
{
    if (r == CUDA_SUCCESS) return true;
    g_last_cuda_error = kDriverErrorBase + static_cast<int>(r);
    return false;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, int64_t abytes, const void *b, int64_t bbytes)
{
    if (!a || !b || abytes <= 0 || bbytes <= 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Driver entry points, through the runtime (no libcuda link).
struct DriverCalls {
    CUresult (*pointer_attr)(void *, CUpointer_attribute, CUdeviceptr) = nullptr;
    CUresult (*ctx_get_current)(CUcontext *) = nullptr;
    CUresult (*ctx_get_device)(CUdevice *) = nullptr;
    CUresult (*ctx_set_current)(CUcontext) = nullptr;
    CUresult (*ctx_get_id)(CUcontext, unsigned long long *) = nullptr;
    bool ok() const { return pointer_attr && ctx_get_current && ctx_get_device && ctx_set_current && ctx_get_id; }
};

const DriverCalls &driver()
{
    static DriverCalls d;
    static std::once_flag once;
    std::call_once(once, [] {
        auto get = [](const char *name) -> void * {
            void *f = nullptr;
            cudaDriverEntryPointQueryResult q;
            return cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) == cudaSuccess &&
                           q == cudaDriverEntryPointSuccess ? f : nullptr;
        };
        d.pointer_attr = reinterpret_cast<decltype(d.pointer_attr)>(get("cuPointerGetAttribute"));
        d.ctx_get_current = reinterpret_cast<decltype(d.ctx_get_current)>(get("cuCtxGetCurrent"));
        d.ctx_get_device = reinterpret_cast<decltype(d.ctx_get_device)>(get("cuCtxGetDevice"));
        d.ctx_set_current = reinterpret_cast<decltype(d.ctx_set_current)>(get("cuCtxSetCurrent"));
        d.ctx_get_id = reinterpret_cast<decltype(d.ctx_get_id)>(get("cuCtxGetId"));
    });
    return d;
}

// For the duration of one call: the GPU that holds the device pointer `p` is
// current on this host thread, with a context. The caller's framework has
// usually made it current already, and then nothing changes. A thread on
// which no CUDA call has run (an autograd worker, a user's own thread) has no
// current context: the TMA descriptor encoding fails there and a launch would
// go to the runtime's default device, so the data's device is made current
// (cudaSetDevice, which binds its primary context) and left so, as the
// framework itself would. When another device's context is current, it is
// switched for the call and restored afterwards. The device comes from the
// pointer, so no other GPU's context is created.
class DeviceScope {
public:
    explicit DeviceScope(const void *p)
    {
        const DriverCalls &d = driver();
        if (!d.ok()) {
            status = cuda_status(cudaErrorNotSupported);
            return;
        }
        int ordinal = -1;
        if (!encoded(d.pointer_attr(&ordinal, CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL, reinterpret_cast<CUdeviceptr>(p)))) {
            status = REGEN_ERR_CUDA;
            return;
        }
        CUcontext cur = nullptr;
        if (!encoded(d.ctx_get_current(&cur))) {
            status = REGEN_ERR_CUDA;
            return;
        }
        if (cur != nullptr) {
            CUdevice dev = -1;
            if (!encoded(d.ctx_get_device(&dev))) {
                status = REGEN_ERR_CUDA;
                return;
            }
            if (static_cast<int>(dev) == ordinal) return;   // already the data's device
            prev_ = cur;
        }
        status = cuda_status(cudaSetDevice(ordinal));
    }
    ~DeviceScope()
    {
        if (prev_ != nullptr) driver().ctx_set_current(prev_);
    }
    DeviceScope(const DeviceScope &) = delete;
    DeviceScope &operator=(const DeviceScope &) = delete;
    int status = REGEN_OK;

private:
    CUcontext prev_ = nullptr;
};

// The driver's unique ID of the context current on this thread (the one
// DeviceScope bound); false when there is none or the driver cannot say.
bool current_context_id(unsigned long long *id)
{
    const DriverCalls &d = driver();
    CUcontext cur = nullptr;
    if (!d.ok() || !encoded(d.ctx_get_current(&cur))) return false;
    if (cur == nullptr) {
        g_last_cuda_error = kDriverErrorBase + static_cast<int>(CUDA_ERROR_INVALID_CONTEXT);
        return false;
    }
    return encoded(d.ctx_get_id(cur, id));
}

// One value per CUDA context, computed on the first call made in that context
// (ctx_cache.h): a kernel's shared-memory limit and a __device__ symbol's
// address belong to the module as loaded in one context, not to the process.
template <typename T>
class PerContext {
public:
    template <typename F>
    int get(F &&setup, T *value)
    {
        unsigned long long id = 0;
        if (!current_context_id(&id)) return REGEN_ERR_CUDA;
        return cache_.get(id, std::forward<F>(setup), value);
    }

private:
    regen::CtxCache<T, REGEN_ERR_CUDA> cache_;
};

// Raise a kernel's dynamic shared-memory limit in the current context and
// check that its compiled register count leaves room for the in-kernel
// register re-allocation (else REGEN_ERR_UNSUPPORTED: the split would wait
// forever, so the kernel is never launched).
// A setmaxnreg split of a 384-thread block (one 128-thread warpgroup down to
// `low` registers, two up to `high`) must fit the registers the block is
// launched with, `launch` per thread, or the increase waits forever.
// kernel_setup refuses a build with fewer than MIN_LAUNCH_REGS registers per
// thread; these checks tie each kernel's split to that minimum.
constexpr bool regsplit_fits(int low, int high, int launch) { return 128 * low + 256 * high <= 384 * launch; }
template <typename C>
constexpr bool split_fits() { return regsplit_fits(C::REGS_LOW, C::REGS_HIGH, C::MIN_LAUNCH_REGS); }
static_assert(split_fits<regen::AttnCfg<128>>() && split_fits<regen::AttnCfg<64>>(), "attention register split");
static_assert(split_fits<regen::Fp8Cfg>(), "FP8 attention register split");
static_assert(split_fits<regen::ProjCfg>(), "projection register split");
static_assert(split_fits<regen::BwdCfg<128>>() && split_fits<regen::BwdCfg<64>>(), "dK/dV register split");
static_assert(regsplit_fits(regen::BwdCfg<128>::B_REGS_LOW, regen::BwdCfg<128>::B_REGS_HIGH,
                            regen::BwdCfg<128>::B_MIN_LAUNCH_REGS),
              "dQ register split");

int kernel_setup(const void *fn, int smem_bytes, int min_regs)
{
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) {
        cudaGetLastError();   // not sticky: clear the runtime's record
        return cuda_status(e);
    }
    return fa.numRegs < min_regs ? static_cast<int>(REGEN_ERR_UNSUPPORTED) : static_cast<int>(REGEN_OK);
}

// [BH, S, D] bf16 viewed as a 3D tensor (D innermost), boxes of 64 x 128 x 1
// with the 128-byte swizzle; out-of-range rows read as zero.
bool make_bhsd_map(CUtensorMap *map, const void *base, int64_t BH, int64_t S, int64_t D)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D * 2), static_cast<cuuint64_t>(S * D * 2)};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return encoded(r);
}

// [BH, S, 128] E4M3 codes as a 3D tensor (128 codes innermost), boxes of
// 128 x 128 x 1 with the 128-byte swizzle; out-of-range rows read as zero.
bool make_u8_map(CUtensorMap *map, const void *base, int64_t BH, int64_t S)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(S * 128)};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return encoded(r);
}

// bf16 [d2][d1][d0] (d0 innermost) as a 3D tensor with boxes of box0 x box1 x 1
// and the 128-byte swizzle (box0 = 64: one 128-byte row); out-of-range reads zero.
bool make_bf16_map3(CUtensorMap *map, const void *base, int64_t d0, int64_t d1, int64_t d2, uint32_t box0,
                    uint32_t box1)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d0), static_cast<cuuint64_t>(d1), static_cast<cuuint64_t>(d2)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d0 * 2), static_cast<cuuint64_t>(d0 * d1 * 2)};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return encoded(r);
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return n;
}

template <int MODE>
int launch_proj(const CUtensorMap &ta, const CUtensorMap &tb, const regen::ProjShape &shape,
                const regen::ProjEpi &ep, cudaStream_t stream)
{
    using C = regen::ProjCfg;
    static PerContext<int> ready;
    const int attr_status = ready.get([](int *) {
        return kernel_setup(reinterpret_cast<const void *>(regen::proj_gemm_kernel<MODE>), C::SMEM_BYTES,
                            C::MIN_LAUNCH_REGS);
    }, nullptr);
    if (attr_status != REGEN_OK) return attr_status;
    const int64_t total = static_cast<int64_t>(shape.num_mt) * shape.num_nt;   // pair tiles
    const int sms = num_sms();
    if (sms < 2) return REGEN_ERR_CUDA;
    const int pairs = static_cast<int>(total < sms / 2 ? total : sms / 2);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const uint64_t limit = g_wait_limit_ns.load();
    if (cudaLaunchKernelEx(&cfg, regen::proj_gemm_kernel<MODE>, ta, tb, shape, ep, limit) != cudaSuccess)
        return REGEN_ERR_CUDA;
    return launched();
}

template <bool NEG>
int launch_attn_fp8(const uint8_t *q8, const float *qs, const uint8_t *k8, const float *ks, const uint8_t *v8,
                    const float *vs, regen_bf16 *out, float *lse, int64_t BH, int Sq, int Skv, float scale,
                    cudaStream_t stream)
{
    using C = regen::Fp8Cfg;
    static PerContext<int> ready;
    const int attr_status = ready.get([](int *) {
        return kernel_setup(reinterpret_cast<const void *>(regen::attn_fwd_fp8_kernel<NEG>), C::SMEM_BYTES,
                            C::MIN_LAUNCH_REGS);
    }, nullptr);
    if (attr_status != REGEN_OK) return attr_status;
    CUtensorMap tq, tk, tv, to;
    if (!make_u8_map(&tq, q8, BH, Sq) || !make_u8_map(&tk, k8, BH, Skv) || !make_u8_map(&tv, v8, BH, Skv) ||
        !make_bhsd_map(&to, out, BH, Sq, 128))
        return REGEN_ERR_CUDA;
    const int64_t grid = (Sq + 2 * C::BM - 1) / (2 * C::BM) * BH;
    if (grid > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    regen::attn_fwd_fp8_kernel<NEG><<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(
        tq, tk, tv, to, qs, ks, vs, lse, Sq, Skv, scale_log2, g_wait_limit_ns.load());
    return launched();
}

// Skv keys in k, v; with KV2 the first Skv1 of them in k, v and the other
// Skv - Skv1 in k2, v2 (one softmax over both).
template <int HD, bool NEG, bool ROPE_Q = false, bool KV2 = false>
int launch_attn(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v, regen_bf16 *out,
                float *lse, int64_t BH, int Sq, int Skv, float scale, cudaStream_t stream,
                regen::RopeTabs rope_tab = regen::RopeTabs{}, regen::RopeGeom geom = regen::RopeGeom{},
                const regen_bf16 *k2 = nullptr, const regen_bf16 *v2 = nullptr, int Skv1 = 0)
{
    using C = regen::AttnCfg<HD>;
    static PerContext<int> ready;
    const int attr_status = ready.get([](int *) {
        return kernel_setup(reinterpret_cast<const void *>(regen::attn_fwd_kernel<HD, NEG, ROPE_Q, KV2>),
                            C::SMEM_BYTES, C::MIN_LAUNCH_REGS);
    }, nullptr);
    if (attr_status != REGEN_OK) return attr_status;
    CUtensorMap tq, tk, tv, to, tk2, tv2;
    const int skv_a = KV2 ? Skv1 : Skv;
    if (!make_bhsd_map(&tq, q, BH, Sq, HD) || !make_bhsd_map(&tk, k, BH, skv_a, HD) ||
        !make_bhsd_map(&tv, v, BH, skv_a, HD) || !make_bhsd_map(&to, out, BH, Sq, HD))
        return REGEN_ERR_CUDA;
    if (KV2) {
        if (!make_bhsd_map(&tk2, k2, BH, Skv - Skv1, HD) || !make_bhsd_map(&tv2, v2, BH, Skv - Skv1, HD))
            return REGEN_ERR_CUDA;
    } else {
        tk2 = tk;   // unused by this instantiation
        tv2 = tv;
    }
    const int64_t npairs = (Sq + 2 * C::BM - 1) / (2 * C::BM);
    const int64_t grid = npairs * BH;
    if (grid > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    static_assert(!(ROPE_Q && KV2), "the RoPE-fused attention has one key source");
    regen::attn_fwd_kernel<HD, NEG, ROPE_Q, KV2><<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(
        tq, tk, tv, to, tk2, tv2, lse, Sq, Skv, Skv1, scale_log2, g_wait_limit_ns.load(), rope_tab, geom);
    return launched();
}

// Gradient launches: prep (delta, lse2) -> dK/dV -> dQ, all on `stream`.
template <int HD>
int launch_bwd(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v, const regen_bf16 *out,
               const float *lse, const regen_bf16 *dout, regen_bf16 *dq, regen_bf16 *dk, regen_bf16 *dv,
               int64_t BH, int Sq, int Skv, float scale, float *ws, bool accumulate, cudaStream_t stream);

int grid_for(int64_t work, int threads)
{
    int64_t blocks = (work + threads - 1) / threads;
    const int64_t cap = 148 * 32;  // grid-stride beyond ~32 resident blocks per SM
    if (blocks > cap) blocks = cap;
    return static_cast<int>(blocks < 1 ? 1 : blocks);
}

// The gradient launches: prep, dK/dV over the key tiles of both sources, dQ
// over both. A second key source (k2, v2, dk2, dv2; Skv2 keys) shares the
// queries, out, LSE and dO; Skv2 = 0 for one source.
template <int HD>
int launch_bwd(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v, const regen_bf16 *out,
               const float *lse, const regen_bf16 *dout, regen_bf16 *dq, regen_bf16 *dk, regen_bf16 *dv,
               int64_t BH, int Sq, int Skv, float scale, float *ws, bool acc_dq, bool acc_dkdv,
               cudaStream_t stream, const regen_bf16 *k2 = nullptr, const regen_bf16 *v2 = nullptr,
               regen_bf16 *dk2 = nullptr, regen_bf16 *dv2 = nullptr, int Skv2 = 0)
{
    using C = regen::BwdCfg<HD>;
    static PerContext<int> ready;
    const int attr_status = ready.get([](int *) {
        int st = kernel_setup(reinterpret_cast<const void *>(regen::attn_bwd_dkdv_kernel<HD, false>),
                              C::A_SMEM_BYTES, C::MIN_LAUNCH_REGS);
        if (st == REGEN_OK)
            st = kernel_setup(reinterpret_cast<const void *>(regen::attn_bwd_dkdv_kernel<HD, true>),
                              C::A_SMEM_BYTES, C::MIN_LAUNCH_REGS);
        if (st == REGEN_OK)
            st = kernel_setup(reinterpret_cast<const void *>(regen::attn_bwd_dq_kernel<HD, false>),
                              C::B_SMEM_BYTES, C::B_MIN_LAUNCH_REGS);
        if (st == REGEN_OK)
            st = kernel_setup(reinterpret_cast<const void *>(regen::attn_bwd_dq_kernel<HD, true>),
                              C::B_SMEM_BYTES, C::B_MIN_LAUNCH_REGS);
        return st;
    }, nullptr);
    if (attr_status != REGEN_OK) return attr_status;
    CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
    if (!make_bhsd_map(&tq, q, BH, Sq, HD) || !make_bhsd_map(&tk, k, BH, Skv, HD) ||
        !make_bhsd_map(&tv, v, BH, Skv, HD) || !make_bhsd_map(&tdo, dout, BH, Sq, HD) ||
        !make_bhsd_map(&tdq, dq, BH, Sq, HD) || !make_bhsd_map(&tdk, dk, BH, Skv, HD) ||
        !make_bhsd_map(&tdv, dv, BH, Skv, HD))
        return REGEN_ERR_CUDA;
    CUtensorMap tk2 = tk, tv2 = tv, tdk2 = tdk, tdv2 = tdv;   // not read when Skv2 = 0
    if (Skv2 > 0 &&
        (!make_bhsd_map(&tk2, k2, BH, Skv2, HD) || !make_bhsd_map(&tv2, v2, BH, Skv2, HD) ||
         !make_bhsd_map(&tdk2, dk2, BH, Skv2, HD) || !make_bhsd_map(&tdv2, dv2, BH, Skv2, HD)))
        return REGEN_ERR_CUDA;
    const int nq = (Sq + C::BM - 1) / C::BM;
    const int nkv = (Skv + C::BN - 1) / C::BN + (Skv2 + C::BN - 1) / C::BN;   // key tiles, both sources
    if (BH * nq > 0x7FFFFFFF || BH * nkv > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    const int64_t prep_work = BH * nq * 128 * (HD / 8);
    regen::attn_bwd_prep_kernel<<<grid_for(prep_work, 256), 256, 0, stream>>>(
        reinterpret_cast<const uint4 *>(out), reinterpret_cast<const uint4 *>(dout), lse, ws, BH, Sq, HD, nq);
    if (launched() != REGEN_OK) return REGEN_ERR_CUDA;
    const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    const uint64_t limit = g_wait_limit_ns.load();
    const uint16_t *dk_old = reinterpret_cast<const uint16_t *>(dk);
    const uint16_t *dv_old = reinterpret_cast<const uint16_t *>(dv);
    const uint16_t *dk_old2 = reinterpret_cast<const uint16_t *>(dk2);
    const uint16_t *dv_old2 = reinterpret_cast<const uint16_t *>(dv2);
    if (acc_dkdv)
        regen::attn_bwd_dkdv_kernel<HD, true><<<static_cast<unsigned>(BH * nkv), C::THREADS, C::A_SMEM_BYTES, stream>>>(
            tq, tk, tv, tdo, tdk, tdv, tk2, tv2, tdk2, tdv2, ws, Sq, Skv, Skv2, scale, scale_log2, limit, dk_old,
            dv_old, dk_old2, dv_old2);
    else
        regen::attn_bwd_dkdv_kernel<HD, false><<<static_cast<unsigned>(BH * nkv), C::THREADS, C::A_SMEM_BYTES, stream>>>(
            tq, tk, tv, tdo, tdk, tdv, tk2, tv2, tdk2, tdv2, ws, Sq, Skv, Skv2, scale, scale_log2, limit, dk_old,
            dv_old, dk_old2, dv_old2);
    if (launched() != REGEN_OK) return REGEN_ERR_CUDA;
    if (acc_dq)
        regen::attn_bwd_dq_kernel<HD, true><<<static_cast<unsigned>(BH * nq), C::THREADS, C::B_SMEM_BYTES, stream>>>(
            tq, tk, tv, tdo, tdq, tk2, tv2, dq, ws, Sq, Skv, Skv2, scale, scale_log2, limit);
    else
        regen::attn_bwd_dq_kernel<HD, false><<<static_cast<unsigned>(BH * nq), C::THREADS, C::B_SMEM_BYTES, stream>>>(
            tq, tk, tv, tdo, tdq, tk2, tv2, dq, ws, Sq, Skv, Skv2, scale, scale_log2, limit);
    return launched();
}

int64_t bwd_workspace_bytes(int64_t BH, int64_t Sq) { return BH * ((Sq + 127) / 128) * 1024; }

// Scratch of the RoPE-fused attention: the fp64 (cos, sin) table, its fp32
// copy, then the rotated K ([B*H, S, D] bf16), each starting on a 256-byte boundary.
int64_t rope_tab64_bytes(const regen::RopeGeom &g) { return (g.entries() * 16 + 255) / 256 * 256; }
int64_t rope_table_bytes(const regen::RopeGeom &g)
{
    return rope_tab64_bytes(g) + (g.entries() * 8 + 255) / 256 * 256;
}

int64_t rope_workspace_bytes(int64_t BH, int64_t S, const regen::RopeGeom &g, int D)
{
    return rope_table_bytes(g) + BH * S * D * 2;
}

// theta^(-local/width) for every pair of head dimension D (<= 512), in the
// RoPE's axis blocks t, h, w of widths D - 4*floor(D/6), 2*floor(D/6), 2*floor(D/6).
regen::RopeFreqs make_rope_freqs(int D, float theta)
{
    regen::RopeFreqs fr{};
    const int dh = 2 * (D / 6), dt = D - 2 * dh;
    for (int d = 0; d + 1 < D && d / 2 < 256; d += 2) {
        int local, width;
        if (d < dt) {
            local = d; width = dt;
        } else if (d < dt + dh) {
            local = d - dt; width = dh;
        } else {
            local = d - dt - dh; width = dh;
        }
        fr.f[d / 2] = std::pow(static_cast<double>(theta), -static_cast<double>(local) / static_cast<double>(width));
    }
    return fr;
}

// Rows per thread of a RoPE kernel whose grid has `blocks_x` blocks per row
// group: the fewest groups (each thread's angles serve the most rows) that
// still give about one wave of 128-thread blocks on a 148-SM part, and at
// least 4 rows per group (one load batch). Returns the rows per group;
// *groups receives the number of groups.
int rope_rows_per_group(int64_t blocks_x, int64_t rows, int64_t *groups)
{
    const int64_t target = 148LL * 8;
    int64_t g = (target + blocks_x - 1) / blocks_x;
    const int64_t gmax = (rows + 3) / 4;
    if (g > gmax) g = gmax;
    if (g > 32767) g = 32767;
    if (g < 1) g = 1;
    const int64_t per = (rows + g - 1) / g;
    *groups = (rows + per - 1) / per;
    return static_cast<int>(per);
}

// Table -> rotated K -> attention with Q rotated in shared memory; every
// argument has been checked by the caller. `scratch` holds at least
// rope_workspace_bytes(...) bytes of device memory.
int attn_rope3d_with_scratch(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v, regen_bf16 *out,
                             float *lse, int64_t BH, int S, int D, float scale, float theta,
                             const regen::RopeGeom &geom, uint8_t *scratch, cudaStream_t st)
{
    double *tab64 = reinterpret_cast<double *>(scratch);
    float2 *tab32 = reinterpret_cast<float2 *>(scratch + rope_tab64_bytes(geom));
    const regen::RopeTabs tab{tab64, tab32};
    regen_bf16 *k_rot = reinterpret_cast<regen_bf16 *>(scratch + rope_table_bytes(geom));
    regen::rope_table_kernel<<<grid_for(geom.entries(), 128), 128, 0, st>>>(tab64, tab32, geom,
                                                                           make_rope_freqs(D, theta));
    if (launched() != REGEN_OK) return REGEN_ERR_CUDA;
    const int64_t chunks = static_cast<int64_t>(S) * (D / 8);  // one thread per (token, chunk) and row group
    const int64_t bx = (chunks + 127) / 128;
    int64_t groups = 1;
    const int per = rope_rows_per_group(bx, BH, &groups);
    regen::rope_apply_kernel<<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(groups)), 128, 0, st>>>(
        k, k_rot, BH, S, D, geom, tab, per);
    if (launched() != REGEN_OK) return REGEN_ERR_CUDA;
    const bool neg = scale < 0.0f;
    if (D == 128)
        return neg ? launch_attn<128, true, true>(q, k_rot, v, out, lse, BH, S, S, scale, st, tab, geom)
                   : launch_attn<128, false, true>(q, k_rot, v, out, lse, BH, S, S, scale, st, tab, geom);
    return neg ? launch_attn<64, true, true>(q, k_rot, v, out, lse, BH, S, S, scale, st, tab, geom)
               : launch_attn<64, false, true>(q, k_rot, v, out, lse, BH, S, S, scale, st, tab, geom);
}

// ---------------------------------------------------------------------------
// Fixed scratch for regen_attn_fwd_rope3d_noalloc (declared in regen_attn.h).
// The array belongs to this library: every device that loads the library
// holds it until the process exits. In host code `g_noalloc_scratch` names
// only a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, looked up in the current context on the first call
// made in that context (the array has one copy per context that loads the
// module) and cached per context.
constexpr int64_t kNoAllocScratchBytes = REGEN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the fixed scratch in the current context. REGEN_ERR_INVALID_ARG
// when the address is not known yet and `st` is capturing a graph: the lookup
// may load the module, which a capture does not allow, so the first call in a
// context must come before any capture.
int noalloc_scratch_in_current_context(cudaStream_t st, uint8_t **scratch)
{
    static PerContext<uint8_t *> addr;
    return addr.get([st](uint8_t **p) {
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        const cudaError_t qe = cudaStreamIsCapturing(st, &cap);
        if (qe != cudaSuccess) {
            cudaGetLastError();
            return cuda_status(qe);
        }
        if (cap != cudaStreamCaptureStatusNone) return static_cast<int>(REGEN_ERR_INVALID_ARG);
        void *a = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
        if (e != cudaSuccess || a == nullptr) {
            cudaGetLastError();
            return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
        }
        *p = static_cast<uint8_t *>(a);
        return static_cast<int>(REGEN_OK);
    }, scratch);
}

// S_local < 0: the whole grid (n0 = 0, S = T*Hh*Ww).
int rope3d_common(regen_bf16 *q, regen_bf16 *k, int T, int Hh, int Ww, float theta, int B, int H, int D,
                  regen_stream_t stream, bool inverse, int n0 = 0, int S_local = -1)
{
    if (T <= 0 || Hh <= 0 || Ww <= 0 || B < 0 || H < 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(theta) || !(theta > 0.0f)) return REGEN_ERR_INVALID_ARG;
    if (D < 8 || D > 512 || (D % 8) != 0) return REGEN_ERR_UNSUPPORTED;
    const int64_t grid_tokens = static_cast<int64_t>(T) * Hh * Ww;
    if (grid_tokens > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (S_local >= 0 && (n0 < 0 || static_cast<int64_t>(n0) + S_local > grid_tokens)) return REGEN_ERR_INVALID_ARG;
    const int64_t S = S_local >= 0 ? S_local : grid_tokens;
    if (S == 0) return REGEN_OK;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0) return REGEN_OK;
    if (!q && !k) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k)) return REGEN_ERR_MISALIGNED;
    const int64_t bytes = BH * S * D * 2;
    if (overlaps(q, bytes, k, bytes)) return REGEN_ERR_INVALID_ARG;
    const int64_t work = S * (D / 8);
    const int threads = 128;
    const int64_t blocks = (work + threads - 1) / threads;
    if (blocks > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    int64_t groups = 1;   // row groups per tensor (q, then k: blockIdx.y)
    const int per = rope_rows_per_group((q && k) ? 2 * blocks : blocks, BH, &groups);
    const DeviceScope device(q ? q : k);
    if (device.status != REGEN_OK) return device.status;
    const dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(2 * groups));
    regen::rope3d_kernel<<<grid, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<uint16_t *>(q), reinterpret_cast<uint16_t *>(k), BH, static_cast<int>(S), Hh, Ww, D,
        make_rope_freqs(D, theta), inverse, S_local >= 0 ? n0 : 0, per, static_cast<int>(groups));
    return launched();
}


}  // namespace

extern "C" {

REGEN_API int regen_attn_fwd(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v,
                             regen_bf16 *out, float *lse, int B, int H, int Sq, int Skv, int D,
                             float scale, regen_stream_t stream)
{
    if (B < 0 || H < 0 || Sq < 0 || Skv < 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return REGEN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0 || Sq == 0) return REGEN_OK;
    if (BH > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (!q || !out || (Skv > 0 && (!k || !v))) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || !aligned16(lse) || (Skv > 0 && (!aligned16(k) || !aligned16(v))))
        return REGEN_ERR_MISALIGNED;
    const int64_t qbytes = BH * Sq * D * 2, kvbytes = BH * Skv * D * 2, lbytes = BH * Sq * 4;
    if (overlaps(out, qbytes, q, qbytes) || overlaps(out, qbytes, k, kvbytes) ||
        overlaps(out, qbytes, v, kvbytes) || overlaps(lse, lbytes, q, qbytes) ||
        overlaps(lse, lbytes, k, kvbytes) || overlaps(lse, lbytes, v, kvbytes) ||
        overlaps(lse, lbytes, out, qbytes))
        return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(out);
    if (device.status != REGEN_OK) return device.status;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (Skv == 0) {
        const int64_t n16 = qbytes / 16;
        regen::attn_empty_kernel<<<grid_for(n16, 256), 256, 0, st>>>(reinterpret_cast<uint4 *>(out), n16,
                                                                      lse, BH * Sq);
        return launched();
    }
    const bool neg = scale < 0.0f;
    if (D == 128)
        return neg ? launch_attn<128, true>(q, k, v, out, lse, BH, Sq, Skv, scale, st)
                   : launch_attn<128, false>(q, k, v, out, lse, BH, Sq, Skv, scale, st);
    return neg ? launch_attn<64, true>(q, k, v, out, lse, BH, Sq, Skv, scale, st)
               : launch_attn<64, false>(q, k, v, out, lse, BH, Sq, Skv, scale, st);
}

REGEN_API int regen_attn_fwd_kv2(const regen_bf16 *q, const regen_bf16 *k_a, const regen_bf16 *v_a,
                                 const regen_bf16 *k_b, const regen_bf16 *v_b, regen_bf16 *out, float *lse, int B,
                                 int H, int Sq, int Skv_a, int Skv_b, int D, float scale, regen_stream_t stream)
{
    if (B < 0 || H < 0 || Sq < 0 || Skv_a < 0 || Skv_b < 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return REGEN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(Skv_a) + Skv_b > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    // one source empty: the plain attention over the other
    if (Skv_b == 0) return regen_attn_fwd(q, k_a, v_a, out, lse, B, H, Sq, Skv_a, D, scale, stream);
    if (Skv_a == 0) return regen_attn_fwd(q, k_b, v_b, out, lse, B, H, Sq, Skv_b, D, scale, stream);
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0 || Sq == 0) return REGEN_OK;
    if (BH > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (!q || !out || !k_a || !v_a || !k_b || !v_b) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || !aligned16(lse) || !aligned16(k_a) || !aligned16(v_a) ||
        !aligned16(k_b) || !aligned16(v_b))
        return REGEN_ERR_MISALIGNED;
    const int64_t qbytes = BH * Sq * D * 2, abytes = BH * Skv_a * D * 2, bbytes = BH * Skv_b * D * 2,
                  lbytes = BH * Sq * 4;
    struct Span { const void *p; int64_t n; };
    const Span ins[5] = {{q, qbytes}, {k_a, abytes}, {v_a, abytes}, {k_b, bbytes}, {v_b, bbytes}};
    for (const Span &in : ins)
        if (overlaps(out, qbytes, in.p, in.n) || overlaps(lse, lbytes, in.p, in.n)) return REGEN_ERR_INVALID_ARG;
    if (overlaps(lse, lbytes, out, qbytes)) return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(out);
    if (device.status != REGEN_OK) return device.status;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int Skv = Skv_a + Skv_b;
    const bool neg = scale < 0.0f;
    const regen::RopeTabs nt{};
    const regen::RopeGeom ng{};
    if (D == 128)
        return neg ? launch_attn<128, true, false, true>(q, k_a, v_a, out, lse, BH, Sq, Skv, scale, st, nt, ng, k_b,
                                                         v_b, Skv_a)
                   : launch_attn<128, false, false, true>(q, k_a, v_a, out, lse, BH, Sq, Skv, scale, st, nt, ng,
                                                          k_b, v_b, Skv_a);
    return neg ? launch_attn<64, true, false, true>(q, k_a, v_a, out, lse, BH, Sq, Skv, scale, st, nt, ng, k_b, v_b,
                                                    Skv_a)
               : launch_attn<64, false, false, true>(q, k_a, v_a, out, lse, BH, Sq, Skv, scale, st, nt, ng, k_b, v_b,
                                                     Skv_a);
}

REGEN_API int64_t regen_attn_fwd_rope3d_workspace_bytes(int B, int H, int T, int Hh, int Ww, int D)
{
    if (B < 0 || H < 0 || T <= 0 || Hh <= 0 || Ww <= 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    const int64_t S = static_cast<int64_t>(T) * Hh * Ww;
    if (S > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    return rope_workspace_bytes(static_cast<int64_t>(B) * H, S, regen::RopeGeom::make(T, Hh, Ww, D), D);
}

REGEN_API int regen_attn_fwd_rope3d(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v,
                                    regen_bf16 *out, float *lse, int B, int H, int Sq, int Skv, int D,
                                    float scale, regen_stream_t stream, int T, int Hh, int Ww, float theta,
                                    void *workspace, int64_t workspace_bytes)
{
    if (B < 0 || H < 0 || Sq < 0 || Skv < 0 || D < 0 || T <= 0 || Hh <= 0 || Ww <= 0 || workspace_bytes < 0)
        return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !std::isfinite(theta) || !(theta > 0.0f)) return REGEN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    const int64_t S = static_cast<int64_t>(T) * Hh * Ww;
    if (S > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (Sq != S || Skv != S) return REGEN_ERR_INVALID_ARG;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0) return REGEN_OK;
    if (BH > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !out || !workspace) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return REGEN_ERR_MISALIGNED;
    const regen::RopeGeom geom = regen::RopeGeom::make(T, Hh, Ww, D);
    const int64_t need = rope_workspace_bytes(BH, S, geom, D);
    if (workspace_bytes < need) return REGEN_ERR_INVALID_ARG;
    const int64_t tbytes = BH * S * D * 2, lbytes = BH * S * 4;
    const void *ins[3] = {q, k, v};
    for (const void *in : ins)
        if (overlaps(out, tbytes, in, tbytes) || overlaps(lse, lbytes, in, tbytes) ||
            overlaps(workspace, need, in, tbytes))
            return REGEN_ERR_INVALID_ARG;
    if (overlaps(lse, lbytes, out, tbytes) || overlaps(workspace, need, out, tbytes) ||
        overlaps(workspace, need, lse, lbytes))
        return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(out);
    if (device.status != REGEN_OK) return device.status;
    return attn_rope3d_with_scratch(q, k, v, out, lse, BH, static_cast<int>(S), D, scale, theta, geom,
                                    static_cast<uint8_t *>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

REGEN_API int regen_attn_fwd_rope3d_noalloc(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v,
                                            regen_bf16 *out, float *lse, int B, int H, int Sq, int Skv, int D,
                                            float scale, regen_stream_t stream, int T, int Hh, int Ww,
                                            float theta)
{
    if (B < 0 || H < 0 || Sq < 0 || Skv < 0 || D < 0 || T <= 0 || Hh <= 0 || Ww <= 0)
        return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !std::isfinite(theta) || !(theta > 0.0f)) return REGEN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    const int64_t S = static_cast<int64_t>(T) * Hh * Ww;
    if (S > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (Sq != S || Skv != S) return REGEN_ERR_INVALID_ARG;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0) return REGEN_OK;
    if (BH > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    const regen::RopeGeom geom = regen::RopeGeom::make(T, Hh, Ww, D);
    // the whole scratch (table + rotated K) must fit the fixed array
    if (rope_workspace_bytes(BH, S, geom, D) > kNoAllocScratchBytes) return REGEN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !out) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
        return REGEN_ERR_MISALIGNED;
    const int64_t tbytes = BH * S * D * 2, lbytes = BH * S * 4;
    const void *ins[3] = {q, k, v};
    for (const void *in : ins)
        if (overlaps(out, tbytes, in, tbytes) || overlaps(lse, lbytes, in, tbytes)) return REGEN_ERR_INVALID_ARG;
    if (overlaps(lse, lbytes, out, tbytes)) return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(out);
    if (device.status != REGEN_OK) return device.status;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *scratch = nullptr;
    const int found = noalloc_scratch_in_current_context(st, &scratch);
    if (found != REGEN_OK) return found;
    // Every scratch byte this call reads is written earlier in the same call
    // (table, then rotated K), so nothing left by a previous call matters.
    return attn_rope3d_with_scratch(q, k, v, out, lse, BH, static_cast<int>(S), D, scale, theta, geom, scratch, st);
}

REGEN_API int64_t regen_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }


REGEN_API int regen_rope3d(regen_bf16 *q, regen_bf16 *k, int T, int Hh, int Ww, float theta, int B,
                           int H, int D, regen_stream_t stream)
{
    return rope3d_common(q, k, T, Hh, Ww, theta, B, H, D, stream, false);
}

REGEN_API int regen_rope3d_bwd(regen_bf16 *dq, regen_bf16 *dk, int T, int Hh, int Ww, float theta, int B,
                               int H, int D, regen_stream_t stream)
{
    return rope3d_common(dq, dk, T, Hh, Ww, theta, B, H, D, stream, true);
}

REGEN_API int regen_rope3d_shard(regen_bf16 *q, regen_bf16 *k, int T, int Hh, int Ww, float theta, int B, int H,
                                 int D, int n0, int S_local, int inverse, regen_stream_t stream)
{
    if (S_local < 0 || (inverse != 0 && inverse != 1)) return REGEN_ERR_INVALID_ARG;
    return rope3d_common(q, k, T, Hh, Ww, theta, B, H, D, stream, inverse != 0, n0, S_local);
}

REGEN_API int64_t regen_attn_bwd_workspace_bytes(int B, int H, int Sq, int D)
{
    if (B < 0 || H < 0 || Sq < 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    return bwd_workspace_bytes(static_cast<int64_t>(B) * H, Sq);
}

REGEN_API int regen_attn_bwd(const regen_bf16 *q, const regen_bf16 *k, const regen_bf16 *v,
                             const regen_bf16 *out, const float *lse, const regen_bf16 *dout, regen_bf16 *dq,
                             regen_bf16 *dk, regen_bf16 *dv, int B, int H, int Sq, int Skv, int D, float scale,
                             regen_stream_t stream, void *workspace, int64_t workspace_bytes, int accumulate)
{
    if (B < 0 || H < 0 || Sq < 0 || Skv < 0 || D < 0 || workspace_bytes < 0) return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return REGEN_ERR_INVALID_ARG;
    if (accumulate < 0 || accumulate > (REGEN_ACCUM_DQ | REGEN_ACCUM_DKDV)) return REGEN_ERR_INVALID_ARG;
    const bool acc_dq = (accumulate & REGEN_ACCUM_DQ) != 0, acc_dkdv = (accumulate & REGEN_ACCUM_DKDV) != 0;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0 || (Sq == 0 && Skv == 0)) return REGEN_OK;
    if (BH > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    const int64_t qbytes = BH * Sq * D * 2, kvbytes = BH * Skv * D * 2, lbytes = BH * Sq * 4;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (Sq == 0) {  // no query: dk = dv = 0 (unchanged when accumulating)
        if (!dk || !dv) return REGEN_ERR_INVALID_ARG;
        if (!aligned16(dk) || !aligned16(dv)) return REGEN_ERR_MISALIGNED;
        if (overlaps(dk, kvbytes, dv, kvbytes)) return REGEN_ERR_INVALID_ARG;
        if (acc_dkdv) return REGEN_OK;
        const DeviceScope device(dk);
        if (device.status != REGEN_OK) return device.status;
        for (regen_bf16 *z : {dk, dv}) {
            regen::attn_empty_kernel<<<grid_for(kvbytes / 16, 256), 256, 0, st>>>(reinterpret_cast<uint4 *>(z),
                                                                                 kvbytes / 16, nullptr, 0);
            if (launched() != REGEN_OK) return REGEN_ERR_CUDA;
        }
        return REGEN_OK;
    }
    if (Skv == 0) {  // no key: dq = 0 (unchanged when accumulating)
        if (!dq) return REGEN_ERR_INVALID_ARG;
        if (!aligned16(dq)) return REGEN_ERR_MISALIGNED;
        if (acc_dq) return REGEN_OK;
        const DeviceScope device(dq);
        if (device.status != REGEN_OK) return device.status;
        regen::attn_empty_kernel<<<grid_for(qbytes / 16, 256), 256, 0, st>>>(reinterpret_cast<uint4 *>(dq),
                                                                            qbytes / 16, nullptr, 0);
        return launched();
    }
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
        !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return REGEN_ERR_MISALIGNED;
    const int64_t need = bwd_workspace_bytes(BH, Sq);
    if (workspace_bytes < need) return REGEN_ERR_INVALID_ARG;
    struct Span { const void *p; int64_t n; };
    const Span ins[6] = {{q, qbytes}, {k, kvbytes}, {v, kvbytes}, {out, qbytes}, {lse, lbytes}, {dout, qbytes}};
    const Span outs[4] = {{dq, qbytes}, {dk, kvbytes}, {dv, kvbytes}, {workspace, need}};
    for (int a = 0; a < 4; ++a) {
        for (const Span &in : ins)
            if (overlaps(outs[a].p, outs[a].n, in.p, in.n)) return REGEN_ERR_INVALID_ARG;
        for (int b = a + 1; b < 4; ++b)
            if (overlaps(outs[a].p, outs[a].n, outs[b].p, outs[b].n)) return REGEN_ERR_INVALID_ARG;
    }
    float *ws = static_cast<float *>(workspace);
    const DeviceScope device(dq);
    if (device.status != REGEN_OK) return device.status;
    if (D == 128)
        return launch_bwd<128>(q, k, v, out, lse, dout, dq, dk, dv, BH, Sq, Skv, scale, ws, acc_dq, acc_dkdv, st);
    return launch_bwd<64>(q, k, v, out, lse, dout, dq, dk, dv, BH, Sq, Skv, scale, ws, acc_dq, acc_dkdv, st);
}

REGEN_API int regen_attn_bwd_kv2(const regen_bf16 *q, const regen_bf16 *k_a, const regen_bf16 *v_a,
                                 const regen_bf16 *k_b, const regen_bf16 *v_b, const regen_bf16 *out,
                                 const float *lse, const regen_bf16 *dout, regen_bf16 *dq, regen_bf16 *dk_a,
                                 regen_bf16 *dv_a, regen_bf16 *dk_b, regen_bf16 *dv_b, int B, int H, int Sq,
                                 int Skv_a, int Skv_b, int D, float scale, regen_stream_t stream,
                                 void *workspace, int64_t workspace_bytes, int accumulate)
{
    if (B < 0 || H < 0 || Sq < 0 || Skv_a < 0 || Skv_b < 0 || D < 0 || workspace_bytes < 0)
        return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return REGEN_ERR_INVALID_ARG;
    if (accumulate < 0 || accumulate > (REGEN_ACCUM_DQ | REGEN_ACCUM_DKDV)) return REGEN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(Skv_a) + Skv_b > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0) return REGEN_OK;
    if (Skv_b == 0)
        return regen_attn_bwd(q, k_a, v_a, out, lse, dout, dq, dk_a, dv_a, B, H, Sq, Skv_a, D, scale, stream,
                              workspace, workspace_bytes, accumulate);
    if (Skv_a == 0)
        return regen_attn_bwd(q, k_b, v_b, out, lse, dout, dq, dk_b, dv_b, B, H, Sq, Skv_b, D, scale, stream,
                              workspace, workspace_bytes, accumulate);
    if (Sq == 0) {  // dk = dv = 0 for both sources (unchanged when accumulating)
        // every check of both calls first, so that an error launches nothing
        if (!dk_a || !dv_a || !dk_b || !dv_b) return REGEN_ERR_INVALID_ARG;
        if (!aligned16(dk_a) || !aligned16(dv_a) || !aligned16(dk_b) || !aligned16(dv_b)) return REGEN_ERR_MISALIGNED;
        const int64_t ba = BH * Skv_a * D * 2, bb = BH * Skv_b * D * 2;
        if (overlaps(dk_a, ba, dv_a, ba) || overlaps(dk_b, bb, dv_b, bb) || overlaps(dk_a, ba, dk_b, bb) ||
            overlaps(dk_a, ba, dv_b, bb) || overlaps(dv_a, ba, dk_b, bb) || overlaps(dv_a, ba, dv_b, bb))
            return REGEN_ERR_INVALID_ARG;
        const int st = regen_attn_bwd(q, k_a, v_a, out, lse, dout, dq, dk_a, dv_a, B, H, 0, Skv_a, D, scale,
                                      stream, workspace, workspace_bytes, accumulate);
        if (st != REGEN_OK) return st;
        return regen_attn_bwd(q, k_b, v_b, out, lse, dout, dq, dk_b, dv_b, B, H, 0, Skv_b, D, scale, stream,
                              workspace, workspace_bytes, accumulate);
    }
    const bool acc_dq = (accumulate & REGEN_ACCUM_DQ) != 0, acc_dkdv = (accumulate & REGEN_ACCUM_DKDV) != 0;
    if (BH > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (!q || !k_a || !v_a || !k_b || !v_b || !out || !lse || !dout || !dq || !dk_a || !dv_a || !dk_b || !dv_b ||
        !workspace)
        return REGEN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_a) || !aligned16(v_a) || !aligned16(k_b) || !aligned16(v_b) ||
        !aligned16(out) || !aligned16(lse) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk_a) ||
        !aligned16(dv_a) || !aligned16(dk_b) || !aligned16(dv_b) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return REGEN_ERR_MISALIGNED;
    const int64_t need = bwd_workspace_bytes(BH, Sq);
    if (workspace_bytes < need) return REGEN_ERR_INVALID_ARG;
    const int64_t qbytes = BH * Sq * D * 2, abytes = BH * Skv_a * D * 2, bbytes = BH * Skv_b * D * 2,
                  lbytes = BH * Sq * 4;
    struct Span { const void *p; int64_t n; };
    const Span ins[8] = {{q, qbytes},   {k_a, abytes}, {v_a, abytes},  {k_b, bbytes},
                         {v_b, bbytes}, {out, qbytes}, {lse, lbytes},  {dout, qbytes}};
    const Span outs[6] = {{dq, qbytes},   {dk_a, abytes}, {dv_a, abytes},
                          {dk_b, bbytes}, {dv_b, bbytes}, {workspace, need}};
    for (int a = 0; a < 6; ++a) {
        for (const Span &in : ins)
            if (overlaps(outs[a].p, outs[a].n, in.p, in.n)) return REGEN_ERR_INVALID_ARG;
        for (int b = a + 1; b < 6; ++b)
            if (overlaps(outs[a].p, outs[a].n, outs[b].p, outs[b].n)) return REGEN_ERR_INVALID_ARG;
    }
    float *ws = static_cast<float *>(workspace);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const DeviceScope device(dq);
    if (device.status != REGEN_OK) return device.status;
    if (D == 128)
        return launch_bwd<128>(q, k_a, v_a, out, lse, dout, dq, dk_a, dv_a, BH, Sq, Skv_a, scale, ws, acc_dq,
                               acc_dkdv, st, k_b, v_b, dk_b, dv_b, Skv_b);
    return launch_bwd<64>(q, k_a, v_a, out, lse, dout, dq, dk_a, dv_a, BH, Sq, Skv_a, scale, ws, acc_dq, acc_dkdv,
                          st, k_b, v_b, dk_b, dv_b, Skv_b);
}

REGEN_API int regen_lse_merge(const regen_bf16 *o_a, const float *lse_a, const regen_bf16 *o_b,
                              const float *lse_b, regen_bf16 *out, float *lse_out, int64_t rows, int D,
                              regen_stream_t stream)
{
    if (rows < 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (D < 8 || D > 512 || (D % 8) != 0) return REGEN_ERR_UNSUPPORTED;
    if (rows == 0) return REGEN_OK;
    if (!o_a || !lse_a || !o_b || !lse_b || !out) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(out) || !aligned16(lse_a) || !aligned16(lse_b) ||
        !aligned16(lse_out))
        return REGEN_ERR_MISALIGNED;
    const int64_t obytes = rows * D * 2, lbytes = rows * 4;
    if (overlaps(lse_out, lbytes, lse_a, lbytes) || overlaps(lse_out, lbytes, lse_b, lbytes) ||
        overlaps(lse_out, lbytes, o_a, obytes) || overlaps(lse_out, lbytes, o_b, obytes) ||
        overlaps(lse_out, lbytes, out, obytes) || overlaps(out, obytes, lse_a, lbytes) ||
        overlaps(out, obytes, lse_b, lbytes))
        return REGEN_ERR_INVALID_ARG;
    // out may coincide exactly with o_a or o_b (each chunk is read before it is
    // written by the same thread); a partial overlap is rejected.
    if ((overlaps(out, obytes, o_a, obytes) && out != o_a) || (overlaps(out, obytes, o_b, obytes) && out != o_b))
        return REGEN_ERR_INVALID_ARG;
    const int64_t work = rows * (D / 8);
    const DeviceScope device(out);
    if (device.status != REGEN_OK) return device.status;
    regen::lse_merge_kernel<<<grid_for(work, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4 *>(o_a), lse_a, reinterpret_cast<const uint4 *>(o_b), lse_b,
        reinterpret_cast<uint4 *>(out), lse_out, rows, D);
    return launched();
}

REGEN_API int regen_quant_e4m3(const regen_bf16 *x, uint8_t *codes, float *scales, int B, int H, int S, int D,
                               regen_stream_t stream)
{
    if (B < 0 || H < 0 || S < 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return REGEN_ERR_UNSUPPORTED;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0 || S == 0) return REGEN_OK;
    if (!x || !codes || !scales) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return REGEN_ERR_MISALIGNED;
    const int64_t nb = (S + 127) / 128;
    if (BH * nb > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    const int64_t xbytes = BH * S * D * 2, cbytes = BH * S * D, sbytes = BH * nb * 4;
    if (overlaps(codes, cbytes, x, xbytes) || overlaps(scales, sbytes, x, xbytes) ||
        overlaps(scales, sbytes, codes, cbytes))
        return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(codes);
    if (device.status != REGEN_OK) return device.status;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>(BH * nb);
    if (D == 128)
        regen::quant_e4m3_kernel<128><<<grid, 256, 0, st>>>(reinterpret_cast<const uint4 *>(x),
                                                            reinterpret_cast<uint2 *>(codes), scales, S,
                                                            static_cast<int>(nb));
    else
        regen::quant_e4m3_kernel<64><<<grid, 256, 0, st>>>(reinterpret_cast<const uint4 *>(x),
                                                           reinterpret_cast<uint2 *>(codes), scales, S,
                                                           static_cast<int>(nb));
    return launched();
}

REGEN_API int regen_attn_fwd_fp8(const uint8_t *q8, const float *q_scale, const uint8_t *k8, const float *k_scale,
                                 const uint8_t *v8, const float *v_scale, regen_bf16 *out, float *lse, int B, int H,
                                 int Sq, int Skv, int D, float scale, regen_stream_t stream)
{
    if (B < 0 || H < 0 || Sq < 0 || Skv < 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return REGEN_ERR_INVALID_ARG;
    if (D != 128) return REGEN_ERR_UNSUPPORTED;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH == 0 || Sq == 0) return REGEN_OK;
    if (BH > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (!q8 || !q_scale || !out || (Skv > 0 && (!k8 || !k_scale || !v8 || !v_scale))) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(q8) || !aligned16(out) || !aligned16(lse) || (Skv > 0 && (!aligned16(k8) || !aligned16(v8))) ||
        (reinterpret_cast<uintptr_t>(q_scale) & 3u) || (reinterpret_cast<uintptr_t>(k_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(v_scale) & 3u))
        return REGEN_ERR_MISALIGNED;
    const int64_t obytes = BH * Sq * D * 2, lbytes = BH * Sq * 4;
    const int64_t qb = BH * Sq * D, kvb = BH * Skv * D;
    const int64_t qsb = BH * ((Sq + 127) / 128) * 4, kvsb = BH * ((Skv + 127) / 128) * 4;
    struct Span { const void *p; int64_t n; };
    const Span ins[6] = {{q8, qb}, {k8, kvb}, {v8, kvb}, {q_scale, qsb}, {k_scale, kvsb}, {v_scale, kvsb}};
    for (const Span &in : ins)
        if (overlaps(out, obytes, in.p, in.n) || overlaps(lse, lbytes, in.p, in.n)) return REGEN_ERR_INVALID_ARG;
    if (overlaps(lse, lbytes, out, obytes)) return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(out);
    if (device.status != REGEN_OK) return device.status;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (Skv == 0) {
        regen::attn_empty_kernel<<<grid_for(obytes / 16, 256), 256, 0, st>>>(reinterpret_cast<uint4 *>(out),
                                                                            obytes / 16, lse, BH * Sq);
        return launched();
    }
    return scale < 0.0f ? launch_attn_fp8<true>(q8, q_scale, k8, k_scale, v8, v_scale, out, lse, BH, Sq, Skv, scale, st)
                        : launch_attn_fp8<false>(q8, q_scale, k8, k_scale, v8, v_scale, out, lse, BH, Sq, Skv, scale, st);
}

REGEN_API int64_t regen_qkv_proj_workspace_bytes(int T, int Hh, int Ww, int D)
{
    if (T <= 0 || Hh <= 0 || Ww <= 0 || D < 0) return REGEN_ERR_INVALID_ARG;
    if (D != 128) return REGEN_ERR_UNSUPPORTED;
    return (regen::RopeGeom::make(T, Hh, Ww, D).entries() * 8 + 255) / 256 * 256;
}

REGEN_API int regen_qkv_proj(const regen_bf16 *x, const regen_bf16 *w, const float *bias, const float *gamma_q,
                             const float *gamma_k, regen_bf16 *q, regen_bf16 *k, regen_bf16 *v, int B, int S, int C,
                             int H, int D, int T, int Hh, int Ww, float theta, float eps, regen_stream_t stream,
                             void *workspace, int64_t workspace_bytes)
{
    if (B < 0 || S < 0 || C < 0 || H < 0 || D < 0 || T <= 0 || Hh <= 0 || Ww <= 0 || workspace_bytes < 0)
        return REGEN_ERR_INVALID_ARG;
    if (!std::isfinite(theta) || !(theta > 0.0f) || !std::isfinite(eps) || eps < 0.0f) return REGEN_ERR_INVALID_ARG;
    if (D != 128 || (C % 8) != 0) return REGEN_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(T) * Hh * Ww != S) return REGEN_ERR_INVALID_ARG;
    if (B == 0 || S == 0 || H == 0) return REGEN_OK;
    const int64_t N = 3LL * H * 128;
    if (C == 0 || N > 0x7FFFFFFF || static_cast<int64_t>(B) * H > 0x7FFFFFFF) return REGEN_ERR_UNSUPPORTED;
    if (!x || !w || !q || !k || !v || !workspace) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(bias) ||
        !aligned16(gamma_q) || !aligned16(gamma_k) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return REGEN_ERR_MISALIGNED;
    const regen::RopeGeom geom = regen::RopeGeom::make(T, Hh, Ww, D);
    const int64_t tab_bytes = geom.entries() * 8;
    if (workspace_bytes < tab_bytes) return REGEN_ERR_INVALID_ARG;
    const int64_t xb = static_cast<int64_t>(B) * S * C * 2, wb = N * C * 2, ob = static_cast<int64_t>(B) * H * S * 256;
    struct Span { const void *p; int64_t n; };
    const Span ins[6] = {{x, xb}, {w, wb}, {bias, N * 4}, {gamma_q, H * 512LL}, {gamma_k, H * 512LL}, {workspace, tab_bytes}};
    const Span outs[3] = {{q, ob}, {k, ob}, {v, ob}};
    for (int a = 0; a < 3; ++a) {
        for (const Span &in : ins)
            if (overlaps(outs[a].p, outs[a].n, in.p, in.n)) return REGEN_ERR_INVALID_ARG;
        for (int b2 = a + 1; b2 < 3; ++b2)
            if (overlaps(outs[a].p, outs[a].n, outs[b2].p, outs[b2].n)) return REGEN_ERR_INVALID_ARG;
    }
    for (int a = 0; a < 5; ++a)
        if (overlaps(workspace, tab_bytes, ins[a].p, ins[a].n)) return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(q);
    if (device.status != REGEN_OK) return device.status;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float2 *tab = static_cast<float2 *>(workspace);
    regen::rope_table_f32_kernel<<<grid_for(geom.entries(), 128), 128, 0, st>>>(tab, geom, make_rope_freqs(D, theta));
    if (launched() != REGEN_OK) return REGEN_ERR_CUDA;
    CUtensorMap ta, tb;
    if (!make_bf16_map3(&ta, x, C, S, B, 64, 128) || !make_bf16_map3(&tb, w, C, N, 1, 64, 128)) return REGEN_ERR_CUDA;
    regen::ProjShape shape{B, S, C, static_cast<int>(N), H, B * ((S + 255) / 256), static_cast<int>((N + 255) / 256)};
    regen::ProjEpi ep{bias, gamma_q, gamma_k, q, k, v, tab, geom, eps};
    return launch_proj<regen::PROJ_QKV>(ta, tb, shape, ep, st);
}

REGEN_API int regen_out_proj(const regen_bf16 *o, const regen_bf16 *w, const float *bias, regen_bf16 *y, int B,
                             int S, int H, int D, int N, regen_stream_t stream)
{
    if (B < 0 || S < 0 || H < 0 || D < 0 || N < 0) return REGEN_ERR_INVALID_ARG;
    if (D != 128 || (N % 8) != 0) return REGEN_ERR_UNSUPPORTED;
    if (B == 0 || S == 0 || N == 0) return REGEN_OK;
    if (H == 0) return REGEN_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * H > 0x7FFFFFFF || static_cast<int64_t>(H) * 128 > 0x7FFFFFFF)
        return REGEN_ERR_UNSUPPORTED;
    if (!o || !w || !y) return REGEN_ERR_INVALID_ARG;
    if (!aligned16(o) || !aligned16(w) || !aligned16(y) || !aligned16(bias)) return REGEN_ERR_MISALIGNED;
    const int64_t K = static_cast<int64_t>(H) * 128;
    const int64_t obytes = static_cast<int64_t>(B) * H * S * 256, wbytes = N * K * 2,
                  ybytes = static_cast<int64_t>(B) * S * N * 2;
    if (overlaps(y, ybytes, o, obytes) || overlaps(y, ybytes, w, wbytes) || overlaps(y, ybytes, bias, N * 4LL))
        return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(y);
    if (device.status != REGEN_OK) return device.status;
    CUtensorMap ta, tb;
    if (!make_bhsd_map(&ta, o, static_cast<int64_t>(B) * H, S, 128) || !make_bf16_map3(&tb, w, K, N, 1, 64, 128))
        return REGEN_ERR_CUDA;
    regen::ProjShape shape{B, S, static_cast<int>(K), N, H, B * ((S + 255) / 256), (N + 255) / 256};
    regen::ProjEpi ep{bias, nullptr, nullptr, y, nullptr, nullptr, nullptr, regen::RopeGeom{}, 0.0f};
    return launch_proj<regen::PROJ_OUT>(ta, tb, shape, ep, reinterpret_cast<cudaStream_t>(stream));
}

REGEN_API int regen_selftest_exp2(const float *x, float *y, int64_t n, regen_stream_t stream)
{
    if (n < 0 || (n & 1)) return REGEN_ERR_INVALID_ARG;
    if (n == 0) return REGEN_OK;
    if (!x || !y) return REGEN_ERR_INVALID_ARG;
    const int64_t npairs = n / 2;
    const DeviceScope device(y);
    if (device.status != REGEN_OK) return device.status;
    regen::exp2_poly_selftest_kernel<<<grid_for(npairs, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        x, y, npairs);
    return launched();
}

REGEN_API int regen_selftest_bounded_wait(uint64_t limit_ns, int *done, regen_stream_t stream)
{
    if (!done) return REGEN_ERR_INVALID_ARG;
    if (limit_ns == 0 || limit_ns > 5000000000ull) return REGEN_ERR_INVALID_ARG;
    const DeviceScope device(done);
    if (device.status != REGEN_OK) return device.status;
    regen::bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, done);
    return launched();
}

REGEN_API int regen_last_cuda_error(const char **name)
{
    const int e = g_last_cuda_error;
    g_last_cuda_error = 0;
    if (name) {
        if (e == 0) {
            *name = "none";
        } else if (e >= kDriverErrorBase) {
            *name = "a driver call failed: descriptor encoding or context query (CUresult = code - 100000)";
        } else {
            *name = cudaGetErrorName(static_cast<cudaError_t>(e));
        }
    }
    return e;
}

REGEN_API const char *regen_status_str(int status)
{
    switch (status) {
    case REGEN_OK: return "ok";
    case REGEN_ERR_INVALID_ARG: return "invalid argument";
    case REGEN_ERR_UNSUPPORTED: return "unsupported size or head dim";
    case REGEN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case REGEN_ERR_CUDA: return "CUDA error";
    case REGEN_ERR_TIMEOUT: return "kernel gave up on a bounded wait";
    default: return "unknown status";
    }
}

REGEN_API int regen_last_device_error(uint32_t *detail)
{
    if (detail) *detail = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return REGEN_ERR_CUDA;
    int code = 0;
    unsigned int site = 0;
    if (cudaMemcpyFromSymbol(&code, regen::g_regen_err, sizeof code) != cudaSuccess ||
        cudaMemcpyFromSymbol(&site, regen::g_regen_err_site, sizeof site) != cudaSuccess)
        return REGEN_ERR_CUDA;
    if (code != 0) {
        const int zero = 0;
        const unsigned int uzero = 0;
        if (cudaMemcpyToSymbol(regen::g_regen_err, &zero, sizeof zero) != cudaSuccess ||
            cudaMemcpyToSymbol(regen::g_regen_err_site, &uzero, sizeof uzero) != cudaSuccess)
            return REGEN_ERR_CUDA;
    }
    if (detail) *detail = site;
    return code == 0 ? REGEN_OK : code;
}

REGEN_API int regen_set_wait_limit_ns(uint64_t ns)
{
    g_wait_limit_ns.store(ns == 0 ? kDefaultWaitLimitNs : ns);
    return REGEN_OK;
}

REGEN_API int regen_version(void) { return 100; }

}  // extern "C"
