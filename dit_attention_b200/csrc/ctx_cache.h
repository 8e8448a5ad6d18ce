// ctx_cache.h -- one-time set-up results cached per CUDA context (host C++).
//
// A kernel's dynamic shared-memory limit (cudaFuncSetAttribute) and the
// device address of a __device__ array belong to the module as loaded in one
// CUDA context, not to the process: a process that drives a second GPU, or a
// host application that creates contexts of its own, has to redo that set-up
// in each. The cache is keyed by the driver's context ID (cuCtxGetId), which
// a process never reuses, unlike a context pointer after the context is
// destroyed. Only results that a retry cannot change are kept: when the
// set-up reports `kRetryStatus` (a failing CUDA call), it runs again on the
// next call. Kept free of CUDA headers so that host tests can build it alone.
#pragma once

#include <mutex>
#include <utility>

namespace regen {

template <typename T, int kRetryStatus>
class CtxCache {
public:
    // The value set up for context `id`: runs `setup(T *out) -> status` the
    // first time `id` is seen (and again while it returns kRetryStatus).
    // Returns the set-up's status; *value (if not null) receives the value.
    template <typename F>
    int get(unsigned long long id, F &&setup, T *value)
    {
        std::lock_guard<std::mutex> lock(mu_);
        for (int i = 0; i < n_; ++i)
            if (ids_[i] == id) {
                if (value) *value = values_[i];
                return status_[i];
            }
        T v{};
        const int st = setup(&v);
        if (st != kRetryStatus && n_ < kSlots) {   // past kSlots contexts, set-up reruns per call
            ids_[n_] = id;
            status_[n_] = st;
            values_[n_] = v;
            ++n_;
        }
        if (value) *value = v;
        return st;
    }

private:
    static constexpr int kSlots = 256;
    std::mutex mu_;
    unsigned long long ids_[kSlots] = {};
    int status_[kSlots] = {};
    T values_[kSlots] = {};
    int n_ = 0;
};

}  // namespace regen
