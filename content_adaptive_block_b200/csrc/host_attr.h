// Host-side helpers shared by both translation units of libgsa (no device
// code, so either may include it): per-device kernel attributes and the NVTX
// range every exported call opens.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <map>
#include <mutex>
#include <utility>

namespace gsa {

// Function attributes belong to one device's context, so a kernel is opted in
// to `bytes` of dynamic shared memory once per (kernel, device): on the
// device current at the call.  False when the device cannot be read or the
// runtime refuses the size (the caller then reports a CUDA error and
// launches nothing); a refused size is asked for again on the next call.
inline bool smem_opt_in_fn(const void* fn, int bytes) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, int> granted;
    std::lock_guard<std::mutex> lock(mu);
    int& have = granted[{fn, dev}];
    if (have >= bytes) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    have = bytes;
    return true;
}
template <typename F>
inline bool smem_opt_in(F* kernel, int bytes) {
    return smem_opt_in_fn(reinterpret_cast<const void*>(kernel), bytes);
}

// An NVTX range named after the C-ABI call, open for the call's host-side
// work (checks, descriptor set-up, launches), so a timeline tool shows each
// call around the kernels it launched.  Costs a few nanoseconds when no tool
// is attached (NVTX3 is header-only and loads a tool only when one is named).
struct CallRange {
    explicit CallRange(const char* name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange&) = delete;
    CallRange& operator=(const CallRange&) = delete;
};

}  // namespace gsa
