// ep_host.h -- host-side helpers of the C ABI: argument validation, device
// queries, launch-error mapping.  Internal to the library.
#pragma once

#include <algorithm>
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "ep.h"

namespace ep {

// NVTX range named after the entry point, open for the duration of the host
// call (validation and launches), so a timeline tool shows which C-ABI call
// enqueued which kernels.  Without a tool attached a push/pop costs a few
// nanoseconds.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
#define EP_NVTX_RANGE(name) ::ep::NvtxRange ep_nvtx_range_(name)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline size_t round_up16(size_t x) { return (x + 15) & ~size_t(15); }

// Shape checks shared by layout / dispatch / combine.
inline int check_dims(const ep_dims_t& d) {
    if (d.num_ranks <= 0 || d.num_tokens < 0 || d.num_topk <= 0 || d.num_experts <= 0 || d.hidden <= 0)
        return EP_ERR_INVALID;
    if (d.num_experts % d.num_ranks != 0) return EP_ERR_INVALID;
    if (d.num_topk > d.num_experts) return EP_ERR_INVALID;
    if (d.hidden % 8 != 0) return EP_ERR_INVALID;
    if (d.num_ranks > EP_MAX_RANKS || d.num_topk > EP_MAX_TOPK || d.num_experts > EP_MAX_EXPERTS)
        return EP_ERR_UNSUPPORTED;
    const int64_t pairs = int64_t(d.num_ranks) * d.num_tokens * d.num_topk;
    if (pairs >= (int64_t(1) << 31)) return EP_ERR_UNSUPPORTED;
    return EP_OK;
}

// Launch with programmatic dependent launch: the kernel may be scheduled while
// the previous kernel in the stream is finishing, and must call pdl_wait()
// before reading anything produced upstream.  Overlaps launch latency and
// prologues across the back-to-back kernels of a layout -> dispatch -> combine
// step.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kernel, args...);
}

// Streaming-multiprocessor count of the current device (cached per device).
// Which thread-block cluster sizes of one kernel the device can hold at once:
// [device][CTAs], 0 = not asked yet, 1 = fits, -1 = does not (static storage,
// so it starts zeroed; a race only repeats the same query).
struct ClusterFitCache {
    std::atomic<int> v[64][17];
};

// The largest cluster of at most `want` CTAs (trying want, then 8, 4, 2) of
// `kernel` with `threads` threads and `smem` bytes of dynamic shared memory that
// the current device can hold at once, as the occupancy calculator answers;
// 1 if none.  Ask with the kernel's largest `smem` so that one answer holds for
// every shape; the kernel's dynamic shared-memory limit must already allow it.
template <typename... KArgs>
int fitting_cluster(void (*kernel)(KArgs...), int want, int threads, size_t smem, ClusterFitCache& cache) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
    int cl = std::min(16, std::max(1, want));
    for (; cl > 1; cl = cl > 8 ? 8 : cl / 2) {
        int known = cache.v[dev][cl].load(std::memory_order_relaxed);
        if (known == 0) {
            cudaLaunchConfig_t lc = {};
            lc.gridDim = dim3(cl);
            lc.blockDim = dim3(threads);
            lc.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = cl;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            lc.attrs = attr;
            lc.numAttrs = 1;
            int n = 0;
            const bool ok = cudaOccupancyMaxActiveClusters(&n, kernel, &lc) == cudaSuccess && n >= 1;
            if (!ok) cudaGetLastError();
            known = ok ? 1 : -1;
            cache.v[dev][cl].store(known, std::memory_order_relaxed);
        }
        if (known > 0) return cl;
    }
    return 1;
}

int sm_count();

// Largest dynamic shared memory a CTA may opt into on the current device.
int max_smem_optin();

// EP_ERR_CUDA if the last launch on this thread failed, EP_OK otherwise.
int launch_result();

}  // namespace ep
