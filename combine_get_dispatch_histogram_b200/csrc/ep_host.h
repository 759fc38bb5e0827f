// ep_host.h -- host-side helpers of the C ABI: argument validation, device
// queries, launch-error mapping.  Internal to the library.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "ep.h"

namespace ep {

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
int sm_count();

// Largest dynamic shared memory a CTA may opt into on the current device.
int max_smem_optin();

// EP_ERR_CUDA if the last launch on this thread failed, EP_OK otherwise.
int launch_result();

}  // namespace ep
