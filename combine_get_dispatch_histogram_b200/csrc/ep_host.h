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

// Streaming-multiprocessor count of the current device (cached per device).
int sm_count();

// Largest dynamic shared memory a CTA may opt into on the current device.
int max_smem_optin();

// EP_ERR_CUDA if the last launch on this thread failed, EP_OK otherwise.
int launch_result();

}  // namespace ep
