// ep_convert.cu -- int64 routing ids to the library's int32 form.
//
// The NeMo AutoModel page "nemo_automodel.components.moe.uccl_ep.buffer"
// passes topk_idx as torch.int64 to Buffer.get_dispatch_layout and
// Buffer.dispatch; the ai-dynamo/nixl PR "nixl_ep: Optimize low-latency NVLink
// path" moved the index to 32 bits, which every kernel here reads.  This
// conversion saturates instead of truncating: an id above 2^31 - 1 becomes
// 2^31 - 1 and one below -2^31 becomes -2^31, both outside [-1, E) for every
// supported E, so the layout, dispatch, combine and reroute kernels drop the
// pair and raise EP_STATUS_BAD_EXPERT instead of routing a wrapped id to a
// real expert.  -1 (no selection) and every id in range keep their value.
#include <algorithm>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

__device__ __forceinline__ int32_t saturate_i32(long long v) {
    return v > 2147483647LL ? 2147483647 : (v < -2147483648LL ? int32_t(-2147483647 - 1) : int32_t(v));
}

// One id per thread per step: coalesced 8-byte loads and 4-byte stores.
__global__ void __launch_bounds__(256) topk_idx_to_i32_kernel(const long long* in, int32_t* out, int64_t n) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
        out[i] = saturate_i32(in[i]);
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" int ep_topk_idx_to_int32(const int64_t* topk_idx64, int32_t* topk_idx32, int64_t n, void* stream) {
    EP_NVTX_RANGE("ep_topk_idx_to_int32");
    if (n < 0) return EP_ERR_INVALID;
    if (n == 0) return EP_OK;
    if (!topk_idx64 || !topk_idx32) return EP_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(topk_idx64) & 7u) || (reinterpret_cast<uintptr_t>(topk_idx32) & 3u))
        return EP_ERR_INVALID;
    const int sms = sm_count();
    if (sms <= 0) return EP_ERR_CUDA;
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(int64_t(sms) * 4, ceil_div(n, 256)));
    if (launch_pdl(topk_idx_to_i32_kernel, dim3(unsigned(blocks)), dim3(256), 0, static_cast<cudaStream_t>(stream),
                   reinterpret_cast<const long long*>(topk_idx64), topk_idx32, n) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}
