// ep_stats.cu -- load statistics for EP load-balance monitoring.
//
// Buffer.low_latency_dispatch on the NeMo AutoModel page
// "nemo_automodel.components.moe.uccl_ep.buffer" can add each call's received
// token count per local expert into a cumulative int tensor
// (cumulative_local_expert_recv_stats, [num_local_experts]), for online EP load
// balance monitoring.  Here that is one small kernel over the receive counts the
// layout (ep_layout's recv_count, [E], or ep_peer_recv_count's, [E_local])
// produced: stats[i] += recv_count[i].
#include <algorithm>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

__global__ void __launch_bounds__(256) recv_stats_kernel(const int32_t* recv_count, int32_t* stats, int n) {
    pdl_wait();
    pdl_launch_dependents();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        stats[i] += recv_count[i];
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" int ep_recv_stats_accumulate(int32_t num, const int32_t* recv_count, int32_t* stats, void* stream) {
    EP_NVTX_RANGE("ep_recv_stats_accumulate");
    if (num < 0) return EP_ERR_INVALID;
    if (num == 0) return EP_OK;
    if (!recv_count || !stats) return EP_ERR_INVALID;
    const int blocks = int(std::min<int64_t>(64, ceil_div(num, 256)));
    if (launch_pdl(recv_stats_kernel, dim3(blocks), dim3(256), 0, static_cast<cudaStream_t>(stream), recv_count,
                   stats, int(num)) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}
