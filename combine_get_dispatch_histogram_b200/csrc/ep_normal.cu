// ep_normal.cu -- receive rows of the normal (high-throughput) mode on sm_100a.
//
// Buffer.dispatch of the NeMo AutoModel page
// "nemo_automodel.components.moe.uccl_ep.buffer" sends a token ONCE to every
// rank it has a live expert on (is_token_in_rank), and Buffer.combine adds the
// returned rows without weights.  A rank's received tokens are ordered by
// (source rank, token): the row of token (r, t) on rank d is the number of
// tokens before it, in that order, that rank d receives.
//
// One CTA per source rank r.  Its first row on rank d is the sum over r' < r
// of num_tokens_per_rank[r'][d]; within the rank, each thread owns a run of
// consecutive tokens, and a block-wide exclusive scan of the runs' counts
// (warp shuffles, then the warp totals) gives each run its first row, for one
// destination rank after another.  CTA 0 also writes recv_tokens and the
// per-expert receive counts rounded up to expert_alignment.
#include <algorithm>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr int kNormalThreads = 1024;

struct NormalLayoutArgs {
    const uint8_t* is_token_in_rank;
    const int32_t* num_tokens_per_rank;
    const int32_t* recv_count;
    int32_t* token_recv_row;
    int32_t* recv_tokens;
    int32_t* num_recv_tokens_per_expert;
    int32_t* status;
    int R, T, E, alignment;
    int64_t capacity;
};

// Exclusive prefix of v over the CTA's threads (in thread order); all threads must call.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_sums) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int32_t w = lane < nw ? warp_sums[lane] : 0;
        int32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        if (lane < nw) warp_sums[lane] = wi - w;
    }
    __syncthreads();
    const int32_t base = warp_sums[warp] + inc - v;
    __syncthreads();
    return base;
}

__global__ void __launch_bounds__(kNormalThreads) normal_layout_kernel(NormalLayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    __shared__ int32_t first_row[EP_MAX_RANKS];
    __shared__ int32_t warp_sums[32];
    const int r = blockIdx.x;
    for (int d = threadIdx.x; d < a.R; d += blockDim.x) {
        int32_t s = 0;
        for (int q = 0; q < r; ++q) s += a.num_tokens_per_rank[q * a.R + d];
        first_row[d] = s;
        if (r == 0) {
            int32_t tot = 0;
            for (int q = 0; q < a.R; ++q) tot += a.num_tokens_per_rank[q * a.R + d];
            a.recv_tokens[d] = tot;
        }
    }
    if (r == 0) {
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            const int32_t n = a.recv_count[e];
            a.num_recv_tokens_per_expert[e] = ((n + a.alignment - 1) / a.alignment) * a.alignment;
        }
    }
    __syncthreads();
    const int per = (a.T + blockDim.x - 1) / blockDim.x;
    const int t0 = min(a.T, int(threadIdx.x) * per), t1 = min(a.T, t0 + per);
    const uint8_t* itr = a.is_token_in_rank + int64_t(r) * a.T * a.R;
    int32_t* rows = a.token_recv_row + int64_t(r) * a.T * a.R;
    bool overflow = false;
    for (int d = 0; d < a.R; ++d) {
        int32_t c = 0;
        for (int t = t0; t < t1; ++t) c += itr[int64_t(t) * a.R + d] != 0;
        int32_t row = first_row[d] + block_exclusive_scan(c, warp_sums);
        for (int t = t0; t < t1; ++t) {
            const bool sent = itr[int64_t(t) * a.R + d] != 0;
            rows[int64_t(t) * a.R + d] = sent ? row : -1;
            if (sent) {
                overflow |= row >= a.capacity;
                ++row;
            }
        }
    }
    if (__syncthreads_or(overflow) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_OVERFLOW);
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" int ep_normal_layout(ep_dims_t d, int32_t recv_capacity, int32_t expert_alignment,
                                const uint8_t* is_token_in_rank, const int32_t* num_tokens_per_rank,
                                const int32_t* recv_count, int32_t* token_recv_row, int32_t* recv_tokens,
                                int32_t* num_recv_tokens_per_expert, int32_t* status, ep_cfg_t cfg, void* stream) {
    (void)cfg;
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    if (recv_capacity < 0 || expert_alignment < 1) return EP_ERR_INVALID;
    if (d.num_ranks > EP_MAX_NORMAL_RANKS) return EP_ERR_UNSUPPORTED;
    if (!num_tokens_per_rank || !recv_count || !recv_tokens || !num_recv_tokens_per_expert) return EP_ERR_INVALID;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (RT > 0 && (!is_token_in_rank || !token_recv_row)) return EP_ERR_INVALID;
    NormalLayoutArgs a;
    a.is_token_in_rank = is_token_in_rank;
    a.num_tokens_per_rank = num_tokens_per_rank;
    a.recv_count = recv_count;
    a.token_recv_row = token_recv_row;
    a.recv_tokens = recv_tokens;
    a.num_recv_tokens_per_expert = num_recv_tokens_per_expert;
    a.status = status;
    a.R = d.num_ranks;
    a.T = d.num_tokens;
    a.E = d.num_experts;
    a.alignment = expert_alignment;
    a.capacity = recv_capacity;
    if (launch_pdl(normal_layout_kernel, dim3(d.num_ranks), dim3(kNormalThreads), 0, static_cast<cudaStream_t>(stream),
                   a) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}
