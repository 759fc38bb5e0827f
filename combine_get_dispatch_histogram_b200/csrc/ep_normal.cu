// ep_normal.cu -- receive rows of the normal (high-throughput) mode on sm_100a.
//
// Buffer.dispatch of the NeMo AutoModel page
// "nemo_automodel.components.moe.uccl_ep.buffer" sends a token ONCE to every
// rank it has a live expert on (is_token_in_rank), and Buffer.combine adds the
// returned rows without weights.  A rank's received tokens are ordered by
// (source rank, token): the row of token (r, t) on rank d is the number of
// tokens before it, in that order, that rank d receives.
//
// One CTA per (source rank r, destination rank d).  Its first row on rank d is
// the sum over r' < r of num_tokens_per_rank[r'][d]; it then walks rank r's
// tokens in tiles of 1024, one token per thread: a ballot gives each token's
// place among the warp's sent tokens, and every warp scans the 32 warp counts
// of the tile (shared memory) to find its base.  CTAs (0, d) also write
// recv_tokens[d], and CTA (0, 0) the per-expert receive counts rounded up to
// expert_alignment.
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

__global__ void __launch_bounds__(kNormalThreads) normal_layout_kernel(NormalLayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    __shared__ int32_t warp_cnt[kNormalThreads / 32];
    __shared__ int32_t first_row;
    const int r = blockIdx.x, d = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kNormalThreads / 32;
    if (warp == 0) {
        // lane q holds num_tokens_per_rank[q][d]: ranks before r give the first row
        const int32_t n = lane < a.R ? a.num_tokens_per_rank[lane * a.R + d] : 0;
        int32_t before = lane < r ? n : 0, all = n;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            before += __shfl_xor_sync(0xffffffffu, before, o);
            all += __shfl_xor_sync(0xffffffffu, all, o);
        }
        if (lane == 0) {
            first_row = before;
            if (r == 0) a.recv_tokens[d] = all;
        }
    }
    if (r == 0 && d == 0) {
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            const int32_t n = a.recv_count[e];
            a.num_recv_tokens_per_expert[e] = ((n + a.alignment - 1) / a.alignment) * a.alignment;
        }
    }
    __syncthreads();
    int32_t running = first_row;
    const uint8_t* itr = a.is_token_in_rank + int64_t(r) * a.T * a.R + d;
    int32_t* rows = a.token_recv_row + int64_t(r) * a.T * a.R + d;
    bool overflow = false;
    int64_t t = threadIdx.x;
    bool sent = t < a.T && itr[t * a.R] != 0;
    for (int64_t t0 = 0; t0 < a.T; t0 += kNormalThreads, t += kNormalThreads) {
        const int64_t tn = t + kNormalThreads;
        const bool sent_next = tn < a.T && itr[tn * a.R] != 0;  // one tile ahead
        const uint32_t bal = __ballot_sync(0xffffffffu, sent);
        if (lane == 0) warp_cnt[warp] = __popc(bal);
        __syncthreads();
        const int32_t c = lane < kWarps ? warp_cnt[lane] : 0;
        int32_t inc = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        const int32_t warp_base = __shfl_sync(0xffffffffu, inc - c, warp);
        const int32_t tile_total = __shfl_sync(0xffffffffu, inc, 31);
        const int32_t row = running + warp_base + __popc(bal & lanemask_lt());
        if (t < a.T) rows[t * a.R] = sent ? row : -1;
        overflow |= sent && row >= a.capacity;
        running += tile_total;
        sent = sent_next;
        __syncthreads();  // warp_cnt is rewritten by the next tile
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
    EP_NVTX_RANGE("ep_normal_layout");
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
    if (launch_pdl(normal_layout_kernel, dim3(d.num_ranks, d.num_ranks), dim3(kNormalThreads), 0,
                   static_cast<cudaStream_t>(stream),
                   a) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}
