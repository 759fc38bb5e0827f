// ep_layout.cu -- dispatch layout on sm_100a: per-expert / per-rank token
// histograms, prefix sums and the stable slab row of every (token, slot) pair.
//
// Defines Buffer.get_dispatch_layout (num_tokens_per_rank, is_token_in_rank,
// num_tokens_per_expert) of the NeMo AutoModel page
// "nemo_automodel.components.moe.uccl_ep.buffer", together with the handle
// that dispatch hands to combine.  The row of a live pair is its position
// among its expert's live pairs in (source rank, token, slot) order: a stable
// counting sort keyed by expert.
//
// Work decomposition.  The R*T*k pairs are cut into CHUNKS of 32 tokens of one
// source rank (chunk g = r * chunks_per_rank + c), and every chunk is owned by
// one warp in two passes:
//   1. count  -- the warp builds a private shared-memory histogram of its
//                chunk; lanes holding the same expert are merged with
//                __match_any_sync so one leader adds the group's popcount
//                (a warp-aggregated update; the histogram is warp-private so no
//                atomics are needed).  It also builds each token's destination
//                rank set (is_token_in_rank) and the chunk's per-rank token
//                counts.
//   2. scan   -- one lane per expert (32 experts per CTA, 32 warps splitting
//                each rank's chunks into segments) sums the chunk histograms of
//                each source rank (num_tokens_per_expert), scans them over ranks
//                (expert_rank_offset, recv_count) and turns every chunk count
//                into the chunk's first row (an exclusive scan over chunks in
//                (rank, chunk) order), in place in the workspace; one warp per
//                (source, destination) rank pair reduces the chunk token counts
//                (num_tokens_per_rank).
//   3. rank   -- the warp walks its chunk again in (token, slot) order, 32
//                pairs at a time; a pair's row is the chunk base of its expert
//                + the warp's running count + its rank among equal experts to
//                its left in the same 32 (popc of the match mask below it).
// Every step is deterministic: rows are unique and identical run to run.
#include <algorithm>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr int kChunkTokens = 32;
constexpr int kBatch = 8;  // 32-pair steps whose loads are issued together
constexpr int kActiveSlots = 64;  // shared-memory copy of the active mask (EP_MAX_RANKS)

struct LayoutArgs {
    const int32_t* topk_idx;
    const uint8_t* active;
    int32_t* chunk_hist;  // workspace [G][E]: counts, then first rows
    int32_t* chunk_tpr;   // workspace [G][R]: tokens of the chunk per destination rank
    int32_t* num_tokens_per_expert;
    int32_t* num_tokens_per_rank;
    uint8_t* is_token_in_rank;
    int32_t* recv_count;
    int32_t* expert_rank_offset;
    int32_t* pair_row;
    int32_t* status;
    int R, T, k, E, E_local;
    int chunks_per_rank, G;
    int64_t cap;
};

__device__ __forceinline__ bool pair_live(int e, int E, int E_local, bool src_ok, const int32_t* act) {
    return e >= 0 && e < E && src_ok && act[e / E_local] != 0;
}

__global__ void layout_count_kernel(LayoutArgs a) {
    extern __shared__ int32_t smem[];
    int32_t* act = smem;
    const int W = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) act[i] = a.active[i];
    __syncthreads();
    const int g = blockIdx.x * W + warp;
    if (g >= a.G) return;
    int32_t* h = smem + kActiveSlots + warp * a.E;
    for (int e = lane; e < a.E; e += 32) h[e] = 0;
    __syncwarp();

    const int r = g / a.chunks_per_rank;
    const int t0 = (g - r * a.chunks_per_rank) * kChunkTokens;
    const int nt = min(kChunkTokens, a.T - t0);
    const bool src_ok = act[r] != 0;
    const int32_t* base = a.topk_idx + (int64_t(r) * a.T + t0) * a.k;
    const int np = nt * a.k;

    bool bad = false;
    for (int p0 = 0; p0 < np; p0 += 32 * kBatch) {
        int ev[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int p = p0 + u * 32 + lane;
            ev[u] = p < np ? __ldg(base + p) : -1;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (p0 + u * 32 >= np) break;
            const int e = ev[u];
            bad |= (e < -1 || e >= a.E);
            const bool live = pair_live(e, a.E, a.E_local, src_ok, act);
            const uint32_t m = __match_any_sync(0xffffffffu, live ? e : -1);
            if (live && lane == __ffs(m) - 1) h[e] += __popc(m);
            __syncwarp();
        }
    }

    // destination-rank set of each token (lane <-> token)
    uint64_t ranks = 0;
    if (lane < nt) {
        const int32_t* tb = base + lane * a.k;
        for (int j = 0; j < a.k; ++j) {
            const int e = __ldg(tb + j);
            if (pair_live(e, a.E, a.E_local, src_ok, act)) ranks |= 1ull << (e / a.E_local);
        }
        uint8_t* itr = a.is_token_in_rank + (int64_t(r) * a.T + t0 + lane) * a.R;
        for (int d = 0; d < a.R; ++d) itr[d] = uint8_t((ranks >> d) & 1u);
    }
    int32_t* tpr = a.chunk_tpr + int64_t(g) * a.R;
    for (int d = 0; d < a.R; ++d) {
        const int n = __popc(__ballot_sync(0xffffffffu, (ranks >> d) & 1u));
        if (lane == 0) tpr[d] = n;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);

    int32_t* out = a.chunk_hist + int64_t(g) * a.E;
    for (int e = lane; e < a.E; e += 32) out[e] = h[e];
}

// One CTA per 32 experts (lane <-> expert).  Each rank's chunk range is cut
// into `segs` segments and every warp takes (rank, segment) items, so each
// lane walks only a few chunks; warp 0 then scans the segment totals in
// (rank, segment) order.  Separately, one warp per (source, destination) rank
// pair sums the per-chunk token counts.
__global__ void __launch_bounds__(1024) layout_scan_kernel(LayoutArgs a, int segs) {
    extern __shared__ int32_t smem[];
    const int NW = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int items = a.R * segs;
    int32_t* seg_sum = smem;                // [items][32]
    int32_t* seg_first = smem + items * 32;  // [items][32]
    const int e = blockIdx.x * 32 + lane;
    const bool ok = e < a.E;
    const int C = a.chunks_per_rank;
    const int seg_len = (C + segs - 1) / segs;

    // tokens per (source, destination) rank: warp-parallel sums over chunks
    const int RR = a.R * a.R;
    for (int pr = blockIdx.x * NW + warp; pr < RR; pr += gridDim.x * NW) {
        const int r = pr / a.R, d = pr - r * a.R;
        const int32_t* col = a.chunk_tpr + int64_t(r) * C * a.R + d;
        int32_t s = 0;
        for (int c = lane; c < C; c += 32) s += col[int64_t(c) * a.R];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) a.num_tokens_per_rank[pr] = s;
    }

    for (int it = warp; it < items; it += NW) {
        const int r = it / segs, sg = it - r * segs;
        const int c0 = sg * seg_len, c1 = min(C, c0 + seg_len);
        int32_t s = 0;
        if (ok) {
            const int32_t* col = a.chunk_hist + int64_t(r) * C * a.E + e;
#pragma unroll 8
            for (int c = c0; c < c1; ++c) s += col[int64_t(c) * a.E];
        }
        seg_sum[it * 32 + lane] = s;
    }
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int r = 0; r < a.R; ++r) {
            const int32_t rank_first = run;
            if (ok) a.expert_rank_offset[int64_t(e) * a.R + r] = rank_first;
            for (int sg = 0; sg < segs; ++sg) {
                seg_first[(r * segs + sg) * 32 + lane] = run;
                run += seg_sum[(r * segs + sg) * 32 + lane];
            }
            if (ok) a.num_tokens_per_expert[int64_t(r) * a.E + e] = run - rank_first;
        }
        if (ok) {
            a.recv_count[e] = run;
            if (run > a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
        }
    }
    __syncthreads();
    if (!ok) return;
    for (int it = warp; it < items; it += NW) {
        const int r = it / segs, sg = it - r * segs;
        const int c0 = sg * seg_len, c1 = min(C, c0 + seg_len);
        int32_t run = seg_first[it * 32 + lane];
        int32_t* col = a.chunk_hist + int64_t(r) * C * a.E + e;
        int c = c0;
        for (; c + 8 <= c1; c += 8) {
            int32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = col[int64_t(c + u) * a.E];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                col[int64_t(c + u) * a.E] = run;
                run += v[u];
            }
        }
        for (; c < c1; ++c) {
            const int32_t v = col[int64_t(c) * a.E];
            col[int64_t(c) * a.E] = run;
            run += v;
        }
    }
}

__global__ void layout_rank_kernel(LayoutArgs a) {
    extern __shared__ int32_t smem[];
    int32_t* act = smem;
    const int W = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) act[i] = a.active[i];
    __syncthreads();
    const int g = blockIdx.x * W + warp;
    if (g >= a.G) return;
    int32_t* next_row = smem + kActiveSlots + warp * a.E;
    const int32_t* first = a.chunk_hist + int64_t(g) * a.E;
    for (int e = lane; e < a.E; e += 32) next_row[e] = first[e];
    __syncwarp();

    const int r = g / a.chunks_per_rank;
    const int t0 = (g - r * a.chunks_per_rank) * kChunkTokens;
    const int nt = min(kChunkTokens, a.T - t0);
    const bool src_ok = act[r] != 0;
    const int64_t pbase = (int64_t(r) * a.T + t0) * a.k;
    const int32_t* base = a.topk_idx + pbase;
    int32_t* rows = a.pair_row + pbase;
    const int np = nt * a.k;
    const uint32_t below = lanemask_lt();

    for (int p0 = 0; p0 < np; p0 += 32 * kBatch) {
        int ev[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int p = p0 + u * 32 + lane;
            ev[u] = p < np ? __ldg(base + p) : -1;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int p = p0 + u * 32 + lane;
            if (p0 + u * 32 >= np) break;
            const int e = ev[u];
            const bool live = pair_live(e, a.E, a.E_local, src_ok, act);
            const uint32_t m = __match_any_sync(0xffffffffu, live ? e : -1);
            const int32_t b = live ? next_row[e] : 0;
            __syncwarp();
            if (live && lane == __ffs(m) - 1) next_row[e] = b + __popc(m);
            __syncwarp();
            if (p < np) rows[p] = live ? b + __popc(m & below) : -1;
        }
    }
}

// Warps per CTA of the count / rank kernels: each warp holds an E-entry histogram.
int chunk_warps(int E) {
    const int per_warp = E * 4;
    const int budget = 96 * 1024 - kActiveSlots * 4;
    return std::max(1, std::min(8, budget / per_warp));
}

size_t layout_ws_hist_bytes(const ep_dims_t& d) {
    const int64_t G = int64_t(d.num_ranks) * ceil_div(d.num_tokens, kChunkTokens);
    return round_up16(size_t(G) * d.num_experts * 4);
}

size_t layout_ws_tpr_bytes(const ep_dims_t& d) {
    const int64_t G = int64_t(d.num_ranks) * ceil_div(d.num_tokens, kChunkTokens);
    return round_up16(size_t(G) * d.num_ranks * 4);
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" size_t ep_layout_workspace_bytes(ep_dims_t d) {
    if (check_dims(d) != EP_OK) return 0;
    return layout_ws_hist_bytes(d) + layout_ws_tpr_bytes(d);
}

extern "C" int ep_layout(ep_dims_t d, const int32_t* topk_idx, const uint8_t* active, void* workspace,
                         size_t workspace_bytes, int32_t* num_tokens_per_expert,
                         int32_t* num_tokens_per_rank, uint8_t* is_token_in_rank, int32_t* recv_count,
                         int32_t* expert_rank_offset, int32_t* pair_row, int32_t* status, ep_cfg_t cfg,
                         void* stream) {
    (void)cfg;
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (!active || !num_tokens_per_expert || !num_tokens_per_rank || !recv_count || !expert_rank_offset)
        return EP_ERR_INVALID;
    if (RT > 0 && (!topk_idx || !is_token_in_rank || !pair_row)) return EP_ERR_INVALID;
    const size_t need = ep_layout_workspace_bytes(d);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return EP_ERR_INVALID;

    LayoutArgs a;
    a.topk_idx = topk_idx;
    a.active = active;
    a.chunk_hist = static_cast<int32_t*>(workspace);
    a.chunk_tpr = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + layout_ws_hist_bytes(d));
    a.num_tokens_per_expert = num_tokens_per_expert;
    a.num_tokens_per_rank = num_tokens_per_rank;
    a.is_token_in_rank = is_token_in_rank;
    a.recv_count = recv_count;
    a.expert_rank_offset = expert_rank_offset;
    a.pair_row = pair_row;
    a.status = status;
    a.R = d.num_ranks;
    a.T = d.num_tokens;
    a.k = d.num_topk;
    a.E = d.num_experts;
    a.E_local = d.num_experts / d.num_ranks;
    a.chunks_per_rank = int(ceil_div(d.num_tokens, kChunkTokens));
    a.G = d.num_ranks * a.chunks_per_rank;
    a.cap = RT;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int W = chunk_warps(d.num_experts);
    const size_t chunk_smem = size_t(kActiveSlots) * 4 + size_t(W) * d.num_experts * 4;
    if (chunk_smem > 48 * 1024) {
        if (cudaFuncSetAttribute(layout_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(chunk_smem)) != cudaSuccess ||
            cudaFuncSetAttribute(layout_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(chunk_smem)) != cudaSuccess)
            return EP_ERR_CUDA;
    }
    const int chunk_blocks = int(ceil_div(a.G, W));
    if (a.G > 0) layout_count_kernel<<<chunk_blocks, 32 * W, chunk_smem, s>>>(a);
    // scan: 32 warps per CTA; segments so that ranks x segments covers the warps
    const int scan_warps = 32;
    const int segs = std::max(1, std::min(a.chunks_per_rank, scan_warps / std::max(1, std::min(d.num_ranks, scan_warps))));
    const size_t scan_smem = size_t(2) * d.num_ranks * segs * 32 * 4;
    layout_scan_kernel<<<int(ceil_div(d.num_experts, 32)), 32 * scan_warps, scan_smem, s>>>(a, segs);
    if (a.G > 0) layout_rank_kernel<<<chunk_blocks, 32 * W, chunk_smem, s>>>(a);
    return launch_result();
}
