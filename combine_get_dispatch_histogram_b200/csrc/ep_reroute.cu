// ep_reroute.cu -- logical expert load, replica placement and routing
// expansion on sm_100a.
//
// Follows the GPU operations of the GitDiagram page "dots-infra/ultraep
// architecture": load computation from the post-gating routing, placement
// planning of replicas, then routing expansion of logical expert ids to
// physical (replica) ids before token dispatch.  The page names the steps but
// not the placement rule; the rule built here adds one replica at a time to
// the logical expert with the largest load/replicas (exact integer
// comparison, ties to the lowest id), and a (token, slot) pair of global
// token g = r*T + t on logical expert e goes to replica g mod n_rep[e] of e,
// i.e. physical id phys_base[e] + g mod n_rep[e].
//
// Two launches:
//   1. load   -- each CTA counts its slice of the routing into a shared
//                histogram with warp-aggregated shared-memory atomics (a
//                match mask from one warp ballot per id bit groups equal ids,
//                one leader adds the group size) and writes it to the
//                workspace;
//   2. expand -- every CTA sums the partial histograms, plans the replicas
//                (one warp: per step, a lane-parallel argmax of load/replicas
//                with shuffles) and rewrites its slice of the routing; CTA 0
//                also publishes load, num_replicas and phys_base.  The plan is
//                integer-exact, so every CTA derives the same one.
#include <algorithm>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr int kRerouteThreads = 512;
constexpr int kRerouteMaxLogical = EP_MAX_EXPERTS;

struct RerouteArgs {
    const int32_t* topk_logical;
    int32_t* partial;  // workspace [blocks][E_log]
    int32_t* load;
    int32_t* n_rep;
    int32_t* phys_base;
    int32_t* topk_phys;
    int32_t* status;
    int T, k, E_log, n_extra;
    int key_bits;  // ceil(log2(E_log))
    int64_t n_pairs;
    int64_t per_block;  // pairs per CTA slice
};

__global__ void __launch_bounds__(kRerouteThreads) reroute_load_kernel(RerouteArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t hist[];
    for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int64_t lo = int64_t(blockIdx.x) * a.per_block;
    const int64_t hi = min(a.n_pairs, lo + a.per_block);
    bool bad = false;
    for (int64_t p0 = lo; p0 < hi; p0 += blockDim.x) {
        const int64_t p = p0 + threadIdx.x;
        const int e = p < hi ? __ldg(a.topk_logical + p) : -1;
        const bool ok = e >= 0 && e < a.E_log;
        bad |= (e < -1 || e >= a.E_log);
        const uint32_t m = match_key(uint32_t(e), a.key_bits, __ballot_sync(0xffffffffu, ok));
        if (ok && (threadIdx.x & 31) == __ffs(m) - 1) atomicAdd(hist + e, __popc(m));
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);
    int32_t* out = a.partial + int64_t(blockIdx.x) * a.E_log;
    for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) out[e] = hist[e];
}

// load[a] / n[a] > load[b] / n[b], or equal with a < b.
__device__ __forceinline__ bool better(int32_t la, int32_t na, int ia, int32_t lb, int32_t nb, int ib) {
    const int64_t x = int64_t(la) * nb, y = int64_t(lb) * na;
    return x > y || (x == y && ia < ib);
}

__global__ void __launch_bounds__(kRerouteThreads) reroute_expand_kernel(RerouteArgs a, int n_partials) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    int32_t* load = sm;                  // [E_log]
    int32_t* n_rep = sm + a.E_log;       // [E_log]
    int32_t* base = sm + 2 * a.E_log;    // [E_log + 1]
    for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) {
        load[e] = 0;
        n_rep[e] = 1;
    }
    __syncthreads();
    const int64_t n_part = int64_t(n_partials) * a.E_log;
    for (int64_t i = threadIdx.x; i < n_part; i += blockDim.x) atomicAdd(load + i % a.E_log, a.partial[i]);
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        for (int step = 0; step < a.n_extra; ++step) {
            int bi = -1;
            int32_t bl = 0, bn = 1;
            for (int e = lane; e < a.E_log; e += 32) {
                const int32_t l = load[e], n = n_rep[e];
                if (bi < 0 || better(l, n, e, bl, bn, bi)) { bi = e; bl = l; bn = n; }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                const int32_t ol = __shfl_xor_sync(0xffffffffu, bl, off);
                const int32_t on = __shfl_xor_sync(0xffffffffu, bn, off);
                if (oi >= 0 && (bi < 0 || better(ol, on, oi, bl, bn, bi))) { bi = oi; bl = ol; bn = on; }
            }
            if (lane == 0) n_rep[bi] += 1;
            __syncwarp();
        }
        if (lane == 0) {
            int32_t run = 0;
            for (int e = 0; e < a.E_log; ++e) { base[e] = run; run += n_rep[e]; }
            base[a.E_log] = run;
        }
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) {
            a.load[e] = load[e];
            a.n_rep[e] = n_rep[e];
            a.phys_base[e] = base[e];
        }
        if (threadIdx.x == 0) a.phys_base[a.E_log] = base[a.E_log];
    }
    const int64_t lo = int64_t(blockIdx.x) * a.per_block;
    const int64_t hi = min(a.n_pairs, lo + a.per_block);
    for (int64_t p = lo + threadIdx.x; p < hi; p += blockDim.x) {
        const int e = __ldg(a.topk_logical + p);
        int32_t phys = -1;
        if (e >= 0 && e < a.E_log) {
            const int64_t token = p / a.k;  // = r*T + t, the global token index
            phys = base[e] + int32_t(token % n_rep[e]);
        }
        a.topk_phys[p] = phys;
    }
}

constexpr int kRerouteMaxBlocks = 256;

int reroute_blocks(int64_t n_pairs) {
    const int64_t by_size = ceil_div(n_pairs, int64_t(kRerouteThreads) * 4);
    return int(std::max<int64_t>(1, std::min<int64_t>(by_size, kRerouteMaxBlocks)));
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" size_t ep_reroute_workspace_bytes(int32_t num_ranks, int32_t num_tokens, int32_t num_topk,
                                             int32_t num_logical) {
    if (num_ranks <= 0 || num_tokens < 0 || num_topk <= 0 || num_logical <= 0) return 0;
    const int64_t n_pairs = int64_t(num_ranks) * num_tokens * num_topk;
    return round_up16(size_t(reroute_blocks(n_pairs)) * num_logical * 4);
}

extern "C" int ep_reroute(int32_t num_ranks, int32_t num_tokens, int32_t num_topk, int32_t num_logical,
                          int32_t num_extra, const int32_t* topk_idx_logical, void* workspace,
                          size_t workspace_bytes, int32_t* load, int32_t* num_replicas, int32_t* phys_base,
                          int32_t* topk_idx_phys, int32_t* status, ep_cfg_t cfg, void* stream) {
    (void)cfg;
    if (num_ranks <= 0 || num_tokens < 0 || num_topk <= 0 || num_logical <= 0 || num_extra < 0)
        return EP_ERR_INVALID;
    if (num_logical > kRerouteMaxLogical || num_topk > EP_MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if (int64_t(num_logical) + num_extra >= (int64_t(1) << 31)) return EP_ERR_UNSUPPORTED;
    const int64_t n_pairs = int64_t(num_ranks) * num_tokens * num_topk;
    if (n_pairs >= (int64_t(1) << 31)) return EP_ERR_UNSUPPORTED;
    if (!load || !num_replicas || !phys_base) return EP_ERR_INVALID;
    if (n_pairs > 0 && (!topk_idx_logical || !topk_idx_phys)) return EP_ERR_INVALID;
    const int blocks = reroute_blocks(n_pairs);
    const size_t need = round_up16(size_t(blocks) * num_logical * 4);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return EP_ERR_INVALID;

    RerouteArgs a;
    a.topk_logical = topk_idx_logical;
    a.partial = static_cast<int32_t*>(workspace);
    a.load = load;
    a.n_rep = num_replicas;
    a.phys_base = phys_base;
    a.topk_phys = topk_idx_phys;
    a.status = status;
    a.T = num_tokens;
    a.k = num_topk;
    a.E_log = num_logical;
    a.n_extra = num_extra;
    a.key_bits = 0;
    while ((1 << a.key_bits) < num_logical) ++a.key_bits;
    a.n_pairs = n_pairs;
    a.per_block = std::max<int64_t>(1, ceil_div(n_pairs, blocks));

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t smem1 = size_t(num_logical) * 4;
    const size_t smem2 = size_t(3 * num_logical + 1) * 4;
    if (smem2 > 48 * 1024) {
        if (cudaFuncSetAttribute(reroute_load_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem1)) !=
                cudaSuccess ||
            cudaFuncSetAttribute(reroute_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem2)) != cudaSuccess)
            return EP_ERR_CUDA;
    }
    if (launch_pdl(reroute_load_kernel, dim3(blocks), dim3(kRerouteThreads), smem1, s, a) != cudaSuccess ||
        launch_pdl(reroute_expand_kernel, dim3(blocks), dim3(kRerouteThreads), smem2, s, a, blocks) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}
