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
// Two paths (ep_cfg_t.variant), the same result:
//   EP_REROUTE_CLUSTER (AUTO): one launch of a thread-block cluster; each CTA
//     counts its slice, reads every CTA's counts from the cluster's shared
//     memories, plans the replicas and rewrites its slice (reroute_cluster_kernel);
//   EP_REROUTE_TWO_LAUNCH:
//     1. load   -- each CTA counts its slice of the routing into a shared
//                  histogram with warp-aggregated shared-memory atomics (a
//                  match mask from one warp ballot per id bit groups equal ids,
//                  one leader adds the group size) and writes it to the
//                  workspace;
//     2. expand -- every CTA sums the partial histograms, plans the replicas
//                  (one warp: per step, a lane-parallel argmax of load/replicas
//                  with shuffles) and rewrites its slice of the routing; CTA 0
//                  also publishes load, num_replicas and phys_base.
// The plan is integer-exact, so every CTA derives the same one.
#include <algorithm>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr int kRerouteThreads = 512;
constexpr int kRerouteMaxLogical = EP_MAX_EXPERTS;
constexpr int kRerouteClusterThreads = 1024;
constexpr int kRerouteClusterMaxCtas = 16;
constexpr int64_t kRerouteClusterPairsPerCta = 1024;

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

// load[a] / n[a] > load[b] / n[b], or equal with a < b.
__device__ __forceinline__ bool better(int32_t la, int32_t na, int ia, int32_t lb, int32_t nb, int ib) {
    const int64_t x = int64_t(la) * nb, y = int64_t(lb) * na;
    return x > y || (x == y && ia < ib);
}

constexpr int kRerouteBatch = 8;  // loads a thread issues before using them

// Warp 0 of a CTA: n_extra times, one more replica for the expert with the largest
// load / replicas (exact integer compare, ties to the lowest id); then base = the
// exclusive prefix of the replica counts (base[E_log] = the physical expert count).
// Lane l keeps the best of its experts l, l + 32, ...; only the lane owning the
// last pick re-evaluates.  Per step, a warp max of float ratios bounds the answer:
// a float ratio is within 6 * 2^-24 of the exact one (two int->float roundings and
// a rounded division), so every lane holding the exact maximum has a ratio of at
// least (1 - 2^-20) times the float maximum; those few lanes are compared exactly.
__device__ void plan_replicas(const RerouteArgs& a, const int32_t* load, int32_t* n_rep, int32_t* base) {
    const int lane = threadIdx.x & 31;
    int bi = -1;
    int32_t bl = 0, bn = 1;
    auto local_best = [&]() {
        bi = -1;
        for (int e = lane; e < a.E_log; e += 32) {
            const int32_t l = load[e], n = n_rep[e];
            if (bi < 0 || better(l, n, e, bl, bn, bi)) { bi = e; bl = l; bn = n; }
        }
    };
    local_best();
    for (int step = 0; step < a.n_extra; ++step) {
        const float ratio = bi >= 0 ? float(bl) / float(bn) : 0.f;
        const float top = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(ratio)));  // ratios >= 0
        uint32_t cand = __ballot_sync(0xffffffffu, bi >= 0 && ratio >= top * (1.0f - 0x1p-20f));
        int wi = -1;
        int32_t wl = 0, wn = 1;
        while (cand) {  // the same on every lane
            const int c = __ffs(cand) - 1;
            cand &= cand - 1;
            const int ci = __shfl_sync(0xffffffffu, bi, c);
            const int32_t cl = __shfl_sync(0xffffffffu, bl, c), cn = __shfl_sync(0xffffffffu, bn, c);
            if (wi < 0 || better(cl, cn, ci, wl, wn, wi)) { wi = ci; wl = cl; wn = cn; }
        }
        if (wi < 0) break;  // cannot happen (the lane with the float maximum is a candidate); uniform
        if (lane == (wi & 31)) {
            n_rep[wi] += 1;
            local_best();
        }
        __syncwarp();
    }
    // exclusive prefix of n_rep, 32 experts per step (lane-parallel scan, carried across steps)
    int32_t carry = 0;
    for (int e0 = 0; e0 < a.E_log; e0 += 32) {
        const int e = e0 + lane;
        const int32_t v = e < a.E_log ? n_rep[e] : 0;
        int32_t inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
        }
        if (e < a.E_log) base[e] = carry + inc - v;
        carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) base[a.E_log] = carry;
}

// Count the routing pairs [lo, hi) into the shared histogram (warp-aggregated:
// a ballot match groups equal ids, one leader adds the group size); true if an
// id outside [-1, E_log) was seen by this thread.  Each thread issues
// kRerouteBatch loads before using them.
__device__ bool count_slice(const RerouteArgs& a, int64_t lo, int64_t hi, int32_t* hist) {
    bool bad = false;
    const int64_t stride = int64_t(blockDim.x) * kRerouteBatch;
    for (int64_t p0 = lo; p0 < hi; p0 += stride) {
        int ev[kRerouteBatch];
#pragma unroll
        for (int u = 0; u < kRerouteBatch; ++u) {
            const int64_t p = p0 + int64_t(u) * blockDim.x + threadIdx.x;
            ev[u] = p < hi ? __ldg(a.topk_logical + p) : -1;
        }
#pragma unroll
        for (int u = 0; u < kRerouteBatch; ++u) {
            if (p0 + int64_t(u) * blockDim.x + (threadIdx.x & ~31u) >= hi) break;  // the same for the warp
            const int e = ev[u];
            const bool ok = e >= 0 && e < a.E_log;
            bad |= (e < -1 || e >= a.E_log);
            const uint32_t m = match_key(uint32_t(e), a.key_bits, __ballot_sync(0xffffffffu, ok));
            if (ok && (threadIdx.x & 31) == __ffs(m) - 1) atomicAdd(hist + e, __popc(m));
        }
    }
    return bad;
}

// Physical ids of the routing pairs [lo, hi).  Pair indices are below 2^31 (the
// host checks), so the token index and its replica are taken in unsigned 32-bit
// arithmetic (the indices below stay below 2^32).  Loads are batched as above.
__device__ void expand_slice(const RerouteArgs& a, int64_t lo, int64_t hi, const int32_t* n_rep,
                             const int32_t* base) {
    const uint32_t end = uint32_t(hi), k = uint32_t(a.k);
    const uint32_t stride = blockDim.x * kRerouteBatch;
    for (uint32_t p0 = uint32_t(lo); p0 < end; p0 += stride) {
        int ev[kRerouteBatch];
#pragma unroll
        for (int u = 0; u < kRerouteBatch; ++u) {
            const uint32_t p = p0 + u * blockDim.x + threadIdx.x;
            ev[u] = p < end ? __ldg(a.topk_logical + p) : -1;
        }
#pragma unroll
        for (int u = 0; u < kRerouteBatch; ++u) {
            const uint32_t p = p0 + u * blockDim.x + threadIdx.x;
            if (p >= end) continue;
            const int e = ev[u];
            int32_t phys = -1;
            if (e >= 0 && e < a.E_log) {
                const uint32_t token = p / k;  // = r*T + t, the global token index
                phys = base[e] + int32_t(token % uint32_t(n_rep[e]));
            }
            a.topk_phys[p] = phys;
        }
    }
}

__global__ void __launch_bounds__(kRerouteThreads) reroute_load_kernel(RerouteArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t hist[];
    for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int64_t lo = int64_t(blockIdx.x) * a.per_block;
    const int64_t hi = min(a.n_pairs, lo + a.per_block);
    const bool bad = count_slice(a, lo, hi, hist);
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);
    int32_t* out = a.partial + int64_t(blockIdx.x) * a.E_log;
    for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) out[e] = hist[e];
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
    if (threadIdx.x < 32) plan_replicas(a, load, n_rep, base);
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
    expand_slice(a, lo, min(a.n_pairs, lo + a.per_block), n_rep, base);
}

// One launch (EP_REROUTE_CLUSTER, the default): a thread-block cluster of CL CTAs.
// CTA c counts slice c of the routing into its shared histogram; after a cluster
// barrier every CTA adds up the CL histograms straight from the cluster's shared
// memories (the global load); after a second one (no shared memory is read across
// CTAs past it) each CTA plans the replicas itself -- the plan is integer-exact,
// so all agree -- and rewrites its slice; CTA 0 publishes load, num_replicas and
// phys_base.  No workspace and no second launch.
__global__ void __launch_bounds__(kRerouteClusterThreads) reroute_cluster_kernel(RerouteArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    int32_t* hist = sm;                  // [E_log] this CTA's counts
    int32_t* load = sm + a.E_log;        // [E_log]
    int32_t* n_rep = load + a.E_log;     // [E_log]
    int32_t* base = n_rep + a.E_log;     // [E_log + 1]
    const uint32_t cta = cluster_ctarank(), CL = cluster_nctarank();
    for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int64_t lo = int64_t(cta) * a.per_block;
    const int64_t hi = min(a.n_pairs, lo + a.per_block);
    const bool bad = count_slice(a, lo, hi, hist);
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);
    cluster_sync();  // every CTA's histogram is final
    for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) {
        int32_t n = 0;
        for (uint32_t c = 0; c < CL; ++c) n += ld_dsmem_s32(dsmem_addr(hist + e, c));
        load[e] = n;
        n_rep[e] = 1;
    }
    cluster_sync();  // no shared memory is read across CTAs after this
    if (threadIdx.x < 32) plan_replicas(a, load, n_rep, base);
    __syncthreads();
    if (cta == 0) {
        for (int e = threadIdx.x; e < a.E_log; e += blockDim.x) {
            a.load[e] = load[e];
            a.n_rep[e] = n_rep[e];
            a.phys_base[e] = base[e];
        }
        if (threadIdx.x == 0) a.phys_base[a.E_log] = base[a.E_log];
    }
    expand_slice(a, lo, hi, n_rep, base);
}

constexpr int kRerouteMaxBlocks = 256;

ClusterFitCache g_reroute_cluster_fit;

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
    EP_NVTX_RANGE("ep_reroute");
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
    const int variant = cfg.variant == EP_VARIANT_AUTO ? int(EP_REROUTE_CLUSTER) : cfg.variant;
    if (variant != EP_REROUTE_CLUSTER && variant != EP_REROUTE_TWO_LAUNCH) return EP_ERR_INVALID;
    if (variant == EP_REROUTE_CLUSTER) {
        const size_t smem = size_t(4 * num_logical + 1) * 4;
        const size_t smem_max = size_t(4 * kRerouteMaxLogical + 1) * 4;  // the path's largest need
        if (cudaFuncSetAttribute(reroute_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem_max)) != cudaSuccess ||
            cudaFuncSetAttribute(reroute_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess)
            return EP_ERR_CUDA;
        // one CTA per kRerouteClusterPairsPerCta pairs, up to kRerouteClusterMaxCtas, as many as fit
        const int want = int(std::min<int64_t>(kRerouteClusterMaxCtas,
                                               std::max<int64_t>(1, ceil_div(n_pairs, kRerouteClusterPairsPerCta))));
        const int cl = fitting_cluster(reroute_cluster_kernel, want, kRerouteClusterThreads, smem_max,
                                       g_reroute_cluster_fit);
        a.per_block = std::max<int64_t>(1, ceil_div(n_pairs, cl));
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(cl);
        lc.blockDim = dim3(kRerouteClusterThreads);
        lc.dynamicSmemBytes = smem;
        lc.stream = s;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cl;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = attr;
        lc.numAttrs = 2;
        if (cudaLaunchKernelEx(&lc, reroute_cluster_kernel, a) != cudaSuccess) return EP_ERR_CUDA;
        return launch_result();
    }
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
