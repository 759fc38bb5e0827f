// ep_peer.cu -- expert-parallel dispatch / combine between processes that each
// own one GPU (a real EP world), over peer memory (NVLink / NVSwitch).
//
// The pages' low-latency kernels (the NeMo AutoModel page
// "nemo_automodel.components.moe.uccl_ep.buffer", Buffer.low_latency_dispatch /
// Buffer.low_latency_combine, intranode NVLink; the ai-dynamo/nixl PR "nixl_ep:
// Optimize low-latency NVLink path") move token rows with stores straight into
// the destination rank's receive buffer and tell the receiver with a flag.
// This file is that transport for B200 processes:
//
//   rank r:  ep_layout_local          counts and rows of r's own routing
//            (all-gather of the [E] counts by the caller, e.g. NCCL)
//            ep_dispatch_peer         rows -> every destination's slab, then one
//                                     release flag per destination
//   rank d:  ep_wait_peers            bounded acquire-wait for every active
//                                     source's flag; ep_peer_recv_count
//            (experts run on the slab)
//            ep_signal_peers          "outputs ready" flag into every rank
//   rank r:  ep_wait_peers            bounded wait for every destination
//            ep_combine_peer          weighted gather of the expert outputs from
//                                     the peers' slabs back into r's tokens
//
// Addresses of the peers' buffers come from a table of R device addresses per
// buffer kind (slab, src_info, flag words), mapped by the caller (CUDA IPC:
// ep_ipc_export / ep_ipc_import, or one process's own allocations when the
// ranks are emulated on one GPU).  Every peer access is a plain 16-byte load or
// store or an 8-byte release/acquire flag access: no bulk or tensor copy and no
// multicast touches peer memory.  The compact receive layout is the one the
// single-GPU path uses: the row of source r's pair inside expert e is
// (rows of e from sources before r) + (the pair's row among r's own pairs of e),
// the first term summed from the all-gathered count matrix inside the kernels.
#include <algorithm>
#include <cstdint>
#include <cstring>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr int kPeerThreads = 256;
constexpr int kPeerSlotGroup = 8;  // slots whose rows a lane loads before it accumulates them

__device__ __forceinline__ void st_release_sys_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_acquire_sys_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// 16-byte load of a row read once; plain (coherent) load, so it may target peer memory.
__device__ __forceinline__ uint4 ld_peer_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

struct PeerArgs {
    const uint8_t* x;          // dispatch: this rank's tokens [T, H]
    const int32_t* topk_idx;   // [T, k]
    const float* w;            // combine: [T, k]
    const int32_t* local_row;  // [T, k] from ep_layout_local
    const int32_t* counts;     // [R, E] every rank's live pairs per expert
    const uint8_t* active;     // [R]
    const uint64_t* slab;      // [R] address of rank d's slab [E_local, CAP, H]
    const uint64_t* src_info;  // [R] address of rank d's src_info [E_local, CAP, 2] (dispatch)
    const uint64_t* flags;     // [R] address of rank d's flag words [R] (dispatch)
    uint32_t* done;            // dispatch: this rank's CTA-completion counter
    uint8_t* out;              // combine: [T, H]
    int32_t* status;
    int R, T, k, E, E_local, rank;
    int64_t cap, row_bytes;
    uint64_t signal;
};

// off[e] = rows of expert e that come from sources before `rank` (exclusive
// prefix over the ranks of the count matrix).
__device__ __forceinline__ void source_offsets(const PeerArgs& a, int32_t* off) {
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int32_t s = 0;
        for (int r = 0; r < a.rank; ++r) s += __ldg(a.counts + int64_t(r) * a.E + e);
        off[e] = s;
    }
}

// Slot `lane` of token t: destination address of its row (0 if the slot is not
// sent), the destination rank and local row; flags malformed slots once.
struct PeerSlot {
    uint64_t addr;
    int d, le, row;
    float w;
};

__device__ __forceinline__ PeerSlot peer_slot(const PeerArgs& a, const int32_t* act, const int32_t* off,
                                              int64_t t, int lane, bool src_ok, bool flag) {
    PeerSlot s{0ull, -1, -1, -1, 0.f};
    if (lane >= a.k) return s;
    const int64_t p = t * a.k + lane;
    const int e = __ldg(a.topk_idx + p);
    const int lr = __ldg(a.local_row + p);
    if (a.w) s.w = __ldg(a.w + p);
    const bool in_range = e >= 0 && e < a.E;
    if (lr < 0) return s;
    if (!in_range) {
        if (flag) flag_status(a.status, EP_STATUS_BAD_EXPERT);
        return s;
    }
    const int d = e / a.E_local;
    const int64_t row = int64_t(off[e]) + lr;
    if (row >= a.cap) {
        if (flag) flag_status(a.status, EP_STATUS_OVERFLOW);
        return s;
    }
    if (!src_ok || act[d] == 0) return s;
    s.d = d;
    s.le = e - d * a.E_local;
    s.row = int(row);
    s.addr = __ldg(a.slab + d) + uint64_t((int64_t(s.le) * a.cap + row) * a.row_bytes);
    return s;
}

// ---------------------------------------------------------------------------- dispatch

// Warps take units (token, piece of 32*U 16-byte columns) strided over the grid.
// A lane loads its columns of the token row once and stores them to
// every destination row; the row's (src_rank, src_token) goes to the
// destination's src_info.  After the CTA's last store one thread fences at
// system scope and counts the CTA done; the CTA that finishes last releases
// signal into every active destination's flag word for this source.
template <int U>
__global__ void __launch_bounds__(kPeerThreads) dispatch_peer_kernel(PeerArgs a) {
    extern __shared__ int32_t off[];  // [E]
    __shared__ int32_t act[EP_MAX_RANKS];
    __shared__ int last;
    pdl_wait();  // nothing upstream is read before this
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) act[i] = a.active[i];
    source_offsets(a, off);
    __syncthreads();
    const bool src_ok = act[a.rank] != 0;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int nvec = int(a.row_bytes >> 4);
    const int piece_vec = 32 * U;
    const int np = (nvec + piece_vec - 1) / piece_vec;
    const int64_t n_units = int64_t(a.T) * np;
    // units strided over the warps, so the grid works on one window of consecutive tokens at a time
    // (the rows it writes to a busy expert are neighbours in its slab)
    const int64_t my_n = gw < n_units ? (n_units - 1 - gw) / warps + 1 : 0;

    int64_t cur_tok = -1;
    uint32_t mask = 0;
    uint64_t my_addr = 0;
    for (int64_t i = 0; i < my_n; ++i) {
        const int64_t u = gw + i * warps;
        const int64_t t = u / np;
        const int pc = int(u - t * np);
        if (t != cur_tok) {
            cur_tok = t;
            const PeerSlot s = peer_slot(a, act, off, t, lane, src_ok, pc == 0);
            my_addr = s.addr;
            mask = __ballot_sync(0xffffffffu, s.addr != 0ull);
            if (pc == 0 && s.addr != 0ull) {
                int2* si = reinterpret_cast<int2*>(__ldg(a.src_info + s.d));
                si[int64_t(s.le) * a.cap + s.row] = make_int2(a.rank, int(t));
            }
        }
        if (mask == 0u) continue;
        const int v0 = pc * piece_vec + lane;
        const uint8_t* src = a.x + t * a.row_bytes;
        uint4 xv[U];
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int v = v0 + 32 * uu;
            if (v < nvec) xv[uu] = ld_stream_v4(src + int64_t(v) * 16);
        }
        for (uint32_t m = mask; m; m &= m - 1u) {
            const int j = __ffs(m) - 1;
            uint8_t* dst = reinterpret_cast<uint8_t*>(__shfl_sync(0xffffffffu, my_addr, j));
#pragma unroll
            for (int uu = 0; uu < U; ++uu) {
                const int v = v0 + 32 * uu;
                if (v < nvec) st_global_v4(dst + int64_t(v) * 16, xv[uu]);
            }
        }
    }
    // every row store of the CTA is visible to the whole system before the CTA counts as done: the
    // barrier orders all threads' stores before thread 0's system-scope fence, which is cumulative,
    // so one fence per CTA covers them (a fence in every thread: 870 against 856 us for the emulated
    // world's eight prefill dispatches on one box)
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence_system();
        last = atomicInc(a.done, gridDim.x - 1) == gridDim.x - 1;
    }
    __syncthreads();
    if (last && src_ok && int(threadIdx.x) < a.R && act[threadIdx.x] != 0) {
        __threadfence_system();  // after every other CTA's fenced stores (seen through the counter)
        st_release_sys_u64(reinterpret_cast<uint64_t*>(__ldg(a.flags + threadIdx.x)) + a.rank, a.signal);
    }
}

// ---------------------------------------------------------------------------- waits and signals

// Thread s waits until this rank's flag word s holds at least `signal`, for every
// active source s, giving up after kWaitTimeoutNs (EP_STATUS_TIMEOUT).  With
// wait_ns, the nanoseconds it waited for source s (until the flag or the give-up)
// are added to wait_ns[s].
__global__ void __launch_bounds__(EP_MAX_RANKS) wait_peers_kernel(const uint64_t* flags, int R, uint64_t signal,
                                                                  const uint8_t* active, int32_t* status,
                                                                  int64_t* wait_ns) {
    pdl_wait();
    const int s = threadIdx.x;
    if (s >= R || active[s] == 0) return;
    const uint64_t t0 = global_timer_ns();
    uint64_t t = t0;
    for (uint32_t it = 0;; ++it) {
        if (ld_acquire_sys_u64(flags + s) >= signal) break;
        if ((it & 63u) == 63u) {
            t = global_timer_ns();
            if (t - t0 > kWaitTimeoutNs) {
                flag_status(status, EP_STATUS_TIMEOUT);
                break;
            }
        }
        __nanosleep(64);
    }
    if (wait_ns) wait_ns[s] += int64_t(global_timer_ns() - t0);
}

// Thread d releases `signal` into word `rank` of every active rank d's flags.
__global__ void __launch_bounds__(EP_MAX_RANKS) signal_peers_kernel(const uint64_t* peer_flags, int R, int rank,
                                                                    const uint8_t* active, uint64_t signal) {
    pdl_wait();  // the kernels before this one in the stream have completed and their writes are visible
    const int d = threadIdx.x;
    if (d >= R || active[rank] == 0 || active[d] == 0) return;
    __threadfence_system();
    st_release_sys_u64(reinterpret_cast<uint64_t*>(__ldg(peer_flags + d)) + rank, signal);
}

// recv_count[le] = sum over ranks s of counts[s][rank * E_local + le].
__global__ void __launch_bounds__(256) peer_recv_count_kernel(const int32_t* counts, int R, int E, int rank,
                                                              int32_t* recv_count) {
    pdl_wait();
    const int E_local = E / R;
    for (int le = blockIdx.x * blockDim.x + threadIdx.x; le < E_local; le += gridDim.x * blockDim.x) {
        int32_t n = 0;
        for (int s = 0; s < R; ++s) n += __ldg(counts + int64_t(s) * E + int64_t(rank) * E_local + le);
        recv_count[le] = n;
    }
}

// ---------------------------------------------------------------------------- combine

// The vector combine over peer rows: for every token, slots j = 0..k-1 in order,
// acc = fmaf(w_j, y_j, acc) in float32 from +0, rounded to bf16 (nearest even).
// Slots are taken in groups of kPeerSlotGroup: a lane issues the group's loads,
// then accumulates them in slot order.
template <int U>
__global__ void __launch_bounds__(kPeerThreads, 2) combine_peer_kernel(PeerArgs a) {
    extern __shared__ int32_t off[];  // [E]
    __shared__ int32_t act[EP_MAX_RANKS];
    pdl_wait();
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) act[i] = a.active[i];
    source_offsets(a, off);
    __syncthreads();
    const bool src_ok = act[a.rank] != 0;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int nvec = int(a.row_bytes >> 4);
    const int piece_vec = 32 * U;
    const int np = (nvec + piece_vec - 1) / piece_vec;
    const int64_t n_units = int64_t(a.T) * np;
    // contiguous, balanced ranges of units per warp: on the emulated world this ran 963 us at
    // prefill against 1144 us with units strided over the grid from the last token
    const int64_t q = n_units / warps, rem = n_units % warps;
    const int64_t u0 = gw * q + (gw < rem ? gw : rem);
    const int64_t u1 = u0 + q + (gw < rem ? 1 : 0);

    int64_t cur_tok = -1;
    uint32_t mask = 0;
    uint64_t my_addr = 0;
    float my_w = 0.f;
    for (int64_t u = u0; u < u1; ++u) {
        const int64_t t = u / np;
        const int pc = int(u - t * np);
        if (t != cur_tok) {
            cur_tok = t;
            const PeerSlot s = peer_slot(a, act, off, t, lane, src_ok, pc == 0);
            my_addr = s.addr;
            my_w = s.w;
            mask = __ballot_sync(0xffffffffu, s.addr != 0ull);
        }
        const int v0 = pc * piece_vec + lane;
        float acc[U][8];
#pragma unroll
        for (int uu = 0; uu < U; ++uu)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[uu][c] = 0.f;
        for (int jb = 0; jb < a.k; jb += kPeerSlotGroup) {
            if (((mask >> jb) & ((1u << kPeerSlotGroup) - 1u)) == 0u) continue;
            uint4 yv[U][kPeerSlotGroup];
            float wt[kPeerSlotGroup];
#pragma unroll
            for (int j = 0; j < kPeerSlotGroup; ++j) {
                const int jj = jb + j;
                const bool on = jj < a.k && ((mask >> jj) & 1u);
                const uint64_t p = __shfl_sync(0xffffffffu, my_addr, jj & 31);
                wt[j] = __shfl_sync(0xffffffffu, my_w, jj & 31);
#pragma unroll
                for (int uu = 0; uu < U; ++uu) {
                    const int v = v0 + 32 * uu;
                    if (on && v < nvec) yv[uu][j] = ld_peer_v4(reinterpret_cast<const uint8_t*>(p) + int64_t(v) * 16);
                }
            }
#pragma unroll
            for (int j = 0; j < kPeerSlotGroup; ++j) {
                const int jj = jb + j;
                if (jj >= a.k || !((mask >> jj) & 1u)) continue;
#pragma unroll
                for (int uu = 0; uu < U; ++uu) {
                    const uint32_t wd[4] = {yv[uu][j].x, yv[uu][j].y, yv[uu][j].z, yv[uu][j].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[uu][2 * i] = fmaf(wt[j], __uint_as_float(wd[i] << 16), acc[uu][2 * i]);
                        acc[uu][2 * i + 1] = fmaf(wt[j], __uint_as_float(wd[i] & 0xffff0000u), acc[uu][2 * i + 1]);
                    }
                }
            }
        }
        uint8_t* dst = a.out + t * a.row_bytes;
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int v = v0 + 32 * uu;
            if (v >= nvec) continue;
            uint32_t words[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(acc[uu][2 * i], acc[uu][2 * i + 1]);
                words[i] = *reinterpret_cast<const uint32_t*>(&h);
            }
            st_global_v4_stream(dst + int64_t(v) * 16, make_uint4(words[0], words[1], words[2], words[3]));
        }
    }
}

// ---------------------------------------------------------------------------- host helpers

int check_peer_dims(const ep_dims_t& d, int rank) {
    const int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    if (rank < 0 || rank >= d.num_ranks) return EP_ERR_INVALID;
    return EP_OK;
}

bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

template <typename K>
int launch_peer_stream(K kernel, const PeerArgs& a, int units, const ep_cfg_t& cfg, cudaStream_t stream) {
    const int sms = sm_count();
    if (sms <= 0) return EP_ERR_CUDA;
    const size_t smem = size_t(a.E) * 4;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return EP_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kPeerThreads, smem) != cudaSuccess)
        return EP_ERR_CUDA;
    int64_t grid = int64_t(sms) * std::max(1, occ);
    if (cfg.max_ctas > 0) grid = std::min<int64_t>(grid, cfg.max_ctas);
    grid = std::max<int64_t>(1, std::min<int64_t>(grid, ceil_div(units, 8)));
    if (launch_pdl(kernel, dim3(unsigned(grid)), dim3(kPeerThreads), smem, stream, a) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

// Driver entry points reached through the runtime, so the library needs no link
// against libcuda.
PFN_cuMemGetAddressRange_v3020 g_get_range = nullptr;
bool driver_range_fn() {
    if (g_get_range) return true;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
        cudaGetLastError();
        return false;
    }
    g_get_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
    return true;
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" int ep_peer_offsets(int32_t num_ranks, int32_t num_experts, int32_t rank, const int32_t* counts,
                               int32_t* expert_rank_offset, int32_t* recv_count) {
    if (num_ranks <= 0 || num_experts <= 0 || num_experts % num_ranks != 0) return EP_ERR_INVALID;
    if (rank < 0 || rank >= num_ranks || !counts || !expert_rank_offset || !recv_count) return EP_ERR_INVALID;
    const int E_local = num_experts / num_ranks;
    for (int e = 0; e < num_experts; ++e) {
        int64_t s = 0;
        for (int r = 0; r < rank; ++r) s += counts[int64_t(r) * num_experts + e];
        if (s > INT32_MAX) return EP_ERR_INVALID;
        expert_rank_offset[e] = int32_t(s);
    }
    for (int le = 0; le < E_local; ++le) {
        int64_t n = 0;
        for (int r = 0; r < num_ranks; ++r) n += counts[int64_t(r) * num_experts + int64_t(rank) * E_local + le];
        if (n > INT32_MAX) return EP_ERR_INVALID;
        recv_count[le] = int32_t(n);
    }
    return EP_OK;
}

extern "C" size_t ep_dispatch_peer_workspace_bytes(void) { return 16; }

extern "C" int ep_dispatch_peer(ep_dims_t d, int32_t rank, ep_peer_table_t peers, const uint16_t* x,
                                const int32_t* topk_idx, const int32_t* local_row, const int32_t* counts,
                                const uint8_t* active, uint64_t signal, void* workspace, size_t workspace_bytes,
                                int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_dispatch_peer");
    int rc = check_peer_dims(d, rank);
    if (rc != EP_OK) return rc;
    if (!peers.slab || !peers.src_info || !peers.flags || !counts || !active) return EP_ERR_INVALID;
    if (!workspace || workspace_bytes < ep_dispatch_peer_workspace_bytes() || !aligned8(workspace))
        return EP_ERR_INVALID;
    if (d.num_tokens > 0 && (!x || !topk_idx || !local_row || !aligned16(x))) return EP_ERR_INVALID;
    PeerArgs a{};
    a.x = reinterpret_cast<const uint8_t*>(x);
    a.topk_idx = topk_idx;
    a.w = nullptr;
    a.local_row = local_row;
    a.counts = counts;
    a.active = active;
    a.slab = peers.slab;
    a.src_info = peers.src_info;
    a.flags = peers.flags;
    a.done = static_cast<uint32_t*>(workspace);
    a.status = status;
    a.R = d.num_ranks;
    a.T = d.num_tokens;
    a.k = d.num_topk;
    a.E = d.num_experts;
    a.E_local = d.num_experts / d.num_ranks;
    a.rank = rank;
    a.cap = int64_t(d.num_ranks) * d.num_tokens;
    a.row_bytes = int64_t(d.hidden) * 2;
    a.signal = signal;
    // every call launches, even with no tokens: the flags tell the receivers this source is done
    const int64_t units = std::max<int64_t>(1, int64_t(d.num_tokens) * ceil_div(a.row_bytes >> 4, 32 * 4));
    return launch_peer_stream(dispatch_peer_kernel<4>, a, int(std::min<int64_t>(units, INT32_MAX)), cfg,
                              static_cast<cudaStream_t>(stream));
}

extern "C" int ep_wait_peers(int32_t num_ranks, const uint64_t* flags, uint64_t signal, const uint8_t* active,
                             int64_t* wait_ns, int32_t* status, void* stream) {
    EP_NVTX_RANGE("ep_wait_peers");
    if (num_ranks <= 0 || num_ranks > EP_MAX_RANKS || !flags || !active || !status || !aligned8(flags) ||
        (wait_ns && !aligned8(wait_ns)))
        return EP_ERR_INVALID;
    if (launch_pdl(wait_peers_kernel, dim3(1), dim3(EP_MAX_RANKS), 0, static_cast<cudaStream_t>(stream), flags,
                   int(num_ranks), signal, active, status, wait_ns) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

extern "C" int ep_signal_peers(int32_t num_ranks, int32_t rank, const uint64_t* peer_flags, const uint8_t* active,
                               uint64_t signal, void* stream) {
    EP_NVTX_RANGE("ep_signal_peers");
    if (num_ranks <= 0 || num_ranks > EP_MAX_RANKS || rank < 0 || rank >= num_ranks || !peer_flags || !active)
        return EP_ERR_INVALID;
    if (launch_pdl(signal_peers_kernel, dim3(1), dim3(EP_MAX_RANKS), 0, static_cast<cudaStream_t>(stream),
                   peer_flags, int(num_ranks), int(rank), active, signal) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

extern "C" int ep_peer_recv_count(int32_t num_ranks, int32_t num_experts, int32_t rank, const int32_t* counts,
                                  int32_t* recv_count, void* stream) {
    EP_NVTX_RANGE("ep_peer_recv_count");
    if (num_ranks <= 0 || num_experts <= 0 || num_experts % num_ranks != 0 || rank < 0 || rank >= num_ranks ||
        !counts || !recv_count)
        return EP_ERR_INVALID;
    const int E_local = num_experts / num_ranks;
    const int blocks = int(std::min<int64_t>(64, ceil_div(E_local, 256)));
    if (launch_pdl(peer_recv_count_kernel, dim3(blocks), dim3(256), 0, static_cast<cudaStream_t>(stream), counts,
                   int(num_ranks), int(num_experts), int(rank), recv_count) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

extern "C" int ep_combine_peer(ep_dims_t d, int32_t rank, const uint64_t* y_slabs, const int32_t* topk_idx,
                               const float* topk_weights, const int32_t* local_row, const int32_t* counts,
                               const uint8_t* active, uint16_t* out, int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_combine_peer");
    int rc = check_peer_dims(d, rank);
    if (rc != EP_OK) return rc;
    if (d.num_tokens == 0) return EP_OK;
    if (!y_slabs || !topk_idx || !topk_weights || !local_row || !counts || !active || !out || !aligned16(out))
        return EP_ERR_INVALID;
    PeerArgs a{};
    a.topk_idx = topk_idx;
    a.w = topk_weights;
    a.local_row = local_row;
    a.counts = counts;
    a.active = active;
    a.slab = y_slabs;
    a.out = reinterpret_cast<uint8_t*>(out);
    a.status = status;
    a.R = d.num_ranks;
    a.T = d.num_tokens;
    a.k = d.num_topk;
    a.E = d.num_experts;
    a.E_local = d.num_experts / d.num_ranks;
    a.rank = rank;
    a.cap = int64_t(d.num_ranks) * d.num_tokens;
    a.row_bytes = int64_t(d.hidden) * 2;
    // cfg.threads = 2: two 16-byte columns per lane and unit (emulated world, prefill: 941-960 against
    // 962-979 us; at 8 x 512 tokens 166-170 against 158-162 us); otherwise one.  (Four spill registers
    // under the two-CTAs-per-SM bound and ran 1587 us.)
    const int U = cfg.threads == 2 ? 2 : 1;
    const int64_t units = int64_t(d.num_tokens) * ceil_div(a.row_bytes >> 4, 32 * U);
    const int n = int(std::min<int64_t>(units, INT32_MAX));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return U == 2 ? launch_peer_stream(combine_peer_kernel<2>, a, n, cfg, st)
                  : launch_peer_stream(combine_peer_kernel<1>, a, n, cfg, st);
}

extern "C" int ep_ipc_export(const void* ptr, void* handle, uint64_t* offset) {
    EP_NVTX_RANGE("ep_ipc_export");
    if (!ptr || !handle || !offset) return EP_ERR_INVALID;
    if (!driver_range_fn()) return EP_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (g_get_range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return EP_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
        cudaGetLastError();
        return EP_ERR_CUDA;
    }
    static_assert(sizeof(h) == EP_IPC_HANDLE_BYTES, "CUDA IPC handle size");
    std::memcpy(handle, &h, sizeof(h));
    *offset = uint64_t(reinterpret_cast<CUdeviceptr>(ptr) - base);
    return EP_OK;
}

extern "C" int ep_ipc_import(const void* handle, uint64_t offset, void** ptr, void** base) {
    EP_NVTX_RANGE("ep_ipc_import");
    if (!handle || !ptr || !base) return EP_ERR_INVALID;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void* b = nullptr;
    if (cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess || b == nullptr) {
        cudaGetLastError();
        return EP_ERR_CUDA;
    }
    *base = b;
    *ptr = static_cast<char*>(b) + offset;
    return EP_OK;
}

extern "C" int ep_ipc_close(void* base) {
    EP_NVTX_RANGE("ep_ipc_close");
    if (!base) return EP_ERR_INVALID;
    if (cudaIpcCloseMemHandle(base) != cudaSuccess) {
        cudaGetLastError();
        return EP_ERR_CUDA;
    }
    return EP_OK;
}
