// ep_combine.cu -- top-k weighted gather-reduce on sm_100a.
//
// Defines Buffer.low_latency_combine of the NeMo AutoModel page
// "nemo_automodel.components.moe.uccl_ep.buffer": the expert outputs in the
// receive slabs [num_local_experts, num_ranks * num_max_dispatch_tokens_per_rank,
// hidden] are reduced WITH weights back to [num_tokens, hidden] bf16, with -1
// indices skipped.  The active-rank mask is re-read at combine time, as in the
// ai-dynamo/nixl PR "nixl_ep: Optimize low-latency NVLink path" (combine active
// rank mask optimization): experts of a masked rank contribute nothing and a
// masked source rank's tokens come out as zeros.
//
// Numerics: acc starts at +0.0f and, for j = 0..k-1 in that order,
// acc = fmaf(w[j], float(y_j), acc) over the live slots; the result is
// rounded to bf16 to nearest-even.
//
// Two data paths (ep_cfg_t.variant; EP_VARIANT_AUTO picks the vector path when
// k <= 8, the faster one on B200: 6.3 TB/s against 4.2 TB/s at the prefill
// shape, because every staged byte must pass through registers for the FMA
// anyway and the vector path keeps k * 2 16-byte loads in flight per lane).
//
// Bulk path.  A persistent grid, one CTA per SM; CTA b owns a contiguous,
// balanced range of tokens and walks its units (one token, one piece of its
// row: pieces keep k staged rows within one pipeline stage) in order.
// Warp 0 is the producer: lane j reads slot j's routing and, when the slot is
// live, issues a cp.async.bulk global->shared load of that row piece into the
// stage, all completing on the stage's "full" mbarrier; the slot weights and
// live mask go into the stage header.  The other warps are consumers: each
// thread owns 16-byte columns of the piece, reads the k staged vectors from
// shared memory, accumulates in float32, and streams the bf16 result to the
// output; then each consumer warp arrives on the stage's "empty" mbarrier so
// the producer can refill it.  The producer reads a token's routing once for
// all its pieces and prefetches the next token's routing while it streams the
// current one, so it runs up to S stages ahead: S * k * piece bytes of loads
// in flight per SM.
#include <algorithm>
#include <atomic>
#include <cstdint>

#include <cuda_bf16.h>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr uint32_t kCombinePieceMax = 4096;   // bytes of one slot's row piece
constexpr uint32_t kCombineStageMax = 49152;  // k * piece bytes per stage at most
constexpr int kCombineMaxStages = 16;
constexpr int kActiveSlots = 64;

struct CombineArgs {
    const uint8_t* y;
    const int32_t* topk_idx;
    const float* w;
    const int32_t* pair_row;
    const uint8_t* active;
    uint8_t* out;
    int32_t* status;
    int R, T, k, E, E_local;
    int64_t row_bytes;
    int64_t cap;
    int n_pieces;
    uint32_t piece_bytes;
    uint32_t slot_bytes;   // stride of a slot inside a stage (>= piece_bytes)
    uint32_t stage_bytes;  // k * slot_bytes
    int stages;
    int64_t n_units;
};

struct StageHeader {
    float w[32];
    uint32_t live;
    uint32_t pad[3];
};

__device__ __forceinline__ uint32_t piece_size(const CombineArgs& a, int q) {
    return q + 1 < a.n_pieces ? a.piece_bytes : uint32_t(a.row_bytes - int64_t(q) * a.piece_bytes);
}

__device__ __forceinline__ void fma_bf16x8(float* acc, float w, uint4 v) {
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(words[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(words[i] & 0xffff0000u), acc[2 * i + 1]);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float* acc) {
    uint32_t words[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        words[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(words[0], words[1], words[2], words[3]);
}

struct SlotMeta {
    int e;
    int row;
    float w;
};

// Slot `lane` of a token: its slab (expert; in normal mode the destination rank
// itself), slab row and weight (1 in normal mode: the sum is unweighted).
template <bool NORMAL>
__device__ __forceinline__ SlotMeta load_slot(const CombineArgs& a, int64_t tok, int lane) {
    SlotMeta m{-1, -1, 0.f};
    if (lane < a.k) {
        const int64_t p = tok * a.k + lane;
        m.e = NORMAL ? lane : __ldg(a.topk_idx + p);
        m.row = __ldg(a.pair_row + p);
        m.w = NORMAL ? 1.0f : __ldg(a.w + p);
    }
    return m;
}

template <bool NORMAL>
__global__ void combine_kernel(CombineArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int S = a.stages;
    uint8_t* data = smem;
    StageHeader* hdr = reinterpret_cast<StageHeader*>(smem + size_t(S) * a.stage_bytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(hdr + S);
    uint64_t* empty = full + S;
    int32_t* act = reinterpret_cast<int32_t*>(empty + S);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int consumer_warps = (blockDim.x >> 5) - 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), consumer_warps);
        }
        mbar_init_fence();
    }
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) act[i] = a.active[i];
    __syncthreads();

    // contiguous, balanced token range of this CTA; its units are (token, piece) in order
    const int64_t n_tok = a.n_units / a.n_pieces;
    const int64_t q_tok = n_tok / gridDim.x, rem = n_tok % gridDim.x;
    const int64_t tok0 = int64_t(blockIdx.x) * q_tok + (int64_t(blockIdx.x) < rem ? int64_t(blockIdx.x) : rem);
    const int64_t my_tok = q_tok + (int64_t(blockIdx.x) < rem ? 1 : 0);
    const int64_t my_n = my_tok * a.n_pieces;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = policy_evict_first();
        SlotMeta nxt = my_tok > 0 ? load_slot<NORMAL>(a, tok0, lane) : SlotMeta{-1, -1, 0.f};
        for (int64_t t = 0; t < my_tok; ++t) {
            const int64_t tok = tok0 + t;
            const SlotMeta cur = nxt;
            if (t + 1 < my_tok) nxt = load_slot<NORMAL>(a, tok + 1, lane);  // prefetch the next token's routing
            const int r = int(tok / a.T);
            const bool in_range = cur.e >= 0 && cur.e < a.E;
            const bool live = lane < a.k && cur.row >= 0 && cur.row < a.cap && in_range && act[r] != 0 &&
                              act[cur.e / a.E_local] != 0;
            if (lane < a.k && cur.row >= 0 && !in_range) flag_status(a.status, EP_STATUS_BAD_EXPERT);
            if (lane < a.k && cur.row >= a.cap && in_range) flag_status(a.status, EP_STATUS_OVERFLOW);
            const uint32_t mask = __ballot_sync(0xffffffffu, live);
            const uint8_t* src_row = live ? a.y + (int64_t(cur.e) * a.cap + cur.row) * a.row_bytes : nullptr;
            for (int q = 0; q < a.n_pieces; ++q) {
                const int64_t i = t * a.n_pieces + q;
                const int s = int(i % S);
                const uint32_t parity = uint32_t((i / S) & 1);
                const bool free_stage = __all_sync(0xffffffffu, mbar_wait(smem_u32(empty + s), parity ^ 1u));
                if (!free_stage) {
                    if (lane == 0) flag_status(a.status, EP_STATUS_TIMEOUT);
                    return;
                }
                const uint32_t bytes = piece_size(a, q);
                if (lane < a.k) hdr[s].w[lane] = live ? cur.w : 0.f;
                if (lane == 0) hdr[s].live = mask;
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(smem_u32(full + s), uint32_t(__popc(mask)) * bytes);
                __syncwarp();
                if (live)
                    bulk_load(smem_u32(data + size_t(s) * a.stage_bytes + size_t(lane) * a.slot_bytes),
                              src_row + int64_t(q) * a.piece_bytes, bytes, smem_u32(full + s), pol);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int ct = threadIdx.x - 32;
    const int nct = consumer_warps * 32;
    for (int64_t i = 0; i < my_n; ++i) {
        const int s = int(i % S);
        const uint32_t parity = uint32_t((i / S) & 1);
        const bool landed = __all_sync(0xffffffffu, mbar_wait(smem_u32(full + s), parity));
        if (!landed) {
            if (lane == 0) flag_status(a.status, EP_STATUS_TIMEOUT);
            break;
        }
        const int64_t tok = tok0 + i / a.n_pieces;
        const int q = int(i % a.n_pieces);
        const uint32_t nvec = piece_size(a, q) >> 4;
        const uint32_t mask = hdr[s].live;
        const uint8_t* stage = data + size_t(s) * a.stage_bytes;
        uint8_t* dst = a.out + tok * a.row_bytes + int64_t(q) * a.piece_bytes;
        for (uint32_t v = ct; v < nvec; v += nct) {
            float acc[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = 0.f;
            for (int j0 = 0; j0 < a.k; j0 += 8) {
                uint4 yv[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = j0 + jj;
                    if (j < a.k && ((mask >> j) & 1u))
                        yv[jj] = *reinterpret_cast<const uint4*>(stage + size_t(j) * a.slot_bytes + size_t(v) * 16);
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = j0 + jj;
                    if (j < a.k && ((mask >> j) & 1u)) fma_bf16x8(acc, hdr[s].w[j], yv[jj]);
                }
            }
            st_global_v4_stream(dst + size_t(v) * 16, pack_bf16x8(acc));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(empty + s));
    }
}

// ---------------------------------------------------------------------------
// Vector path (EP_VARIANT_VECTOR, k <= 8): the warps take units (token, piece of
// 32*U 16-byte columns) strided from the end of the token range (low-latency
// mode) or in contiguous ranges (normal mode).  At a new token
// lane j reads slot j's routing and the slot pointers and weights are
// broadcast with shuffles; then each lane issues all k * U 16-byte loads of
// its columns at once (L1 bypassed, 256-byte L2 fetch), accumulates in slot
// order and stores its U result vectors.
constexpr int kVecKMax = 8;

template <int U, bool NORMAL>
__global__ void __launch_bounds__(256) combine_vec_kernel(CombineArgs a) {
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits
    __shared__ int32_t act[kActiveSlots];
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) act[i] = a.active[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int nvec = int(a.row_bytes >> 4);
    const int piece_vec = 32 * U;
    const int np = (nvec + piece_vec - 1) / piece_vec;
    const int64_t n_units = int64_t(a.R) * a.T * np;
    // Low-latency mode takes units strided from the end: warp gw takes units n-1-gw, n-1-gw-W, ...
    // (W = warps), so at any moment the grid works on one window of consecutive tokens, whose rows of
    // the busy experts are neighbours in the slabs, and it starts with the tokens dispatched last,
    // whose rows may still sit in L2.  (Contiguous ranges per warp read ~W scattered regions at once:
    // 649 against 606 us for the whole prefill combine on B200, 682 against 626 us right after a
    // dispatch.)  Normal mode keeps contiguous, balanced ranges per warp: its rows are per destination
    // rank in (source, token) order, and the strided order measured slower there (457 against 444 us).
    int64_t my_n, u0 = 0;
    if (NORMAL) {
        const int64_t q = n_units / warps, rem = n_units % warps;
        u0 = gw * q + (gw < rem ? gw : rem);
        my_n = q + (gw < rem ? 1 : 0);
    } else {
        my_n = gw < n_units ? (n_units - 1 - gw) / warps + 1 : 0;
    }

    int64_t cur_tok = -1;
    uint32_t mask = 0;
    const uint8_t* src[kVecKMax];
    float wt[kVecKMax];
    for (int64_t i = 0; i < my_n; ++i) {
        const int64_t u = NORMAL ? u0 + i : n_units - 1 - gw - i * warps;
        const int64_t tok = u / np;
        const int pc = int(u - tok * np);
        if (tok != cur_tok) {
            cur_tok = tok;
            const int r = int(tok / a.T);
            int e = -1, row = -1;
            float w = 0.f;
            if (lane < a.k) {
                const SlotMeta m = load_slot<NORMAL>(a, tok, lane);
                e = m.e;
                row = m.row;
                w = m.w;
            }
            const bool in_range = e >= 0 && e < a.E;
            const bool live = lane < a.k && row >= 0 && row < a.cap && in_range && act[r] != 0 &&
                              act[e / a.E_local] != 0;
            if (lane < a.k && pc == 0) {
                if (row >= 0 && !in_range) flag_status(a.status, EP_STATUS_BAD_EXPERT);
                if (row >= a.cap && in_range) flag_status(a.status, EP_STATUS_OVERFLOW);
            }
            mask = __ballot_sync(0xffffffffu, live);
            const unsigned long long ptr =
                live ? reinterpret_cast<unsigned long long>(a.y + (int64_t(e) * a.cap + row) * a.row_bytes) : 0ull;
#pragma unroll
            for (int j = 0; j < kVecKMax; ++j) {
                src[j] = reinterpret_cast<const uint8_t*>(__shfl_sync(0xffffffffu, ptr, j));
                wt[j] = __shfl_sync(0xffffffffu, w, j);
            }
        }
        const int v0 = pc * piece_vec + lane;
        uint4 yv[U][kVecKMax];
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int v = v0 + 32 * uu;
#pragma unroll
            for (int j = 0; j < kVecKMax; ++j)
                if (((mask >> j) & 1u) && v < nvec) yv[uu][j] = ld_stream_v4(src[j] + int64_t(v) * 16);
        }
        uint8_t* dst = a.out + tok * a.row_bytes;
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int v = v0 + 32 * uu;
            if (v >= nvec) continue;
            float acc[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
            for (int j = 0; j < kVecKMax; ++j)
                if ((mask >> j) & 1u) fma_bf16x8(acc, wt[j], yv[uu][j]);
            st_global_v4_stream(dst + int64_t(v) * 16, pack_bf16x8(acc));
        }
    }
}

template <int U, bool NORMAL>
int launch_combine_vec(const CombineArgs& a, const ep_cfg_t& cfg, int sms, cudaStream_t stream) {
    static std::atomic<int> per_sm[64];  // resident CTAs per SM, per device; 0 = not asked yet
    int dev = 0;
    cudaGetDevice(&dev);
    int occ = per_sm[dev & 63].load(std::memory_order_relaxed);
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, combine_vec_kernel<U, NORMAL>, 256, 0) != cudaSuccess)
            return EP_ERR_CUDA;
        per_sm[dev & 63].store(occ, std::memory_order_relaxed);
    }
    // default: the CTAs that fit at once (low-latency mode, strided units: a 3x grid measured
    // slower, 619 against 606 us at 8 x 4096 tokens); in normal mode (contiguous unit ranges) three
    // times that for a large problem (>= 128 units per resident warp), whose later waves fill the SMs
    // that finish first; cfg.max_ctas sets the grid
    const int64_t resident = int64_t(sms) * std::max(1, occ);
    const int64_t units = int64_t(a.R) * a.T * ceil_div(a.row_bytes >> 4, 32 * U);
    int64_t grid = cfg.max_ctas > 0 ? int64_t(cfg.max_ctas)
                   : (NORMAL && units >= 128 * resident * (256 / 32) ? 3 * resident : resident);
    const int64_t warps_needed = units;
    grid = std::max<int64_t>(1, std::min<int64_t>(grid, ceil_div(warps_needed, 8)));
    if (launch_pdl(combine_vec_kernel<U, NORMAL>, dim3(unsigned(grid)), dim3(256), 0, stream, a) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

// Vector or bulk path for a filled CombineArgs (a.k slots per token).
template <bool NORMAL>
int run_combine(CombineArgs& a, const ep_cfg_t& cfg, int variant, cudaStream_t stream) {
    if (variant == EP_VARIANT_VECTOR) {
        const int sms = sm_count();
        if (sms <= 0) return EP_ERR_CUDA;
        // cfg.threads selects the columns per lane and unit (1 or 2; 2 measured faster on B200)
        return cfg.threads == 1 ? launch_combine_vec<1, NORMAL>(a, cfg, sms, stream)
                                : launch_combine_vec<2, NORMAL>(a, cfg, sms, stream);
    }
    const uint32_t piece_max =
        std::max<uint32_t>(16, std::min<uint32_t>(kCombinePieceMax, (kCombineStageMax / a.k) & ~15u));
    a.n_pieces = int(ceil_div(a.row_bytes, piece_max));
    a.piece_bytes = uint32_t(round_up16(size_t(ceil_div(a.row_bytes, a.n_pieces))));
    if (int64_t(a.n_pieces - 1) * a.piece_bytes >= a.row_bytes) return EP_ERR_UNSUPPORTED;
    a.slot_bytes = a.piece_bytes;
    a.stage_bytes = uint32_t(a.k) * a.slot_bytes;
    a.n_units = int64_t(a.R) * a.T * a.n_pieces;

    const int sms = sm_count();
    if (sms <= 0) return EP_ERR_CUDA;
    const size_t fixed = size_t(kActiveSlots) * 4 + 1024;
    const size_t per_stage = size_t(a.stage_bytes) + sizeof(StageHeader) + 16;
    const size_t budget = size_t(max_smem_optin()) - fixed;
    int stages = cfg.stages > 0 ? cfg.stages : int(budget / per_stage);
    stages = std::max(2, std::min(kCombineMaxStages, stages));
    a.stages = stages;
    const size_t smem = size_t(stages) * per_stage + size_t(kActiveSlots) * 4;
    if (smem > size_t(max_smem_optin())) return EP_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(combine_kernel<NORMAL>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
        return EP_ERR_CUDA;

    const int nvec = int(a.piece_bytes / 16);
    int consumer_warps = cfg.threads > 0 ? std::max(1, cfg.threads / 32 - 1) : (nvec + 31) / 32;
    consumer_warps = std::max(1, std::min(15, consumer_warps));
    int64_t grid = sms;
    if (cfg.max_ctas > 0) grid = std::min<int64_t>(grid, cfg.max_ctas);
    grid = std::min<int64_t>(grid, int64_t(a.R) * a.T);
    if (launch_pdl(combine_kernel<NORMAL>, dim3(unsigned(grid)), dim3(32 * (1 + consumer_warps)), smem, stream, a) !=
        cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" int ep_combine(ep_dims_t d, const uint16_t* y, const int32_t* topk_idx, const float* topk_weights,
                          const int32_t* pair_row, const uint8_t* active, uint16_t* out, int32_t* status,
                          ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_combine");
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (RT == 0) return EP_OK;
    if (!y || !topk_idx || !topk_weights || !pair_row || !active || !out) return EP_ERR_INVALID;
    if (!aligned16(y) || !aligned16(out)) return EP_ERR_INVALID;

    const int variant = cfg.variant != EP_VARIANT_AUTO ? cfg.variant
                        : (d.num_topk <= kVecKMax ? EP_VARIANT_VECTOR : EP_VARIANT_BULK);
    if (variant != EP_VARIANT_BULK && variant != EP_VARIANT_VECTOR) return EP_ERR_INVALID;
    if (variant == EP_VARIANT_VECTOR && d.num_topk > kVecKMax) return EP_ERR_UNSUPPORTED;

    CombineArgs a;
    a.y = reinterpret_cast<const uint8_t*>(y);
    a.topk_idx = topk_idx;
    a.w = topk_weights;
    a.pair_row = pair_row;
    a.active = active;
    a.out = reinterpret_cast<uint8_t*>(out);
    a.status = status;
    a.R = d.num_ranks;
    a.T = d.num_tokens;
    a.k = d.num_topk;
    a.E = d.num_experts;
    a.E_local = d.num_experts / d.num_ranks;
    a.row_bytes = int64_t(d.hidden) * 2;
    a.cap = RT;
    return run_combine<false>(a, cfg, variant, static_cast<cudaStream_t>(stream));
}


extern "C" int ep_normal_combine(ep_dims_t d, int32_t recv_capacity, const uint16_t* y,
                                 const int32_t* token_recv_row, const uint8_t* active, uint16_t* out,
                                 int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_normal_combine");
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    if (recv_capacity < 0) return EP_ERR_INVALID;
    if (d.num_ranks > EP_MAX_NORMAL_RANKS) return EP_ERR_UNSUPPORTED;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (RT == 0) return EP_OK;
    if (!token_recv_row || !active || !out || (recv_capacity > 0 && !y)) return EP_ERR_INVALID;
    if ((y && !aligned16(y)) || !aligned16(out)) return EP_ERR_INVALID;
    const int variant = cfg.variant != EP_VARIANT_AUTO ? cfg.variant
                        : (d.num_ranks <= kVecKMax ? EP_VARIANT_VECTOR : EP_VARIANT_BULK);
    if (variant != EP_VARIANT_BULK && variant != EP_VARIANT_VECTOR) return EP_ERR_INVALID;
    if (variant == EP_VARIANT_VECTOR && d.num_ranks > kVecKMax) return EP_ERR_UNSUPPORTED;
    // slots are the destination ranks: slab d of y is rank d's receive buffer
    CombineArgs a;
    a.y = reinterpret_cast<const uint8_t*>(y);
    a.topk_idx = nullptr;
    a.w = nullptr;
    a.pair_row = token_recv_row;
    a.active = active;
    a.out = reinterpret_cast<uint8_t*>(out);
    a.status = status;
    a.R = d.num_ranks;
    a.T = d.num_tokens;
    a.k = d.num_ranks;
    a.E = d.num_ranks;
    a.E_local = 1;
    a.row_bytes = int64_t(d.hidden) * 2;
    a.cap = recv_capacity;
    return run_combine<true>(a, cfg, variant, static_cast<cudaStream_t>(stream));
}
