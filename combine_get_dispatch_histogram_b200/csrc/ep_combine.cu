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
// Design.  A persistent grid, one CTA per SM, walks units (one token, one
// piece of its row: pieces keep k staged rows within one pipeline stage).
// Warp 0 is the producer: lane j reads slot j's routing and, when the slot is
// live, issues a cp.async.bulk global->shared load of that row piece into the
// stage, all completing on the stage's "full" mbarrier; the slot weights and
// live mask go into the stage header.  The other warps are consumers: each
// thread owns 16-byte columns of the piece, reads the k staged vectors from
// shared memory, accumulates in float32, and streams the bf16 result to the
// output; then each consumer warp arrives on the stage's "empty" mbarrier so
// the producer can refill it.  The producer runs up to S stages ahead, which
// keeps S * k * piece bytes of loads in flight per SM.
#include <algorithm>
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
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) act[i] = a.active[i];
    __syncthreads();

    const int64_t first = blockIdx.x, step = gridDim.x;
    const int64_t my_n = first < a.n_units ? (a.n_units - 1 - first) / step + 1 : 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = policy_evict_first();
        for (int64_t i = 0; i < my_n; ++i) {
            const int s = int(i % S);
            const uint32_t parity = uint32_t((i / S) & 1);
            const bool free_stage = __all_sync(0xffffffffu, mbar_wait(smem_u32(empty + s), parity ^ 1u));
            if (!free_stage) {
                if (lane == 0) flag_status(a.status, EP_STATUS_TIMEOUT);
                break;
            }
            const int64_t u = first + i * step;
            const int64_t tok = u / a.n_pieces;
            const int q = int(u - tok * a.n_pieces);
            const int r = int(tok / a.T);
            bool live = false;
            int e = -1, row = -1;
            float wt = 0.f;
            if (lane < a.k) {
                const int64_t p = tok * a.k + lane;
                e = __ldg(a.topk_idx + p);
                row = __ldg(a.pair_row + p);
                wt = __ldg(a.w + p);
                const bool in_range = e >= 0 && e < a.E;
                live = row >= 0 && row < a.cap && in_range && act[r] != 0 && act[e / a.E_local] != 0;
                if (q == 0 && row >= 0 && !in_range) flag_status(a.status, EP_STATUS_BAD_EXPERT);
                if (q == 0 && row >= a.cap && in_range) flag_status(a.status, EP_STATUS_OVERFLOW);
                hdr[s].w[lane] = live ? wt : 0.f;
            }
            const uint32_t mask = __ballot_sync(0xffffffffu, live);
            const uint32_t bytes = piece_size(a, q);
            if (lane == 0) hdr[s].live = mask;
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(smem_u32(full + s), uint32_t(__popc(mask)) * bytes);
            __syncwarp();
            if (live) {
                const uint8_t* src = a.y + (int64_t(e) * a.cap + row) * a.row_bytes + int64_t(q) * a.piece_bytes;
                bulk_load(smem_u32(data + size_t(s) * a.stage_bytes + size_t(lane) * a.slot_bytes), src, bytes,
                          smem_u32(full + s), pol);
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
        const int64_t u = first + i * step;
        const int64_t tok = u / a.n_pieces;
        const int q = int(u - tok * a.n_pieces);
        const uint32_t nvec = piece_size(a, q) >> 4;
        const uint32_t mask = hdr[s].live;
        const uint8_t* stage = data + size_t(s) * a.stage_bytes;
        uint8_t* dst = a.out + tok * a.row_bytes + int64_t(q) * a.piece_bytes;
        for (uint32_t v = ct; v < nvec; v += nct) {
            float acc[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = 0.f;
            for (int j = 0; j < a.k; ++j) {
                if ((mask >> j) & 1u) {
                    const uint4 yv = *reinterpret_cast<const uint4*>(stage + size_t(j) * a.slot_bytes + size_t(v) * 16);
                    fma_bf16x8(acc, hdr[s].w[j], yv);
                }
            }
            st_global_v4_stream(dst + size_t(v) * 16, pack_bf16x8(acc));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(empty + s));
    }
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" int ep_combine(ep_dims_t d, const uint16_t* y, const int32_t* topk_idx, const float* topk_weights,
                          const int32_t* pair_row, const uint8_t* active, uint16_t* out, int32_t* status,
                          ep_cfg_t cfg, void* stream) {
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (RT == 0) return EP_OK;
    if (!y || !topk_idx || !topk_weights || !pair_row || !active || !out) return EP_ERR_INVALID;
    if (!aligned16(y) || !aligned16(out)) return EP_ERR_INVALID;

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
    const uint32_t piece_max =
        std::max<uint32_t>(16, std::min<uint32_t>(kCombinePieceMax, (kCombineStageMax / d.num_topk) & ~15u));
    a.n_pieces = int(ceil_div(a.row_bytes, piece_max));
    a.piece_bytes = uint32_t(round_up16(size_t(ceil_div(a.row_bytes, a.n_pieces))));
    if (int64_t(a.n_pieces - 1) * a.piece_bytes >= a.row_bytes) return EP_ERR_UNSUPPORTED;
    a.slot_bytes = a.piece_bytes;
    a.stage_bytes = uint32_t(d.num_topk) * a.slot_bytes;
    a.n_units = RT * a.n_pieces;

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
    if (cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
        return EP_ERR_CUDA;

    const int nvec = int(a.piece_bytes / 16);
    int consumer_warps = cfg.threads > 0 ? std::max(1, cfg.threads / 32 - 1) : (nvec + 31) / 32;
    consumer_warps = std::max(1, std::min(15, consumer_warps));
    int64_t grid = sms;
    if (cfg.max_ctas > 0) grid = std::min<int64_t>(grid, cfg.max_ctas);
    grid = std::min<int64_t>(grid, a.n_units);
    combine_kernel<<<unsigned(grid), 32 * (1 + consumer_warps), smem, static_cast<cudaStream_t>(stream)>>>(a);
    return launch_result();
}
