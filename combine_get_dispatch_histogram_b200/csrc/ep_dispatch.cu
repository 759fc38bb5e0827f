// ep_dispatch.cu -- token dispatch on sm_100a: every token row is read from HBM
// once and written to each expert slab row its live pairs name.
//
// Defines Buffer.low_latency_dispatch (use_fp8=False) of the NeMo AutoModel
// page "nemo_automodel.components.moe.uccl_ep.buffer": bf16 rows into the
// per-local-expert receive slabs [num_local_experts,
// num_ranks * num_max_dispatch_tokens_per_rank, hidden], of which only some
// rows are valid.  The emulated ranks' slabs are consecutive slices of one
// [E, R*T, H] allocation.
//
// Two data paths (ep_cfg_t.variant).  EP_VARIANT_AUTO picks the bulk path,
// measured faster on B200 at the prefill shape (5.75 TB/s against 5.58 TB/s
// for the vector path), since the payload never has to enter registers.
//
// Bulk path.  A persistent grid of single-warp CTAs walks "units" (a token row,
// or a piece of it when a row is longer than one pipeline stage), unit
// u = blockIdx.x + i * gridDim.x.  Each CTA runs an S-stage shared-memory
// ring driven by the Tensor Memory Accelerator's bulk (non-tensor) copies:
//   - lane 0 issues one cp.async.bulk global->shared load of the row piece,
//     completing on the stage's mbarrier (skipped when no pair is live);
//   - after the stage's mbarrier flips, lane j (< k) issues one
//     cp.async.bulk shared->global store of the staged piece to its slab row
//     and writes the row's (src_rank, src_token);
//   - a stage is refilled once the stores that read it have finished reading
//     shared memory (cp.async.bulk.wait_group.read), one iteration later so
//     the wait is normally already satisfied.
// No thread touches the payload: HBM traffic is one read of each live token
// plus one write per live pair, issued by the copy engine.  The routing of
// the unit being refilled is prefetched one iteration ahead into registers
// and parked in shared memory for the consumer.
#include <algorithm>
#include <atomic>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr uint32_t kDispatchPieceMax = 16384;  // largest row piece staged at once
constexpr int kDispatchMaxStages = 16;
// Paced reads (EP_VARIANT_PACED), measured on B200 at the prefill shape: one CTA per SM with a
// 14-stage ring, L2 prefetches issued in the first 6 us of every 40 us, ~300 KB of rows ahead per
// CTA (about 45 MB of L2 in all).
constexpr uint64_t kPacePeriodNs = 40000;
constexpr uint64_t kPaceWindowNs = 6000;
constexpr int64_t kPaceAheadBytes = 300 * 1024;
// AUTO paces a low-latency dispatch only where it measured faster on B200 (L2 flushed before each
// call): >= 32 rows per SM and rows whose k stores add up to >= 48 KB.  With >= 96 KB per row one
// CTA per SM runs a 14-row ring (about one read period of stores); k = 8, 14 KB rows, 8 ranks:
// T = 4096 672 against 767 us, 2048 345 against 387, 1024 180 against 192, 640 (35 rows per SM)
// 121 against 129; T = 512 (28 rows per SM) 98 against 94 and T = 256 57 against 51.  Between 48
// and 96 KB per row (the replica workload: k = 6, 8 KB rows) two CTAs per SM share the schedule
// from 96 rows per SM on: 8 x 2048 tokens 166 against 176 us unpaced (167 against 169 on another
// box), 8 x 4096 324 against 340, but 8 x 1024 (55 rows per SM) 88 against 84.  One ring per SM
// took 253 us there (its one issuing warp cannot keep up with 8 KB copies) and three 184 us; the
// read period and window made no difference.
// Normal mode (one row per destination rank) is never paced by AUTO: 849 against 455 us.
constexpr int kPaceMinUnitsPerCta = 32;
constexpr int kPaceTwoRingMinUnitsPerSm = 96;
constexpr int64_t kPaceMinStoreBytesPerRow = 48 * 1024;
constexpr int64_t kPaceOneRingStoreBytesPerRow = 96 * 1024;
// Unpaced normal-mode grid, measured on B200 (L2 flushed before each call, 2 against 4 CTAs per SM).
// A CTA is one issuing warp that also writes every live rank's slot metadata, so four CTAs per SM
// issue faster where a 4-way split of shared memory still leaves a ring of >= 6 rows, or where
// there are few rows: 8 x 2048 tokens of 8 KB (replica) 139 against 195 us, decode (1024 rows of
// 14 KB) 22.5 against 24.6, T = 512 with rank 5 masked 59 against 63, T = 512 74 against 74.  At
// prefill (221 rows of 14 KB per SM) four CTAs get 3-row rings: 497 against 466 us.
constexpr int kNormalWideCtasPerSm = 4;
constexpr int kNormalWideMinStages = 6;
constexpr int kNormalWideMaxUnitsPerSm = 32;

struct DispatchArgs {
    const uint8_t* x;
    const int32_t* topk_idx;   // low-latency mode: slot experts; unused in normal mode
    const int32_t* pair_row;   // low-latency mode: [R*T, k] rows; normal mode: token_recv_row [R*T, R]
    uint8_t* recv_x;
    int32_t* src_info;
    int32_t* status;
    int T, k, E;               // lanes per token (k, or R in normal mode) and their slab count
    // normal mode only: the token's slots, to fill recv_topk_idx / recv_topk_weights
    const int32_t* slot_idx;
    const float* slot_w;
    const uint8_t* active;
    int32_t* recv_topk_idx;
    float* recv_topk_weights;
    int slots, slot_E, slot_E_local;
    int64_t row_bytes;
    int64_t cap;
    int n_pieces;
    uint32_t piece_bytes;
    uint32_t stage_bytes;
    int stages;
    int64_t n_units;
    // Paced reads (read_period_ns 0: off).  The rows a CTA will stage next are brought into L2
    // by prefetches issued only while globaltimer % read_period_ns < read_window_ns, up to
    // read_ahead units past the one being stored, so every SM reads in the same short windows
    // and HBM serves the stores alone in between; the staging loads then hit L2.
    uint64_t read_period_ns, read_window_ns;
    int read_ahead;
};

struct UnitMeta {
    int e;      // slab (expert; destination rank in normal mode)
    int row;
    int se;     // normal mode: this lane's slot expert if live, else -1
    float sw;   // normal mode: its weight
};

template <bool NORMAL>
__device__ __forceinline__ UnitMeta load_meta(const DispatchArgs& a, int64_t unit, int lane) {
    UnitMeta m{-1, -1, -1, 0.f};
    const int64_t tok = unit / a.n_pieces;
    if (lane < a.k) {
        const int64_t p = tok * a.k + lane;
        m.e = NORMAL ? lane : __ldg(a.topk_idx + p);
        m.row = __ldg(a.pair_row + p);
    }
    if (NORMAL && lane < a.slots) {
        const int64_t p = tok * a.slots + lane;
        const int e = __ldg(a.slot_idx + p);
        const int r = int(tok / a.T);
        const bool live = e >= 0 && e < a.slot_E && a.active[r] && a.active[e / a.slot_E_local];
        m.se = live ? e : -1;
        m.sw = __ldg(a.slot_w + p);
    }
    return m;
}

__device__ __forceinline__ uint32_t piece_size(const DispatchArgs& a, int q) {
    return q + 1 < a.n_pieces ? a.piece_bytes : uint32_t(a.row_bytes - int64_t(q) * a.piece_bytes);
}

// NOLOAD (the ceiling diagnostic only): the row loads are left out and the zeroed ring is
// stored as it is, so the kernel issues the dispatch's row stores (and, paced, its L2 prefetches)
// without waiting for any read.
template <bool NORMAL, bool NOLOAD>
__global__ void __launch_bounds__(32) dispatch_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x;
    const int S = a.stages;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(S) * a.stage_bytes);
    int2* meta = reinterpret_cast<int2*>(full + S);  // [S][32] (e, row) of the staged unit
    int2* slot = meta + S * 32;                       // [S][32] normal mode: (slot expert, weight bits)

    if (NOLOAD)
        for (size_t i = lane; i < size_t(S) * a.stage_bytes / 16; i += 32)
            reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (NOLOAD) fence_proxy_async_shared();  // the zeroed ring is read by the bulk stores
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(smem_u32(full + s), 1);
        mbar_init_fence();
    }
    __syncwarp();
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits

    const int64_t first = blockIdx.x, step = gridDim.x;
    const int64_t my_n = first < a.n_units ? (a.n_units - 1 - first) / step + 1 : 0;
    const uint64_t pol_load = policy_evict_first();
    const uint64_t pol_store = policy_evict_first();
    const uint64_t pol_prefetch = policy_evict_last();

    // Paced reads: after each unit, inside the read window (or when fewer than a ring's worth of
    // units are prefetched), prefetch the rows of units [pf, i + read_ahead) that have a live slot.
    // Lane j checks unit pf + j, so 32 units go per round.
    int64_t pf = my_n < S ? my_n : S;  // the first S units are loaded straight from HBM
    auto pace_reads = [&](int64_t i) {
        int go = 0;
        if (lane == 0)
            go = pf <= i + S || global_timer_ns() % a.read_period_ns < a.read_window_ns;
        if (!__shfl_sync(0xffffffffu, go, 0)) return;
        const int64_t want = (i + a.read_ahead) < my_n ? (i + a.read_ahead) : my_n;
        for (; pf < want; pf += 32) {
            const int64_t v = pf + lane;
            if (v >= want) continue;
            const int64_t u = first + v * step;
            const int64_t tok = u / a.n_pieces;
            bool live = false;
            for (int j = 0; j < a.k; ++j) {
                const int row = __ldg(a.pair_row + tok * a.k + j);
                live |= row >= 0 && row < a.cap;
            }
            const int q = int(u - tok * a.n_pieces);
            if (live) bulk_prefetch_l2(a.x + tok * a.row_bytes + int64_t(q) * a.piece_bytes, piece_size(a, q),
                                       pol_prefetch);
        }
        if (pf > want) pf = want;
    };

    // Stage unit i: park its routing in shared memory and start the row load.
    auto issue = [&](int64_t i, UnitMeta m) {
        const int s = int(i % S);
        const int64_t u = first + i * step;
        const int q = int(u % a.n_pieces);
        const bool valid_row = m.row >= 0 && m.row < a.cap;
        const bool live = valid_row && m.e >= 0 && m.e < a.E;
        meta[s * 32 + lane] = make_int2(live ? m.e : -1, m.row);
        if (NORMAL) slot[s * 32 + lane] = make_int2(m.se, __float_as_int(m.sw));
        if (q == 0) {
            if (m.row >= a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
            if (valid_row && !live) flag_status(a.status, EP_STATUS_BAD_EXPERT);
        }
        const bool any = __ballot_sync(0xffffffffu, live) != 0u;
        __syncwarp();
        if (lane == 0) {
            const uint32_t bar = smem_u32(full + s);
            if (any && !NOLOAD) {
                const uint32_t bytes = piece_size(a, q);
                mbar_arrive_expect_tx(bar, bytes);
                const uint8_t* src = a.x + (u / a.n_pieces) * a.row_bytes + int64_t(q) * a.piece_bytes;
                bulk_load(smem_u32(smem + size_t(s) * a.stage_bytes), src, bytes, bar, pol_load);
            } else {
                mbar_arrive(bar);
            }
        }
    };

    const int64_t prologue = my_n < S ? my_n : S;
    for (int64_t i = 0; i < prologue; ++i) issue(i, load_meta<NORMAL>(a, first + i * step, lane));
    UnitMeta next{-1, -1, -1, 0.f};  // routing of the next unit to refill: unit S, if this CTA has one
    if (int64_t(S) < my_n) next = load_meta<NORMAL>(a, first + int64_t(S) * step, lane);

    for (int64_t i = 0; i < my_n; ++i) {
        const int s = int(i % S);
        const uint32_t parity = uint32_t((i / S) & 1);
        const int64_t u = first + i * step;
        const int q = int(u % a.n_pieces);
        const bool landed = __all_sync(0xffffffffu, mbar_wait(smem_u32(full + s), parity));
        if (!landed) {
            if (lane == 0) flag_status(a.status, EP_STATUS_TIMEOUT);
            break;
        }
        const int2 m = meta[s * 32 + lane];
        if (m.x >= 0) {
            const int64_t tok = u / a.n_pieces;
            const int64_t slab_row = int64_t(m.x) * a.cap + m.y;
            bulk_store(a.recv_x + slab_row * a.row_bytes + int64_t(q) * a.piece_bytes,
                       smem_u32(smem + size_t(s) * a.stage_bytes), piece_size(a, q), pol_store);
            if (q == 0) {
                const int src_rank = int(tok / a.T);
                reinterpret_cast<int2*>(a.src_info)[slab_row] = make_int2(src_rank, int(tok - int64_t(src_rank) * a.T));
            }
        }
        if (NORMAL && q == 0) {
            // the received token's slots, in rank d's local expert ids (-1 / 0 for other ranks' slots)
            uint32_t dests = __ballot_sync(0xffffffffu, m.x >= 0);
            const int2 sl = slot[s * 32 + lane];
            while (dests) {
                const int d = __ffs(dests) - 1;
                dests &= dests - 1;
                const int row = __shfl_sync(0xffffffffu, m.y, d);
                if (lane < a.slots) {
                    const bool here = sl.x >= 0 && sl.x / a.slot_E_local == d;
                    const int64_t o = (int64_t(d) * a.cap + row) * a.slots + lane;
                    a.recv_topk_idx[o] = here ? sl.x - d * a.slot_E_local : -1;
                    a.recv_topk_weights[o] = here ? __int_as_float(sl.y) : 0.f;
                }
            }
        }
        bulk_commit();
        if (a.read_period_ns != 0) pace_reads(i);
        // refill the stage of unit i-1 with unit i-1+S once its stores have read it
        const int64_t refill = i - 1 + S;
        if (i >= 1 && refill < my_n) {
            bulk_wait_read<1>();
            __syncwarp();
            const UnitMeta cur = next;
            if (refill + 1 < my_n) next = load_meta<NORMAL>(a, first + (refill + 1) * step, lane);
            issue(refill, cur);
        }
    }
    bulk_wait<0>();
}

// ---------------------------------------------------------------------------
// Vector path (EP_VARIANT_VECTOR, k <= 8): every warp owns a contiguous,
// balanced range of units (token, piece of 32*U 16-byte columns).  At a token
// boundary lane j reads slot j's routing, writes the row's src_info, and the
// destination row pointers are broadcast with shuffles; then each lane loads
// its U columns of the token row once (L1 bypassed) and stores them to every
// live destination row.
constexpr int kVecKMax = 8;

template <int U>
__global__ void __launch_bounds__(256) dispatch_vec_kernel(DispatchArgs a) {
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int nvec = int(a.row_bytes >> 4);
    const int piece_vec = 32 * U;
    const int np = (nvec + piece_vec - 1) / piece_vec;
    const int64_t n_tok = a.n_units / a.n_pieces;
    const int64_t n_units = n_tok * np;
    const int64_t q = n_units / warps, rem = n_units % warps;
    const int64_t u0 = gw * q + (gw < rem ? gw : rem);
    const int64_t u1 = u0 + q + (gw < rem ? 1 : 0);

    int64_t cur_tok = -1;
    uint32_t mask = 0;
    uint8_t* dst[kVecKMax];
    for (int64_t u = u0; u < u1; ++u) {
        const int64_t tok = u / np;
        const int pc = int(u - tok * np);
        if (tok != cur_tok) {
            cur_tok = tok;
            int e = -1, row = -1;
            if (lane < a.k) {
                const int64_t p = tok * a.k + lane;
                e = __ldg(a.topk_idx + p);
                row = __ldg(a.pair_row + p);
            }
            const bool valid_row = row >= 0 && row < a.cap;
            const bool live = valid_row && e >= 0 && e < a.E;
            const int64_t slab_row = live ? int64_t(e) * a.cap + row : 0;
            if (lane < a.k && pc == 0) {
                if (row >= a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
                if (valid_row && !live) flag_status(a.status, EP_STATUS_BAD_EXPERT);
                if (live) {
                    const int src_rank = int(tok / a.T);
                    reinterpret_cast<int2*>(a.src_info)[slab_row] =
                        make_int2(src_rank, int(tok - int64_t(src_rank) * a.T));
                }
            }
            mask = __ballot_sync(0xffffffffu, live);
            const unsigned long long ptr =
                live ? reinterpret_cast<unsigned long long>(a.recv_x + slab_row * a.row_bytes) : 0ull;
#pragma unroll
            for (int j = 0; j < kVecKMax; ++j) dst[j] = reinterpret_cast<uint8_t*>(__shfl_sync(0xffffffffu, ptr, j));
        }
        if (mask == 0u) continue;
        const int v0 = pc * piece_vec + lane;
        const uint8_t* src = a.x + tok * a.row_bytes;
        uint4 xv[U];
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int v = v0 + 32 * uu;
            if (v < nvec) xv[uu] = ld_stream_v4(src + int64_t(v) * 16);
        }
#pragma unroll
        for (int j = 0; j < kVecKMax; ++j) {
            if (!((mask >> j) & 1u)) continue;
#pragma unroll
            for (int uu = 0; uu < U; ++uu) {
                const int v = v0 + 32 * uu;
                if (v < nvec) st_global_v4_stream(dst[j] + int64_t(v) * 16, xv[uu]);
            }
        }
    }
}

template <int U>
int launch_dispatch_vec(const DispatchArgs& a, const ep_cfg_t& cfg, int sms, cudaStream_t stream) {
    static std::atomic<int> per_sm[64];  // resident CTAs per SM, per device; 0 = not asked yet
    int dev = 0;
    cudaGetDevice(&dev);
    int occ = per_sm[dev & 63].load(std::memory_order_relaxed);
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, dispatch_vec_kernel<U>, 256, 0) != cudaSuccess)
            return EP_ERR_CUDA;
        per_sm[dev & 63].store(occ, std::memory_order_relaxed);
    }
    int64_t grid = int64_t(sms) * std::max(1, occ);
    if (cfg.max_ctas > 0) grid = std::min<int64_t>(grid, cfg.max_ctas);
    const int64_t units = (a.n_units / a.n_pieces) * ceil_div(a.row_bytes >> 4, 32 * U);
    grid = std::max<int64_t>(1, std::min<int64_t>(grid, ceil_div(units, 8)));
    if (launch_pdl(dispatch_vec_kernel<U>, dim3(unsigned(grid)), dim3(256), 0, stream, a) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

// Stage count from the shared-memory budget, then the bulk-path launch.
template <bool NORMAL, bool NOLOAD = false>
int launch_bulk_dispatch(DispatchArgs& a, const ep_cfg_t& cfg, int64_t grid, int budget, cudaStream_t stream) {
    const size_t per_stage = size_t(a.stage_bytes) + 8 + 2 * 256;
    int stages = cfg.stages > 0 ? cfg.stages : int(budget / per_stage);
    stages = std::max(2, std::min(kDispatchMaxStages, stages));
    a.stages = stages;
    const size_t smem = size_t(stages) * per_stage;
    if (smem > size_t(max_smem_optin())) return EP_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(dispatch_kernel<NORMAL, NOLOAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem)) != cudaSuccess)
        return EP_ERR_CUDA;
    if (launch_pdl(dispatch_kernel<NORMAL, NOLOAD>, dim3(unsigned(grid)), dim3(32), smem, stream, a) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

// The low-latency arguments of a (validated) ep_dispatch call.
int fill_dispatch_args(DispatchArgs& a, const ep_dims_t& d, const uint16_t* x, const int32_t* topk_idx,
                       const int32_t* pair_row, uint16_t* recv_x, int32_t* src_info, int32_t* status) {
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    a.x = reinterpret_cast<const uint8_t*>(x);
    a.topk_idx = topk_idx;
    a.pair_row = pair_row;
    a.recv_x = reinterpret_cast<uint8_t*>(recv_x);
    a.src_info = src_info;
    a.status = status;
    a.T = d.num_tokens;
    a.k = d.num_topk;
    a.E = d.num_experts;
    a.row_bytes = int64_t(d.hidden) * 2;
    a.cap = RT;
    a.slot_idx = nullptr;
    a.slot_w = nullptr;
    a.active = nullptr;
    a.recv_topk_idx = nullptr;
    a.recv_topk_weights = nullptr;
    a.slots = 0;
    a.slot_E = 0;
    a.slot_E_local = 1;
    a.n_pieces = int(ceil_div(a.row_bytes, kDispatchPieceMax));
    a.piece_bytes = uint32_t(round_up16(size_t(ceil_div(a.row_bytes, a.n_pieces))));
    if (int64_t(a.n_pieces - 1) * a.piece_bytes >= a.row_bytes) return EP_ERR_UNSUPPORTED;
    a.stage_bytes = uint32_t((a.piece_bytes + 127) & ~127u);
    a.n_units = RT * a.n_pieces;
    a.read_period_ns = 0;
    a.read_window_ns = 0;
    a.read_ahead = 0;
    return EP_OK;
}

// AUTO's choice for a low-latency dispatch (see kPaceMinStoreBytesPerRow).
bool paced_by_default(const DispatchArgs& a, int sms) {
    const int64_t stores = int64_t(a.k) * a.row_bytes;
    const int64_t min_units = stores >= kPaceOneRingStoreBytesPerRow ? kPaceMinUnitsPerCta : kPaceTwoRingMinUnitsPerSm;
    return a.n_pieces == 1 && stores >= kPaceMinStoreBytesPerRow && a.n_units >= min_units * sms;
}

// CTAs per SM of a paced dispatch: one deep ring where a row's stores add up to >= 96 KB, else two.
int paced_ctas_per_sm(const DispatchArgs& a) {
    return int64_t(a.k) * a.row_bytes >= kPaceOneRingStoreBytesPerRow ? 1 : 2;
}

// CTAs per SM of an unpaced normal-mode dispatch (see kNormalWideCtasPerSm).
int normal_ctas_per_sm(const DispatchArgs& a, int sms) {
    const int64_t per_stage = int64_t(a.stage_bytes) + 8 + 2 * 256;
    const int64_t budget = max_smem_optin() / kNormalWideCtasPerSm - 1024;
    const bool deep = budget >= kNormalWideMinStages * per_stage;
    const bool few = a.n_units <= int64_t(kNormalWideMaxUnitsPerSm) * sms;
    return deep || few ? kNormalWideCtasPerSm : 2;
}

// Grid, stages and (for the paced path) the read schedule, then the bulk-path launch.  `prefetch`
// (default: as paced) turns the paced read schedule on; the ceiling diagnostic may turn it off.
// `unpaced_per_sm` is the default CTAs per SM without paced reads.
template <bool NORMAL, bool NOLOAD = false>
int run_bulk_dispatch(DispatchArgs& a, const ep_cfg_t& cfg, bool paced, int sms, cudaStream_t stream,
                      int prefetch = -1, int unpaced_per_sm = 2) {
    // default grid: `unpaced_per_sm` CTAs per SM, or with paced reads 1 (one deep ring per SM) or 2
    // (shorter rows, see paced_ctas_per_sm); cfg.max_ctas sets the grid (and so the CTAs sharing an SM)
    int64_t grid = cfg.max_ctas > 0 ? int64_t(cfg.max_ctas)
                                    : int64_t(sms) * (paced ? paced_ctas_per_sm(a) : unpaced_per_sm);
    grid = std::max<int64_t>(1, std::min<int64_t>(grid, a.n_units));
    const int ctas_per_sm = int(std::max<int64_t>(1, ceil_div(grid, sms)));
    int budget = std::max(1, max_smem_optin() / ctas_per_sm - 1024);
    if (paced && prefetch != 0) {
        a.read_period_ns = kPacePeriodNs;
        a.read_window_ns = kPaceWindowNs;
        a.read_ahead = int(std::max<int64_t>(1, kPaceAheadBytes / std::max<int64_t>(1, a.stage_bytes)));
    }
    if (paced) {
        // the ring of the measured schedule: 14 stages (fewer if the budget is smaller)
        if (cfg.stages <= 0) budget = std::min(budget, 14 * int(a.stage_bytes + 8 + 2 * 256));
    }
    return launch_bulk_dispatch<NORMAL, NOLOAD>(a, cfg, grid, budget, stream);
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" int ep_dispatch(ep_dims_t d, const uint16_t* x, const int32_t* topk_idx, const int32_t* pair_row,
                           uint16_t* recv_x, int32_t* src_info, int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_dispatch");
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (RT == 0 || d.hidden == 0) return EP_OK;
    if (!x || !topk_idx || !pair_row || !recv_x || !src_info) return EP_ERR_INVALID;
    if (!aligned16(x) || !aligned16(recv_x) || (reinterpret_cast<uintptr_t>(src_info) & 7u)) return EP_ERR_INVALID;

    const int requested = cfg.variant;
    if (requested != EP_VARIANT_AUTO && requested != EP_VARIANT_BULK && requested != EP_VARIANT_VECTOR &&
        requested != EP_VARIANT_PACED)
        return EP_ERR_INVALID;
    if (requested == EP_VARIANT_VECTOR && d.num_topk > kVecKMax) return EP_ERR_UNSUPPORTED;

    DispatchArgs a;
    rc = fill_dispatch_args(a, d, x, topk_idx, pair_row, recv_x, src_info, status);
    if (rc != EP_OK) return rc;

    const int sms = sm_count();
    if (sms <= 0) return EP_ERR_CUDA;
    const int variant = requested != EP_VARIANT_AUTO ? requested
                        : (paced_by_default(a, sms) ? EP_VARIANT_PACED : EP_VARIANT_BULK);
    if (variant == EP_VARIANT_VECTOR) {
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        switch (cfg.threads) {
            case 1: return launch_dispatch_vec<1>(a, cfg, sms, st);
            case 2: return launch_dispatch_vec<2>(a, cfg, sms, st);
            default: return launch_dispatch_vec<4>(a, cfg, sms, st);
        }
    }
    return run_bulk_dispatch<false>(a, cfg, variant == EP_VARIANT_PACED, sms, static_cast<cudaStream_t>(stream));
}

extern "C" int ep_normal_dispatch(ep_dims_t d, int32_t recv_capacity, const uint16_t* x, const int32_t* topk_idx,
                                  const float* topk_weights, const uint8_t* active, const int32_t* token_recv_row,
                                  uint16_t* recv_x, int32_t* recv_topk_idx, float* recv_topk_weights,
                                  int32_t* src_info, int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_normal_dispatch");
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    if (recv_capacity < 0) return EP_ERR_INVALID;
    if (d.num_ranks > EP_MAX_NORMAL_RANKS) return EP_ERR_UNSUPPORTED;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (RT == 0) return EP_OK;
    if (!x || !topk_idx || !topk_weights || !active || !token_recv_row) return EP_ERR_INVALID;
    if (recv_capacity > 0 && (!recv_x || !recv_topk_idx || !recv_topk_weights || !src_info)) return EP_ERR_INVALID;
    if (!aligned16(x) || (recv_x && !aligned16(recv_x)) || (reinterpret_cast<uintptr_t>(src_info) & 7u))
        return EP_ERR_INVALID;
    // lanes are the destination ranks: slab d of recv_x is rank d's receive buffer
    DispatchArgs a;
    a.x = reinterpret_cast<const uint8_t*>(x);
    a.topk_idx = nullptr;
    a.pair_row = token_recv_row;
    a.recv_x = reinterpret_cast<uint8_t*>(recv_x);
    a.src_info = src_info;
    a.status = status;
    a.T = d.num_tokens;
    a.k = d.num_ranks;
    a.E = d.num_ranks;
    a.row_bytes = int64_t(d.hidden) * 2;
    a.cap = recv_capacity;
    a.slot_idx = topk_idx;
    a.slot_w = topk_weights;
    a.active = active;
    a.recv_topk_idx = recv_topk_idx;
    a.recv_topk_weights = recv_topk_weights;
    a.slots = d.num_topk;
    a.slot_E = d.num_experts;
    a.slot_E_local = d.num_experts / d.num_ranks;
    a.n_pieces = int(ceil_div(a.row_bytes, kDispatchPieceMax));
    a.piece_bytes = uint32_t(round_up16(size_t(ceil_div(a.row_bytes, a.n_pieces))));
    if (int64_t(a.n_pieces - 1) * a.piece_bytes >= a.row_bytes) return EP_ERR_UNSUPPORTED;
    a.stage_bytes = uint32_t((a.piece_bytes + 127) & ~127u);
    a.n_units = RT * a.n_pieces;
    a.read_period_ns = 0;
    a.read_window_ns = 0;
    a.read_ahead = 0;
    const int sms = sm_count();
    if (sms <= 0) return EP_ERR_CUDA;
    // normal mode has only the bulk data path: PACED paces its reads (it measured slower at prefill,
    // so AUTO does not), any other variant runs it unpaced
    const bool paced = cfg.variant == EP_VARIANT_PACED;
    return run_bulk_dispatch<true>(a, cfg, paced, sms, static_cast<cudaStream_t>(stream), -1,
                                   normal_ctas_per_sm(a, sms));
}

extern "C" int ep_diag_dispatch_ceiling(ep_dims_t d, const uint16_t* x, const int32_t* topk_idx,
                                        const int32_t* pair_row, uint16_t* recv_x, int32_t* src_info, int32_t mode,
                                        int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_diag_dispatch_ceiling");
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    if (mode != 0 && mode != 1) return EP_ERR_INVALID;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (RT == 0 || d.hidden == 0) return EP_OK;
    if (!x || !topk_idx || !pair_row || !recv_x || !src_info) return EP_ERR_INVALID;
    if (!aligned16(x) || !aligned16(recv_x) || (reinterpret_cast<uintptr_t>(src_info) & 7u)) return EP_ERR_INVALID;
    DispatchArgs a;
    rc = fill_dispatch_args(a, d, x, topk_idx, pair_row, recv_x, src_info, status);
    if (rc != EP_OK) return rc;
    const int sms = sm_count();
    if (sms <= 0) return EP_ERR_CUDA;
    // the paced path's grid and ring, its L2 prefetch schedule in mode 1
    return run_bulk_dispatch<false, true>(a, cfg, true, sms, static_cast<cudaStream_t>(stream), mode);
}

extern "C" int ep_dispatch_path(ep_dims_t d, ep_cfg_t cfg) {
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    if (cfg.variant != EP_VARIANT_AUTO && cfg.variant != EP_VARIANT_BULK && cfg.variant != EP_VARIANT_VECTOR &&
        cfg.variant != EP_VARIANT_PACED)
        return EP_ERR_INVALID;
    if (cfg.variant == EP_VARIANT_VECTOR && d.num_topk > kVecKMax) return EP_ERR_UNSUPPORTED;
    if (cfg.variant != EP_VARIANT_AUTO) return cfg.variant;
    DispatchArgs a;
    rc = fill_dispatch_args(a, d, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
    if (rc != EP_OK) return rc;
    const int sms = sm_count();
    if (sms <= 0) return EP_ERR_CUDA;
    return paced_by_default(a, sms) ? EP_VARIANT_PACED : EP_VARIANT_BULK;
}
