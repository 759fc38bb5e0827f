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
// Four paths compute the same result (ep_cfg_t.variant selects one; AUTO takes
// the single CTA up to 2048 pairs, the cluster up to 65536, the chunked path
// beyond: the fastest on B200 in each range).  All sort with the same two ideas:
// lanes holding the same expert are merged (a match mask built from one warp
// ballot per expert-id bit) so one leader updates the group's count (a
// warp-aggregated update), and a pair's row inside a run of 32 consecutive
// pairs is its running count plus its rank among equal experts to its left
// (popc of the match mask below it).  Destination ranks come from a shared
// table rank_of[e] (-1 when that rank is masked), so no pair test divides.
//
// Single-CTA path (EP_LAYOUT_SINGLE_CTA; R <= 32, E <= 1024, <= 32768 pairs):
// one 1024-thread CTA, one launch, no workspace.  Each rank's tokens are split
// among 32/R warps in (rank, token) order; every warp walks its part once,
// finding each pair's row within the part and each token's destination ranks;
// the CTA scans the warp histograms per expert (which also yields
// expert_rank_offset, num_tokens_per_expert, recv_count) and the pairs add
// their warp's first row.
//
// Cluster path (EP_LAYOUT_CLUSTER; R <= 32, E <= 1024, <= 65536 pairs): the
// same over a thread-block cluster of 2 to 16 CTAs whose shared memories see
// one another; a CTA's first rows come from the other CTAs' totals, read
// through distributed shared memory after a cluster barrier.
//
// Fused path (EP_LAYOUT_FUSED): the chunked path below in one cooperative
// launch with two bounded grid barriers.
//
// Chunked path (EP_LAYOUT_CHUNKED; any shape): each rank's tokens are cut into
// C contiguous chunks (chunk g = r*C + c, ordered like the sort key; about a
// hundred chunks in all) over three launches:
//   1. count -- one CTA per chunk builds the chunk's expert histogram with
//               warp-aggregated shared atomics, each token's destination-rank
//               set (is_token_in_rank) and the chunk's per-destination token
//               counts, into the workspace;
//   2. scan  -- one CTA per 32 experts (lane <-> expert, warps <-> runs of
//               chunks, values held in registers) turns every chunk count into
//               the chunk's first row (exclusive scan over (rank, chunk)), in
//               place, and writes expert_rank_offset, num_tokens_per_expert,
//               recv_count; warps also reduce num_tokens_per_rank;
//   3. rank  -- one CTA per chunk splits it among its warps, counts each
//               warp's part into a warp-private histogram, scans those over
//               warps on top of the chunk's first rows, and assigns rows.
// Every step is deterministic: rows are unique and identical run to run.
#include <algorithm>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr int kTargetChunks = 32;    // chunks over all ranks at least
constexpr int kPairsPerChunk = 2048;  // aim for this many pairs per chunk
constexpr int kMaxChunks = 148;       // G <= kMaxChunks + R - 1 <= 32 * kScanRowsPerWarp
constexpr int kScanWarps = 32;
constexpr int kScanRowsPerWarp = 8;
constexpr int kSmallThreads = 1024;
constexpr int kSmallMaxPairs = 32768;
constexpr int kSmallMaxExperts = 1024;
constexpr int kSmallMaxRanks = 32;
constexpr int kSmallAutoPairs = 2048;  // AUTO takes the single-CTA path up to here
constexpr int kClusterMaxCtas = 16;     // a non-portable cluster size (8 is the portable limit)
constexpr int kClusterPairsPerCta = 1024;
constexpr int64_t kClusterMaxPairs = 65536;
constexpr int64_t kClusterAutoPairs = 65536;  // AUTO takes the cluster path up to here
constexpr int kMaxWarps = 16;
constexpr int kBatch = 8;           // 32-pair steps whose loads are issued together
constexpr int kActiveSlots = 64;    // shared copy of the active mask (EP_MAX_RANKS)
constexpr int kMaxFlags = 255;      // >= kMaxChunks + EP_MAX_RANKS - 1
constexpr int kFlagsPerLane = (kMaxFlags + 31) / 32;  // flags one lane of the look-back wait polls
constexpr int kSumChunks = 8;  // chunk histograms a look-back warp loads at once (x 2 columns per lane)
// Look-back flags sit kLookbackFlagWords words apart, one per 256 bytes: every CTA polls the
// flags of the chunks before it, and packed into a few lines those polls queue behind each other.
// (Fused-path flags are the first kMaxFlags words after the epoch; every flag word only ever holds
// values of past epochs, below the current one, so the two paths can share the region.)
constexpr int kLookbackFlagWords = 32;
// epoch + flags, at offset 0 of the workspace; what follows starts on a 256-byte boundary
constexpr size_t kSyncBytes = (size_t(1 + kMaxFlags * kLookbackFlagWords) * 8 + 255) / 256 * 256;
static_assert(kSyncBytes % 16 == 0, "the chunk histograms after the flags are read 16 bytes at a time");

struct LayoutArgs {
    const int32_t* topk_idx;
    const uint8_t* active;
    int32_t* chunk_hist;  // workspace [G][E]
    int32_t* chunk_tpr;   // workspace [G][R]: tokens of the chunk per destination rank
    uint64_t* sync;       // workspace prefix: epoch, then one barrier flag per chunk (fused path)
    int32_t* num_tokens_per_expert;
    int32_t* num_tokens_per_rank;
    uint8_t* is_token_in_rank;
    int32_t* recv_count;
    int32_t* expert_rank_offset;
    int32_t* pair_row;
    int32_t* status;
    int R, T, k, E, E_local;  // R: ranks of the EP world (mask, destinations, is_token_in_rank width)
    int Rs, r0;        // source ranks laid out (rows of topk_idx), the first one's rank: R and 0 for
                       // the whole world, 1 and the caller's rank for a rank-local layout
    int key_bits;      // bits that tell experts apart: ceil(log2(E))
    int C, G;          // chunks per rank, chunks
    int chunk_tokens;  // tokens per chunk (the last chunk of a rank may be shorter)
    int64_t cap;
};

struct ChunkGeom {
    int r, t0, t1;
};

__device__ __forceinline__ ChunkGeom chunk_of(const LayoutArgs& a, int g) {
    ChunkGeom c;
    c.r = g / a.C;
    c.t0 = min(a.T, (g - c.r * a.C) * a.chunk_tokens);
    c.t1 = min(a.T, c.t0 + a.chunk_tokens);
    return c;
}

// act[] <- active mask, rank_of[e] <- destination rank of e, or -1 if it is masked.
// act[] is indexed by world rank; source row r is rank r0 + r.
__device__ __forceinline__ void load_tables(const LayoutArgs& a, int32_t* act, int32_t* rank_of) {
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) act[i] = a.active[i];
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        const int d = e / a.E_local;
        rank_of[e] = a.active[d] ? d : -1;
    }
}

__device__ __forceinline__ bool pair_live(int e, int E, bool src_ok, const int32_t* rank_of) {
    return src_ok && e >= 0 && e < E && rank_of[e] >= 0;
}

__global__ void __launch_bounds__(32 * kMaxWarps) layout_count_kernel(LayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t smem[];
    int32_t* act = smem;
    int32_t* tpr = smem + kActiveSlots;
    int32_t* rank_of = smem + 2 * kActiveSlots;
    int32_t* hist = rank_of + a.E;
    load_tables(a, act, rank_of);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
    for (int d = threadIdx.x; d < a.R; d += blockDim.x) tpr[d] = 0;
    __syncthreads();

    const ChunkGeom cg = chunk_of(a, blockIdx.x);
    const bool src_ok = act[a.r0 + cg.r] != 0;
    const int64_t pbase = (int64_t(cg.r) * a.T + cg.t0) * a.k;
    const int32_t* base = a.topk_idx + pbase;
    const int np = (cg.t1 - cg.t0) * a.k;

    bool bad = false;
    const int stride = blockDim.x * kBatch;
    for (int p0 = (threadIdx.x & ~31) * kBatch; p0 < np; p0 += stride) {
        int ev[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int p = p0 + u * 32 + (threadIdx.x & 31);
            ev[u] = p < np ? __ldg(base + p) : -1;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int e = ev[u];
            bad |= (e < -1 || e >= a.E);
            const bool live = pair_live(e, a.E, src_ok, rank_of);
            const uint32_t m = match_key(uint32_t(e), a.key_bits, __ballot_sync(0xffffffffu, live));
            if (live && (threadIdx.x & 31) == __ffs(m) - 1) atomicAdd(hist + e, __popc(m));
        }
    }

    // destination-rank set of each token (thread <-> token)
    const int lane = threadIdx.x & 31;
    for (int t0 = cg.t0 + (threadIdx.x & ~31); t0 < cg.t1; t0 += blockDim.x) {
        const int t = t0 + lane;
        uint64_t ranks = 0;
        if (t < cg.t1) {
            const int32_t* tb = a.topk_idx + (int64_t(cg.r) * a.T + t) * a.k;
            for (int j = 0; j < a.k; ++j) {
                const int e = __ldg(tb + j);
                if (pair_live(e, a.E, src_ok, rank_of)) ranks |= 1ull << rank_of[e];
            }
            uint8_t* itr = a.is_token_in_rank + (int64_t(cg.r) * a.T + t) * a.R;
            for (int d = 0; d < a.R; ++d) itr[d] = uint8_t((ranks >> d) & 1u);
        }
        for (int d = 0; d < a.R; ++d) {
            const int n = __popc(__ballot_sync(0xffffffffu, (ranks >> d) & 1u));
            if (lane == 0 && n) atomicAdd(tpr + d, n);
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);
    int32_t* out = a.chunk_hist + int64_t(blockIdx.x) * a.E;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) out[e] = hist[e];
    for (int d = threadIdx.x; d < a.R; d += blockDim.x) a.chunk_tpr[int64_t(blockIdx.x) * a.R + d] = tpr[d];
}

// One CTA per 32 experts; warp w holds chunk rows [w*rpw, (w+1)*rpw) in registers.
__global__ void __launch_bounds__(32 * kScanWarps) layout_scan_kernel(LayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    __shared__ int32_t seg[kScanWarps][32];
    __shared__ int32_t total[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 32 + lane;
    const bool ok = e < a.E;
    const int rpw = (a.G + kScanWarps - 1) / kScanWarps;
    const int g0 = warp * rpw;
    int32_t v[kScanRowsPerWarp];
    int32_t s = 0;
#pragma unroll
    for (int i = 0; i < kScanRowsPerWarp; ++i) {
        const int g = g0 + i;
        v[i] = (ok && i < rpw && g < a.G) ? a.chunk_hist[int64_t(g) * a.E + e] : 0;
        s += v[i];
    }
    seg[warp][lane] = s;
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int w = 0; w < kScanWarps; ++w) {
            const int32_t t = seg[w][lane];
            seg[w][lane] = run;
            run += t;
        }
        total[lane] = run;
        if (ok) {
            a.recv_count[e] = run;
            if (run > a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
        }
    }
    __syncthreads();
    int32_t run = seg[warp][lane];
#pragma unroll
    for (int i = 0; i < kScanRowsPerWarp; ++i) {
        const int g = g0 + i;
        if (ok && i < rpw && g < a.G) a.chunk_hist[int64_t(g) * a.E + e] = run;
        run += v[i];
    }
    __syncthreads();
    if (ok) {
        for (int r = warp; r < a.Rs; r += kScanWarps) {
            const int32_t off = a.chunk_hist[int64_t(r) * a.C * a.E + e];
            const int32_t next = r + 1 < a.Rs ? a.chunk_hist[int64_t(r + 1) * a.C * a.E + e] : total[lane];
            a.expert_rank_offset[int64_t(e) * a.Rs + r] = off;
            a.num_tokens_per_expert[int64_t(r) * a.E + e] = next - off;
        }
    }
    const int RR = a.Rs * a.R;
    for (int pr = blockIdx.x * kScanWarps + warp; pr < RR; pr += gridDim.x * kScanWarps) {
        const int r = pr / a.R, d = pr - r * a.R;
        const int32_t* col = a.chunk_tpr + int64_t(r) * a.C * a.R + d;
        int32_t t = 0;
        for (int c = lane; c < a.C; c += 32) t += col[int64_t(c) * a.R];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
        if (lane == 0) a.num_tokens_per_rank[pr] = t;
    }
}

// ---------------------------------------------------------------------------
// One-launch paths (single CTA, cluster).  Their warps -- 32 per CTA, a cluster's
// numbered CTA * 32 + warp -- split each rank's tokens into consecutive parts in
// (rank, part) order, and each warp walks its part once.

// A warp's part of the tokens: rank r, tokens [t0, t1), pairs from pbase on.
struct WarpPart {
    int r, t0, t1;
    int64_t pbase;
    int np;          // pairs of the part
    bool has_rank;   // warps past the last rank have no part
    bool one_round;  // np <= 32 * kBatch: the rows within the part stay in registers
};

__device__ __forceinline__ WarpPart warp_part(const LayoutArgs& a, int gw, int wpr) {
    WarpPart w;
    w.r = gw / wpr;
    const int part = gw - w.r * wpr;
    w.has_rank = w.r < a.Rs;
    const int tw = (a.T + wpr - 1) / wpr;
    w.t0 = w.has_rank ? min(a.T, part * tw) : 0;
    w.t1 = w.has_rank ? min(a.T, w.t0 + tw) : 0;
    w.pbase = w.has_rank ? (int64_t(w.r) * a.T + w.t0) * a.k : 0;
    w.np = (w.t1 - w.t0) * a.k;
    w.one_round = w.np <= 32 * kBatch;
    return w;
}

// The part's first round of experts; it needs no table, so it is loaded before
// the barrier that publishes them.
__device__ __forceinline__ void load_first_round(const LayoutArgs& a, const WarpPart& w, int (&ev)[kBatch]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
        const int p = u * 32 + lane;
        ev[u] = p < w.np ? __ldg(a.topk_idx + w.pbase + p) : -1;
    }
}

// A token's destination-rank set (bit d = rank d, d < 8) spread to one byte per
// rank: bytes 0-3 in the low word, 4-7 in the high word, each 0 or 1.
__device__ __forceinline__ uint32_t rank_bytes_lo(uint32_t dst) { return ((dst & 0xFu) * 0x00204081u) & 0x01010101u; }
__device__ __forceinline__ uint32_t rank_bytes_hi(uint32_t dst) {
    return (((dst >> 4) & 0xFu) * 0x00204081u) & 0x01010101u;
}

// Adds a warp's per-lane byte counters of destination ranks (one byte per rank,
// ranks 0-3 in lo, 4-7 in hi) to tpr_row[0..R).  Widened to 16-bit fields before
// the warp sum: a lane counts at most kBatch tokens between two calls.
__device__ __forceinline__ void flush_rank_counts(uint32_t lo, uint32_t hi, int R, int32_t* tpr_row) {
    const int lane = threadIdx.x & 31;
    const uint32_t w0 = __reduce_add_sync(0xffffffffu, __byte_perm(lo, 0, 0x4140));  // ranks 0, 1
    const uint32_t w1 = __reduce_add_sync(0xffffffffu, __byte_perm(lo, 0, 0x4342));  // ranks 2, 3
    const uint32_t w2 = __reduce_add_sync(0xffffffffu, __byte_perm(hi, 0, 0x4140));  // ranks 4, 5
    const uint32_t w3 = __reduce_add_sync(0xffffffffu, __byte_perm(hi, 0, 0x4342));  // ranks 6, 7
    if (lane < R) {
        const uint32_t wv = lane < 2 ? w0 : lane < 4 ? w1 : lane < 6 ? w2 : w3;
        const int n = int((lane & 1) ? (wv >> 16) : (wv & 0xFFFFu));
        if (n) atomicAdd(tpr_row + lane, n);
    }
}

// One pass over the part.  A pair's row within the part is its expert's running
// count in the warp's histogram `mine` plus the matching lanes below it (ballot
// match); it stays in rk (the last round's pairs) or, for a part longer than one
// round, is parked in pair_row.  Each token's destination ranks go to
// is_token_in_rank and its counts to tpr_row[*] (the part's source rank's row of
// per-destination token counts): with k a power of two a token's
// k slots sit in k aligned lanes and an OR over them gives the set, otherwise one
// token per lane re-reads its slots.  True if this lane saw an id outside [-1, E).
//
// The kernels that call this run it once per launch, so the 32-pair steps are a
// rolled loop over one copy of the body (an unrolled copy per step runs from a
// cold instruction cache): step u takes ev[0] and rotates ev/rk by one, which
// after kBatch steps leaves both in their original order.  With R <= 8 a token's
// ranks are written as one word of bytes and counted in per-lane byte counters,
// summed over the warp once per round.
__device__ __forceinline__ bool walk_part(const LayoutArgs& a, const WarpPart& w, const int32_t* act,
                                          const int32_t* rank_of, int32_t* mine, int32_t* tpr_row,
                                          int (&ev)[kBatch], int (&rk)[kBatch]) {
    const int lane = threadIdx.x & 31;
    const bool src_ok = w.has_rank && act[a.r0 + w.r] != 0;
    const int32_t* base = a.topk_idx + w.pbase;
    int32_t* rows = a.pair_row + w.pbase;
    const uint32_t below = lanemask_lt();
    const bool lanes_per_token = (a.k & (a.k - 1)) == 0;  // k divides 32: a token is k aligned lanes
    const bool packed = lanes_per_token && a.R <= 8;
    // a token's row of is_token_in_rank as one store when R is 8 (or 4) and the buffer allows it
    const uintptr_t itr_base = reinterpret_cast<uintptr_t>(a.is_token_in_rank);
    const int itr_word = (a.R == 8 && (itr_base & 7u) == 0) ? 8 : (a.R == 4 && (itr_base & 3u) == 0) ? 4 : 0;
    bool bad = false;
    for (int p0 = 0; p0 < w.np; p0 += 32 * kBatch) {
        if (p0 > 0) {
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int p = p0 + u * 32 + lane;
                ev[u] = p < w.np ? __ldg(base + p) : -1;
            }
        }
        uint32_t cnt_lo = 0, cnt_hi = 0;
#pragma unroll 1
        for (int u = 0; u < kBatch; ++u) {
            const int e = ev[0];
            int r = -1;
            if (p0 + u * 32 < w.np) {  // the same for the whole warp
                const int p = p0 + u * 32 + lane;
                bad |= (e < -1 || e >= a.E);
                const bool live = pair_live(e, a.E, src_ok, rank_of);
                const uint32_t m = match_key(uint32_t(e), a.key_bits, __ballot_sync(0xffffffffu, live));
                const int32_t b = live ? mine[e] : 0;
                __syncwarp();
                if (live && lane == __ffs(m) - 1) mine[e] = b + __popc(m);
                __syncwarp();
                r = live ? b + __popc(m & below) : -1;
                if (!w.one_round && p < w.np) rows[p] = r;
                if (lanes_per_token) {
                    const bool head = p < w.np && (lane & (a.k - 1)) == 0;
                    uint8_t* itr = a.is_token_in_rank + ((w.pbase + p) / a.k) * a.R;
                    if (packed) {
                        // the token's destination ranks (R <= 8: one word)
                        uint32_t dst = live ? (1u << rank_of[e]) : 0u;
                        for (int o = 1; o < a.k; o <<= 1) dst |= __shfl_xor_sync(0xffffffffu, dst, o);
                        const uint32_t lo = rank_bytes_lo(dst), hi = rank_bytes_hi(dst);
                        if (head) {
                            if (itr_word == 8) {
                                *reinterpret_cast<uint2*>(itr) = make_uint2(lo, hi);
                            } else if (itr_word == 4) {
                                *reinterpret_cast<uint32_t*>(itr) = lo;
                            } else {
                                for (int d = 0; d < a.R; ++d) itr[d] = uint8_t((dst >> d) & 1u);
                            }
                            cnt_lo += lo;
                            cnt_hi += hi;
                        }
                    } else {
                        // the token's destination ranks: 64 bits, since R may reach EP_MAX_RANKS
                        uint64_t dst = live ? (1ull << rank_of[e]) : 0ull;
                        for (int o = 1; o < a.k; o <<= 1) dst |= __shfl_xor_sync(0xffffffffu, dst, o);
                        if (head)
                            for (int d = 0; d < a.R; ++d) itr[d] = uint8_t((dst >> d) & 1u);
                        for (int d = 0; d < a.R; ++d) {
                            const int n = __popc(__ballot_sync(0xffffffffu, head && ((dst >> d) & 1u)));
                            if (lane == 0 && n) atomicAdd(tpr_row + d, n);
                        }
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kBatch - 1; ++i) {
                ev[i] = ev[i + 1];
                rk[i] = rk[i + 1];
            }
            ev[kBatch - 1] = e;
            rk[kBatch - 1] = r;
        }
        if (packed) flush_rank_counts(cnt_lo, cnt_hi, a.R, tpr_row);
    }
    if (!lanes_per_token) {
        for (int t0 = w.t0; t0 < w.t1; t0 += 32) {
            const int t = t0 + lane;
            uint64_t ranks = 0;
            if (t < w.t1) {
                const int32_t* tb = a.topk_idx + (int64_t(w.r) * a.T + t) * a.k;
                for (int j = 0; j < a.k; ++j) {
                    const int e = __ldg(tb + j);
                    if (pair_live(e, a.E, src_ok, rank_of)) ranks |= 1ull << rank_of[e];
                }
                uint8_t* itr = a.is_token_in_rank + (int64_t(w.r) * a.T + t) * a.R;
                for (int d = 0; d < a.R; ++d) itr[d] = uint8_t((ranks >> d) & 1u);
            }
            for (int d = 0; d < a.R; ++d) {
                const int n = __popc(__ballot_sync(0xffffffffu, (ranks >> d) & 1u));
                if (lane == 0 && n) atomicAdd(tpr_row + d, n);
            }
        }
    }
    return bad;
}

// Each live pair's row: first_row(e), the part's first row for its expert, plus
// its row within the part.
template <typename FirstRow>
__device__ __forceinline__ void finish_rows(const LayoutArgs& a, const WarpPart& w, const int (&ev)[kBatch],
                                            const int (&rk)[kBatch], FirstRow first_row) {
    const int lane = threadIdx.x & 31;
    int32_t* rows = a.pair_row + w.pbase;
    if (w.one_round) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int p = u * 32 + lane;
            if (u * 32 >= w.np) break;
            if (p < w.np) rows[p] = rk[u] >= 0 ? first_row(ev[u]) + rk[u] : -1;
        }
    } else {
        for (int p = lane; p < w.np; p += 32) {
            const int32_t q = rows[p];  // written by this thread in walk_part
            if (q >= 0) rows[p] = first_row(__ldg(a.topk_idx + w.pbase + p)) + q;
        }
    }
}

// Single CTA: the whole layout in one launch (small problems).  After the walk,
// the warp histograms are scanned per expert in warp (= (rank, part)) order into
// each warp's first row, which the pairs add.
__global__ void __launch_bounds__(kSmallThreads) layout_single_cta_kernel(LayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t smem[];
    constexpr int NW = kSmallThreads / 32;
    const int warp = threadIdx.x >> 5;
    int32_t* act = smem;
    int32_t* tpr = smem + kActiveSlots;                        // [R][R]
    int32_t* rank_of = tpr + kSmallMaxRanks * kSmallMaxRanks;   // [E]
    int32_t* whist = rank_of + a.E;                            // [NW][E]

    const int wpr = NW / a.Rs;  // warps per source rank, Rs <= 32
    const WarpPart w = warp_part(a, warp, wpr);
    int ev[kBatch], rk[kBatch];
    load_first_round(a, w, ev);
    load_tables(a, act, rank_of);
    for (int i = threadIdx.x; i < NW * a.E; i += blockDim.x) whist[i] = 0;
    for (int i = threadIdx.x; i < a.Rs * a.R; i += blockDim.x) tpr[i] = 0;
    __syncthreads();

    int32_t* mine = whist + warp * a.E;
    const bool bad = walk_part(a, w, act, rank_of, mine, tpr + (w.has_rank ? w.r * a.R : 0), ev, rk);
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);

    // scan the warp histograms per expert in warp order = (rank, part) order
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int32_t run = 0;
        for (int rr = 0; rr < a.Rs; ++rr) {
            const int32_t rank_first = run;
            a.expert_rank_offset[int64_t(e) * a.Rs + rr] = rank_first;
            for (int wi = rr * wpr; wi < (rr + 1) * wpr; ++wi) {
                const int32_t c = whist[wi * a.E + e];
                whist[wi * a.E + e] = run;
                run += c;
            }
            a.num_tokens_per_expert[int64_t(rr) * a.E + e] = run - rank_first;
        }
        a.recv_count[e] = run;
        if (run > a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
    }
    for (int i = threadIdx.x; i < a.Rs * a.R; i += blockDim.x) a.num_tokens_per_rank[i] = tpr[i];
    __syncthreads();
    finish_rows(a, w, ev, rk, [&](int e) { return mine[e]; });
}

// Cluster path (EP_LAYOUT_CLUSTER): the single-CTA algorithm over a thread-block
// cluster of CL CTAs, one per SM, whose shared memories are reachable from one
// another:
//  1. each warp walks its part into its CTA's shared memory;
//  2. each CTA scans its own warps' histograms per expert and keeps its totals;
//     after a cluster barrier, its first row per expert is the sum of the totals
//     of the CTAs before it, read from their shared memory; the CTA holding a
//     rank's first warp writes that rank's expert_rank_offset, the last CTA
//     recv_count, CTA 0 the sum of every CTA's num_tokens_per_rank;
//  3. each live pair's row is its CTA's first row + its warp's first row within
//     the CTA + its row within the part;
//  4. after a second cluster barrier (no shared memory is read across CTAs
//     past it), the rank owners take num_tokens_per_expert from neighbouring
//     offsets.
__global__ void __launch_bounds__(kSmallThreads) layout_cluster_kernel(LayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t smem[];
    constexpr int NW = kSmallThreads / 32;
    const int warp = threadIdx.x >> 5;
    const int cta = int(cluster_ctarank()), CL = int(cluster_nctarank());
    int32_t* act = smem;
    int32_t* tpr = smem + kActiveSlots;                        // [R][R], this CTA's tokens
    int32_t* rank_of = tpr + kSmallMaxRanks * kSmallMaxRanks;   // [E]
    int32_t* ctot = rank_of + a.E;                             // [E] this CTA's live pairs per expert
    int32_t* cbase = ctot + a.E;                               // [E] this CTA's first row per expert
    int32_t* whist = cbase + a.E;                              // [NW][E]

    const int wpr = CL * NW / a.Rs;  // warps per source rank, Rs <= 32 <= CL * NW
    const WarpPart w = warp_part(a, cta * NW + warp, wpr);
    int ev[kBatch], rk[kBatch];
    load_first_round(a, w, ev);
    load_tables(a, act, rank_of);
    for (int i = threadIdx.x; i < NW * a.E; i += blockDim.x) whist[i] = 0;
    for (int i = threadIdx.x; i < a.Rs * a.R; i += blockDim.x) tpr[i] = 0;
    __syncthreads();

    int32_t* mine = whist + warp * a.E;
    const bool bad = walk_part(a, w, act, rank_of, mine, tpr + (w.has_rank ? w.r * a.R : 0), ev, rk);
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);

    // this CTA's warps, scanned per expert in warp order; ctot = the CTA's total
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int32_t run = 0;
        for (int wi = 0; wi < NW; ++wi) {
            const int32_t c = whist[wi * a.E + e];
            whist[wi * a.E + e] = run;
            run += c;
        }
        ctot[e] = run;
    }
    cluster_sync();  // every CTA's ctot and tpr are final

    // ranks whose first warp (rank * wpr) is in this CTA
    const int r_lo = (cta * NW + wpr - 1) / wpr;
    const int r_hi = min(a.Rs, ((cta + 1) * NW + wpr - 1) / wpr);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int32_t b = 0;
        for (int c = 0; c < cta; ++c) b += ld_dsmem_s32(dsmem_addr(ctot + e, uint32_t(c)));
        cbase[e] = b;
        for (int rr = r_lo; rr < r_hi; ++rr)
            a.expert_rank_offset[int64_t(e) * a.Rs + rr] = b + whist[(rr * wpr - cta * NW) * a.E + e];
        if (cta == CL - 1) {
            const int32_t n = b + ctot[e];
            a.recv_count[e] = n;
            if (n > a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
        }
    }
    if (cta == 0) {
        for (int i = threadIdx.x; i < a.Rs * a.R; i += blockDim.x) {
            int32_t n = 0;
            for (int c = 0; c < CL; ++c) n += ld_dsmem_s32(dsmem_addr(tpr + i, uint32_t(c)));
            a.num_tokens_per_rank[i] = n;
        }
    }
    __syncthreads();  // cbase
    finish_rows(a, w, ev, rk, [&](int e) { return cbase[e] + mine[e]; });
    cluster_sync();  // expert_rank_offset and recv_count are written; no remote shared reads after this

    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        for (int rr = r_lo; rr < r_hi; ++rr) {
            const int32_t off = cbase[e] + whist[(rr * wpr - cta * NW) * a.E + e];
            const int32_t next = rr + 1 < a.Rs ? a.expert_rank_offset[int64_t(e) * a.Rs + rr + 1] : a.recv_count[e];
            a.num_tokens_per_expert[int64_t(rr) * a.E + e] = next - off;
        }
    }
}

__global__ void __launch_bounds__(32 * kMaxWarps) layout_rank_kernel(LayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t smem[];
    const int W = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t* act = smem;
    int32_t* rank_of = smem + kActiveSlots;
    int32_t* first = rank_of + a.E;   // [E] first row of this chunk, per expert
    int32_t* whist = first + a.E;     // [W][E] per-warp counts, then per-warp first rows
    load_tables(a, act, rank_of);
    for (int i = threadIdx.x; i < W * a.E; i += blockDim.x) whist[i] = 0;
    __syncthreads();

    const int g = blockIdx.x;
    const ChunkGeom cg = chunk_of(a, g);
    const bool src_ok = act[a.r0 + cg.r] != 0;

    // 1. first rows of this chunk (written by the scan)
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) first[e] = a.chunk_hist[int64_t(g) * a.E + e];
    // per-warp counts of this chunk (warp w owns tokens [t0 + w*tw, t0 + (w+1)*tw))
    const int tw = (cg.t1 - cg.t0 + W - 1) / W;
    const int wt0 = min(cg.t1, cg.t0 + warp * tw), wt1 = min(cg.t1, wt0 + tw);
    const int64_t pbase = (int64_t(cg.r) * a.T + wt0) * a.k;
    const int32_t* base = a.topk_idx + pbase;
    int32_t* rows = a.pair_row + pbase;
    const int np = (wt1 - wt0) * a.k;
    int32_t* mine = whist + warp * a.E;
    for (int p0 = 0; p0 < np; p0 += 32 * kBatch) {
        int ev[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int p = p0 + u * 32 + lane;
            ev[u] = p < np ? __ldg(base + p) : -1;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int e = ev[u];
            const bool live = pair_live(e, a.E, src_ok, rank_of);
            const uint32_t m = match_key(uint32_t(e), a.key_bits, __ballot_sync(0xffffffffu, live));
            if (live && lane == __ffs(m) - 1) mine[e] += __popc(m);
            __syncwarp();
        }
    }
    __syncthreads();

    // 2. per-warp first rows: exclusive scan over warps, on top of the chunk's first rows
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int32_t run = first[e];
        for (int w = 0; w < W; ++w) {
            const int32_t v = whist[w * a.E + e];
            whist[w * a.E + e] = run;
            run += v;
        }
    }
    __syncthreads();

    // 3. rows, in (token, slot) order within each warp's part
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
            const bool live = pair_live(e, a.E, src_ok, rank_of);
            const uint32_t m = match_key(uint32_t(e), a.key_bits, __ballot_sync(0xffffffffu, live));
            const int32_t b = live ? mine[e] : 0;
            __syncwarp();
            if (live && lane == __ffs(m) - 1) mine[e] = b + __popc(m);
            __syncwarp();
            if (p < np) rows[p] = live ? b + __popc(m & below) : -1;
        }
    }
}

// ---------------------------------------------------------------------------
// Fused path (EP_LAYOUT_FUSED): the chunked algorithm in ONE cooperative launch
// (all G CTAs co-resident), with two grid barriers instead of kernel
// boundaries.  A barrier is one flag per CTA in the workspace: a CTA publishes
// the barrier's value with a release store and waits (bounded) until every
// flag holds it.  Values come from an epoch word that CTA 0 advances at the
// end of every call (also when a barrier gives up), so repeated calls (and
// replays of a captured graph) never
// see a stale flag as current.  Epoch and flags sit at fixed offsets at the
// start of the workspace, which must be zero before its first use and is left
// consistent by every call (older flags always hold older epochs).  Each warp keeps its part's histogram in shared
// memory from the count phase to the rank phase.
__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// All CTAs of the grid meet here.  False (and EP_STATUS_TIMEOUT) if the wait gave up.
__device__ bool grid_barrier(uint64_t* flags, int G, uint64_t value, int32_t* status) {
    __shared__ int passed;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        st_release_u64(flags + blockIdx.x, value);
    }
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        bool ok = true;
        const uint64_t t0 = global_timer_ns();
        for (int b = 0; b < G && ok; b += 32) {
            const int g = b + lane;
            for (uint32_t it = 0;; ++it) {
                bool here = true;
                if (g < G) {
                    const uint64_t v = ld_acquire_u64(flags + g);
                    here = v == value || v == value + 1;  // value + 1: that CTA has already passed
                }
                if (__all_sync(0xffffffffu, here)) break;
                // the give-up decision must be the same on every lane
                if ((it & 63u) == 63u && __any_sync(0xffffffffu, global_timer_ns() - t0 > kWaitTimeoutNs)) {
                    ok = false;
                    break;
                }
            }
            ok = __all_sync(0xffffffffu, ok);
        }
        if (lane == 0) passed = ok;
    }
    __syncthreads();
    if (!passed && threadIdx.x == 0) flag_status(status, EP_STATUS_TIMEOUT);
    return passed != 0;
}

// Diagnostic (ep_diag_wait_timeout): one CTA enters the fused path's grid barrier
// as if the grid had two CTAs, so it waits for a flag that nothing sets; the
// bounded wait gives up after kWaitTimeoutNs, flags EP_STATUS_TIMEOUT and the
// kernel returns, leaving the context usable.
__global__ void __launch_bounds__(32) diag_wait_timeout_kernel(uint64_t* flags, int32_t* status) {
    grid_barrier(flags, 2, 1, status);
}

__global__ void __launch_bounds__(32 * kMaxWarps) layout_fused_kernel(LayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t smem[];
    __shared__ int32_t seg[kMaxWarps][32];
    __shared__ int32_t col_total[32];
    const int W = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t* act = smem;
    int32_t* tpr = smem + kActiveSlots;
    int32_t* rank_of = smem + 2 * kActiveSlots;
    int32_t* first = rank_of + a.E;
    int32_t* whist = first + a.E;  // [W][E]
    const uint64_t epoch = *reinterpret_cast<volatile uint64_t*>(a.sync);
    uint64_t* flags = a.sync + 1;
    const uint64_t bar0 = 2 * (epoch + 1), bar1 = bar0 + 1;
    load_tables(a, act, rank_of);
    for (int i = threadIdx.x; i < W * a.E; i += blockDim.x) whist[i] = 0;
    for (int d = threadIdx.x; d < a.R; d += blockDim.x) tpr[d] = 0;
    __syncthreads();

    const int g = blockIdx.x;
    const ChunkGeom cg = chunk_of(a, g);
    const bool src_ok = act[a.r0 + cg.r] != 0;
    const int tw = (cg.t1 - cg.t0 + W - 1) / W;
    const int wt0 = min(cg.t1, cg.t0 + warp * tw), wt1 = min(cg.t1, wt0 + tw);
    const int64_t pbase = (int64_t(cg.r) * a.T + wt0) * a.k;
    const int32_t* base = a.topk_idx + pbase;
    int32_t* rows = a.pair_row + pbase;
    const int np = (wt1 - wt0) * a.k;
    int32_t* mine = whist + warp * a.E;

    // ---- phase A: per-warp histograms, token rank sets, chunk histogram
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
            const int e = ev[u];
            bad |= (e < -1 || e >= a.E);
            const bool live = pair_live(e, a.E, src_ok, rank_of);
            const uint32_t m = match_key(uint32_t(e), a.key_bits, __ballot_sync(0xffffffffu, live));
            if (live && lane == __ffs(m) - 1) mine[e] += __popc(m);
            __syncwarp();
        }
    }
    for (int t0 = wt0; t0 < wt1; t0 += 32) {
        const int t = t0 + lane;
        uint64_t ranks = 0;
        if (t < wt1) {
            const int32_t* tb = a.topk_idx + (int64_t(cg.r) * a.T + t) * a.k;
            for (int j = 0; j < a.k; ++j) {
                const int e = __ldg(tb + j);
                if (pair_live(e, a.E, src_ok, rank_of)) ranks |= 1ull << rank_of[e];
            }
            uint8_t* itr = a.is_token_in_rank + (int64_t(cg.r) * a.T + t) * a.R;
            for (int d = 0; d < a.R; ++d) itr[d] = uint8_t((ranks >> d) & 1u);
        }
        for (int d = 0; d < a.R; ++d) {
            const int n = __popc(__ballot_sync(0xffffffffu, (ranks >> d) & 1u));
            if (lane == 0 && n) atomicAdd(tpr + d, n);
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int32_t s = 0;
        for (int w = 0; w < W; ++w) s += whist[w * a.E + e];
        a.chunk_hist[int64_t(g) * a.E + e] = s;
    }
    for (int d = threadIdx.x; d < a.R; d += blockDim.x) a.chunk_tpr[int64_t(g) * a.R + d] = tpr[d];
    if (!grid_barrier(flags, a.G, bar0, a.status)) {
        if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned long long*>(a.sync), epoch + 1);
        return;
    }

    // ---- phase B: columns of 32 experts scanned over the chunks (chunk counts -> first rows)
    const int cols = (a.E + 31) / 32;
    const int rpw = (a.G + W - 1) / W;
    for (int col = g; col < cols; col += a.G) {
        const int e = col * 32 + lane;
        const bool ok = e < a.E;
        const int g0 = warp * rpw, g1 = min(a.G, g0 + rpw);
        int32_t s = 0;
        if (ok)
            for (int gg = g0; gg < g1; ++gg) s += a.chunk_hist[int64_t(gg) * a.E + e];
        seg[warp][lane] = s;
        __syncthreads();
        if (warp == 0) {
            int32_t run = 0;
            for (int w = 0; w < W; ++w) {
                const int32_t t = seg[w][lane];
                seg[w][lane] = run;
                run += t;
            }
            col_total[lane] = run;
            if (ok) {
                a.recv_count[e] = run;
                if (run > a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
            }
        }
        __syncthreads();
        if (ok) {
            int32_t run = seg[warp][lane];
            for (int gg = g0; gg < g1; ++gg) {
                int32_t* q = a.chunk_hist + int64_t(gg) * a.E + e;
                const int32_t v = *q;
                *q = run;
                run += v;
            }
        }
        __syncthreads();
        if (ok) {
            for (int r = warp; r < a.Rs; r += W) {
                const int32_t off = a.chunk_hist[int64_t(r) * a.C * a.E + e];
                const int32_t next = r + 1 < a.Rs ? a.chunk_hist[int64_t(r + 1) * a.C * a.E + e] : col_total[lane];
                a.expert_rank_offset[int64_t(e) * a.Rs + r] = off;
                a.num_tokens_per_expert[int64_t(r) * a.E + e] = next - off;
            }
        }
        __syncthreads();
    }
    const int RR = a.Rs * a.R;
    for (int pr = g * W + warp; pr < RR; pr += a.G * W) {
        const int r = pr / a.R, d = pr - r * a.R;
        const int32_t* colp = a.chunk_tpr + int64_t(r) * a.C * a.R + d;
        int32_t t = 0;
        for (int c = lane; c < a.C; c += 32) t += colp[int64_t(c) * a.R];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
        if (lane == 0) a.num_tokens_per_rank[pr] = t;
    }
    if (!grid_barrier(flags, a.G, bar1, a.status)) {
        if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned long long*>(a.sync), epoch + 1);
        return;
    }

    // ---- phase C: per-warp first rows, then rows
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int32_t run = a.chunk_hist[int64_t(g) * a.E + e];
        for (int w = 0; w < W; ++w) {
            const int32_t v = whist[w * a.E + e];
            whist[w * a.E + e] = run;
            run += v;
        }
    }
    __syncthreads();
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
            const bool live = pair_live(e, a.E, src_ok, rank_of);
            const uint32_t m = match_key(uint32_t(e), a.key_bits, __ballot_sync(0xffffffffu, live));
            const int32_t b = live ? mine[e] : 0;
            __syncwarp();
            if (live && lane == __ffs(m) - 1) mine[e] = b + __popc(m);
            __syncwarp();
            if (p < np) rows[p] = live ? b + __popc(m & below) : -1;
        }
    }
    // every CTA read the epoch before the first barrier; advance it for the next call
    if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned long long*>(a.sync), epoch + 1);
}

// ---------------------------------------------------------------------------
// Look-back path (EP_LAYOUT_LOOKBACK): the chunked algorithm in ONE ordinary
// launch, one CTA per chunk, with no grid-wide barrier.  A chunk's first rows
// need only the histograms of the chunks before it, so each CTA
//   A. counts its chunk (warp histograms kept in shared memory, destination
//      ranks, per-destination token counts), writes the chunk histogram and
//      publishes it with a release flag;
//   B. waits (bounded) for the flags of the chunks before it only -- CTAs are
//      dispatched in index order, so those have started; one warp polls them
//      all, each lane its up to eight flags per round trip -- then sums their
//      histograms: warp w takes chunks w, w + W, ... with all its 16-byte
//      loads in flight, and the warps' sums meet in shared memory;
//   C. assigns rows as the rank kernel does.
// The owners of the per-rank outputs are the chunks that can see them: the
// first chunk of rank r writes expert_rank_offset[:, r], the last chunk of rank
// r num_tokens_per_expert[r] and num_tokens_per_rank[r], the last chunk of all
// recv_count.  Flags use the fused path's epoch scheme (shared workspace
// prefix): the last CTA advances the epoch once every CTA has published, hence
// has read it.
__global__ void __launch_bounds__(32 * kMaxWarps) layout_lookback_kernel(LayoutArgs a) {
    pdl_wait();  // nothing upstream is read before this
    pdl_launch_dependents();
    extern __shared__ int32_t smem[];
    const int NT = blockDim.x;
    const int W = NT >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t* act = smem;
    int32_t* tpr = smem + kActiveSlots;
    int32_t* rank_of = smem + 2 * kActiveSlots;
    int32_t* first = rank_of + a.E;       // [E] rows of the chunks before this one
    int32_t* rank_first = first + a.E;    // [E] rows of the chunks of the ranks before this chunk's rank
    int32_t* whist = rank_first + a.E;    // [W][E]

    const int g = blockIdx.x;
    const ChunkGeom cg = chunk_of(a, g);
    // this warp's part of the chunk: the walk of the one-launch paths, rows within the part kept
    WarpPart w;
    w.r = cg.r;
    w.has_rank = true;
    const int tw = (cg.t1 - cg.t0 + W - 1) / W;
    w.t0 = min(cg.t1, cg.t0 + warp * tw);
    w.t1 = min(cg.t1, w.t0 + tw);
    w.pbase = (int64_t(cg.r) * a.T + w.t0) * a.k;
    w.np = (w.t1 - w.t0) * a.k;
    w.one_round = w.np <= 32 * kBatch;
    int ev[kBatch], rk[kBatch];
    load_first_round(a, w, ev);  // in flight while the tables are set up

    const uint64_t epoch = *reinterpret_cast<volatile uint64_t*>(a.sync);
    uint64_t* flags = a.sync + 1;
    const uint64_t value = 2 * (epoch + 1);
    load_tables(a, act, rank_of);
    for (int i = threadIdx.x; i < W * a.E; i += NT) whist[i] = 0;
    for (int e = threadIdx.x; e < a.E; e += NT) first[e] = rank_first[e] = 0;
    for (int d = threadIdx.x; d < a.R; d += NT) tpr[d] = 0;
    __syncthreads();
    int32_t* mine = whist + warp * a.E;

    // ---- A: warp histograms and rows within the parts, destination ranks, chunk histogram, publish
    const bool bad = walk_part(a, w, act, rank_of, mine, tpr, ev, rk);
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(a.status, EP_STATUS_BAD_EXPERT);
    int32_t* own = a.chunk_hist + int64_t(g) * a.E;
    for (int e = threadIdx.x; e < a.E; e += NT) {
        int32_t s = 0;
        for (int ww = 0; ww < W; ++ww) s += whist[ww * a.E + e];
        own[e] = s;
    }
    for (int d = threadIdx.x; d < a.R; d += NT) a.chunk_tpr[int64_t(g) * a.R + d] = tpr[d];
    // the barrier orders every thread's writes of the chunk before thread 0's release (the release
    // is cumulative), so the flag needs no further fence
    __syncthreads();
    if (threadIdx.x == 0) st_release_u64(flags + int64_t(g) * kLookbackFlagWords, value);

    // ---- B: wait (bounded) for the chunks before this one, then sum their histograms
    __shared__ int passed;
    if (warp == 0) {
        bool ok = true;
        const uint64_t t0 = global_timer_ns();
        uint32_t need = 0;  // bit q: chunk lane + 32 q is before this one and not yet seen published
#pragma unroll
        for (int q = 0; q < kFlagsPerLane; ++q) need |= uint32_t(lane + 32 * q < g) << q;
        for (uint32_t it = 0;; ++it) {
            uint64_t seen[kFlagsPerLane];
#pragma unroll
            for (int q = 0; q < kFlagsPerLane; ++q)
                seen[q] = (need >> q) & 1u ? ld_acquire_u64(flags + int64_t(lane + 32 * q) * kLookbackFlagWords)
                                           : value;
#pragma unroll
            for (int q = 0; q < kFlagsPerLane; ++q)
                if (seen[q] >= value) need &= ~(1u << q);
            if (__all_sync(0xffffffffu, need == 0)) break;
            if ((it & 63u) == 63u && __any_sync(0xffffffffu, global_timer_ns() - t0 > kWaitTimeoutNs)) {
                ok = false;
                break;
            }
        }
        if (lane == 0) passed = ok;
    }
    __syncthreads();
    if (g == a.G - 1 && threadIdx.x == 0)  // every CTA has read the epoch (or the wait gave up)
        atomicMax(reinterpret_cast<unsigned long long*>(a.sync), epoch + 1);
    if (!passed) {
        if (threadIdx.x == 0) flag_status(a.status, EP_STATUS_TIMEOUT);
        return;
    }
    const int rC = cg.r * a.C;  // first chunk of this chunk's rank
    {
        // split at rC into the ranks before this chunk's rank and this rank's earlier chunks.  When
        // E % 4 == 0: warp w takes chunks w, w + W, ...; lane l the 16-byte columns (four experts)
        // l, l + 32, ... of each, kSumChunks chunks by two columns of loads in flight per lane; the
        // warps' sums meet in shared memory.
        if ((a.E & 3) == 0) {
            const int E4 = a.E >> 2;
            for (int c0 = lane; c0 < E4; c0 += 64) {
                const int c1 = c0 + 32;
                int4 sb0 = make_int4(0, 0, 0, 0), sr0 = sb0, sb1 = sb0, sr1 = sb0;
                for (int gg = warp; gg < g; gg += kSumChunks * W) {
                    int4 v0[kSumChunks], v1[kSumChunks];
#pragma unroll
                    for (int u = 0; u < kSumChunks; ++u) {
                        const int gu = gg + u * W;
                        const int4* row = reinterpret_cast<const int4*>(a.chunk_hist + int64_t(gu) * a.E);
                        v0[u] = gu < g ? row[c0] : make_int4(0, 0, 0, 0);
                        v1[u] = (gu < g && c1 < E4) ? row[c1] : make_int4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int u = 0; u < kSumChunks; ++u) {
                        const bool before = gg + u * W < rC;
                        int4& a0 = before ? sb0 : sr0;
                        int4& a1 = before ? sb1 : sr1;
                        a0.x += v0[u].x; a0.y += v0[u].y; a0.z += v0[u].z; a0.w += v0[u].w;
                        a1.x += v1[u].x; a1.y += v1[u].y; a1.z += v1[u].z; a1.w += v1[u].w;
                    }
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c = h ? c1 : c0;
                    if (c >= E4) break;
                    const int4 sb = h ? sb1 : sb0, sr = h ? sr1 : sr0;
                    const int e = 4 * c;
                    if (sb.x | sb.y | sb.z | sb.w) {
                        atomicAdd(rank_first + e, sb.x); atomicAdd(rank_first + e + 1, sb.y);
                        atomicAdd(rank_first + e + 2, sb.z); atomicAdd(rank_first + e + 3, sb.w);
                    }
                    if (sb.x | sb.y | sb.z | sb.w | sr.x | sr.y | sr.z | sr.w) {
                        atomicAdd(first + e, sb.x + sr.x); atomicAdd(first + e + 1, sb.y + sr.y);
                        atomicAdd(first + e + 2, sb.z + sr.z); atomicAdd(first + e + 3, sb.w + sr.w);
                    }
                }
            }
        } else {
            for (int e = lane; e < a.E; e += 32) {
                int32_t sb = 0, sr = 0;
                for (int gg = warp; gg < g; gg += W) {
                    const int32_t v = a.chunk_hist[int64_t(gg) * a.E + e];
                    if (gg < rC) sb += v;
                    else sr += v;
                }
                if (sb) atomicAdd(rank_first + e, sb);
                if (sb | sr) atomicAdd(first + e, sb + sr);
            }
        }
    }
    __syncthreads();
    if (g == rC) {
        for (int e = threadIdx.x; e < a.E; e += NT) a.expert_rank_offset[int64_t(e) * a.Rs + cg.r] = first[e];
    }
    if (g == rC + a.C - 1) {
        for (int e = threadIdx.x; e < a.E; e += NT)
            a.num_tokens_per_expert[int64_t(cg.r) * a.E + e] = first[e] - rank_first[e] + own[e];
        for (int d = warp; d < a.R; d += W) {
            int32_t t = 0;
            for (int c = lane; c < a.C; c += 32) t += a.chunk_tpr[int64_t(rC + c) * a.R + d];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
            if (lane == 0) a.num_tokens_per_rank[int64_t(cg.r) * a.R + d] = t;
        }
    }
    if (g == a.G - 1) {
        for (int e = threadIdx.x; e < a.E; e += NT) {
            const int32_t n = first[e] + own[e];
            a.recv_count[e] = n;
            if (n > a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
        }
    }

    // ---- C: per-warp first rows, then each live pair's row = its warp's first row + its row in the part
    for (int e = threadIdx.x; e < a.E; e += NT) {
        int32_t run = first[e];
        for (int ww = 0; ww < W; ++ww) {
            const int32_t v = whist[ww * a.E + e];
            whist[ww * a.E + e] = run;
            run += v;
        }
    }
    __syncthreads();
    finish_rows(a, w, ev, rk, [&](int e) { return mine[e]; });
}

struct LayoutGeom {
    int C, G, chunk_tokens, warps;
};

// Chunks per source rank, tokens per chunk and warps per CTA for a shape whose
// routing has Rs source ranks (Rs = R for the whole world, 1 for one rank).
// `chunks` > 0 asks for that many chunks in all instead of one per kPairsPerChunk pairs.
LayoutGeom layout_geom(const ep_dims_t& d, int Rs, int chunks = 0) {
    LayoutGeom lg;
    const int64_t pairs = int64_t(Rs) * d.num_tokens * d.num_topk;
    const int64_t target = chunks > 0 ? std::min<int64_t>(kMaxChunks, chunks)
                                      : std::min<int64_t>(kMaxChunks, std::max<int64_t>(kTargetChunks, ceil_div(pairs, kPairsPerChunk)));
    int64_t C = std::max<int64_t>(1, ceil_div(target, Rs));
    C = std::max<int64_t>(1, std::min<int64_t>(C, d.num_tokens));
    lg.chunk_tokens = int(std::max<int64_t>(1, ceil_div(d.num_tokens, C)));
    lg.C = int(std::max<int64_t>(1, ceil_div(std::max(d.num_tokens, 1), lg.chunk_tokens)));
    lg.G = Rs * lg.C;
    // warp-private histograms of the rank kernel: W * E ints within ~96 KB
    const int64_t per_warp = int64_t(d.num_experts) * 4;
    lg.warps = int(std::max<int64_t>(1, std::min<int64_t>(kMaxWarps, (96 * 1024) / per_warp)));
    return lg;
}

size_t layout_ws_hist_bytes(const ep_dims_t& d, const LayoutGeom& lg) {
    return round_up16(size_t(lg.G) * d.num_experts * 4);
}

size_t layout_ws_tpr_bytes(const ep_dims_t& d, const LayoutGeom& lg) {
    return round_up16(size_t(lg.G) * d.num_ranks * 4);
}

// Largest grid of the fused kernel that can be co-resident on the current device (0 if none).
int fused_capacity(int threads, size_t smem) {
    // asked on every call: the answer depends on smem, and only the fused path asks
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    int coop = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) return 0;
    int per_sm = 0;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(layout_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
            cudaSuccess)
        return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, layout_fused_kernel, threads, smem) != cudaSuccess)
        return 0;
    return per_sm * sm_count();
}

}  // namespace
}  // namespace ep

using namespace ep;

namespace ep {
namespace {

size_t cluster_smem_bytes(const ep_dims_t& d) {
    return size_t(kActiveSlots + kSmallMaxRanks * kSmallMaxRanks + 3 * d.num_experts +
                  (kSmallThreads / 32) * d.num_experts) * 4;
}

ClusterFitCache g_layout_cluster_fit;

size_t fused_smem_bytes(const ep_dims_t& d, const LayoutGeom& lg) {
    return size_t(2 * kActiveSlots + 2 * d.num_experts + lg.warps * d.num_experts) * 4;
}

size_t lookback_smem_bytes(const ep_dims_t& d, const LayoutGeom& lg) {
    return size_t(2 * kActiveSlots + 3 * d.num_experts + lg.warps * d.num_experts) * 4;
}

// The path ep_layout takes for these dims and cfg, or a negative EP_ERR_* code.
// AUTO, from graph replays on B200: one CTA up to kSmallAutoPairs pairs (8.6 us at 1024
// pairs, 10.6 us at 2048); a cluster up to kClusterAutoPairs (10.6 us from 4096 to 16384
// pairs, 12.7 us at 32768, 14.7 at 49152, 16.8 at 65536, where one CTA takes 14.7 to 74 us);
// the look-back path beyond, one launch (prefill, 262144 pairs: 21.5 us per stream launch
// against 25.9 for the three chunked launches and 20.3 for the fused cooperative launch,
// which is slower in a graph); the chunked path only if the chunk grid outgrows the flags.
int resolve_layout_path(const ep_dims_t& d, int Rs, const ep_cfg_t& cfg, const LayoutGeom& lg) {
    const int64_t pairs = int64_t(Rs) * d.num_tokens * d.num_topk;
    const bool tables_fit = d.num_ranks <= kSmallMaxRanks && d.num_experts <= kSmallMaxExperts;
    const bool small_ok = tables_fit && pairs <= kSmallMaxPairs;
    const bool cluster_ok = tables_fit && pairs <= kClusterMaxPairs;
    switch (cfg.variant) {
        case EP_VARIANT_AUTO:
            if (small_ok && pairs <= kSmallAutoPairs) return EP_LAYOUT_SINGLE_CTA;
            if (cluster_ok && pairs <= kClusterAutoPairs) return EP_LAYOUT_CLUSTER;
            if (lg.G <= kMaxFlags && lookback_smem_bytes(d, lg) <= size_t(max_smem_optin())) return EP_LAYOUT_LOOKBACK;
            return EP_LAYOUT_CHUNKED;
        case EP_LAYOUT_CHUNKED:
            return EP_LAYOUT_CHUNKED;
        case EP_LAYOUT_SINGLE_CTA:
            return small_ok ? int(EP_LAYOUT_SINGLE_CTA) : int(EP_ERR_UNSUPPORTED);
        case EP_LAYOUT_FUSED:
            return lg.G <= kMaxFlags && lg.G <= fused_capacity(32 * lg.warps, fused_smem_bytes(d, lg))
                       ? int(EP_LAYOUT_FUSED)
                       : int(EP_ERR_UNSUPPORTED);
        case EP_LAYOUT_CLUSTER:
            return cluster_ok ? int(EP_LAYOUT_CLUSTER) : int(EP_ERR_UNSUPPORTED);
        case EP_LAYOUT_LOOKBACK:
            return lg.G <= kMaxFlags && lookback_smem_bytes(d, lg) <= size_t(max_smem_optin())
                       ? int(EP_LAYOUT_LOOKBACK)
                       : int(EP_ERR_UNSUPPORTED);
        default:
            return EP_ERR_INVALID;
    }
}

size_t layout_ws_bytes(const ep_dims_t& d, const LayoutGeom& lg) {
    return kSyncBytes + layout_ws_hist_bytes(d, lg) + layout_ws_tpr_bytes(d, lg);
}

int layout_run(const ep_dims_t& d, int Rs, int r0, const int32_t* topk_idx, const uint8_t* active, void* workspace,
               size_t workspace_bytes, int32_t* num_tokens_per_expert, int32_t* num_tokens_per_rank,
               uint8_t* is_token_in_rank, int32_t* recv_count, int32_t* expert_rank_offset, int32_t* pair_row,
               int32_t* status, const ep_cfg_t& cfg, cudaStream_t s);

}  // namespace
}  // namespace ep

extern "C" int ep_layout_path(ep_dims_t d, ep_cfg_t cfg) {
    const int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    return resolve_layout_path(d, d.num_ranks, cfg, layout_geom(d, d.num_ranks, cfg.max_ctas));
}

extern "C" size_t ep_layout_workspace_bytes(ep_dims_t d) {
    if (check_dims(d) != EP_OK) return 0;
    return layout_ws_bytes(d, layout_geom(d, d.num_ranks));
}

extern "C" int ep_layout(ep_dims_t d, const int32_t* topk_idx, const uint8_t* active, void* workspace,
                         size_t workspace_bytes, int32_t* num_tokens_per_expert, int32_t* num_tokens_per_rank,
                         uint8_t* is_token_in_rank, int32_t* recv_count, int32_t* expert_rank_offset,
                         int32_t* pair_row, int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_layout");
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (!active || !num_tokens_per_expert || !num_tokens_per_rank || !recv_count || !expert_rank_offset)
        return EP_ERR_INVALID;
    if (RT > 0 && (!topk_idx || !is_token_in_rank || !pair_row)) return EP_ERR_INVALID;
    const size_t need = ep_layout_workspace_bytes(d);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return EP_ERR_INVALID;
    return layout_run(d, d.num_ranks, 0, topk_idx, active, workspace, workspace_bytes, num_tokens_per_expert,
                      num_tokens_per_rank, is_token_in_rank, recv_count, expert_rank_offset, pair_row, status, cfg,
                      static_cast<cudaStream_t>(stream));
}

// Rank-local layout: the same kernels over one source rank's routing (Rs = 1),
// with the mask and destinations of the whole world.  Its per-source outputs are
// one row; the offset within each expert (always 0 for a lone source) and the
// receive counts (equal to the local counts) go to the workspace tail.
extern "C" size_t ep_layout_local_workspace_bytes(ep_dims_t d) {
    if (check_dims(d) != EP_OK) return 0;
    return layout_ws_bytes(d, layout_geom(d, 1)) + 2 * round_up16(size_t(d.num_experts) * 4);
}

extern "C" int ep_layout_local(ep_dims_t d, int32_t rank, const int32_t* topk_idx, const uint8_t* active,
                               void* workspace, size_t workspace_bytes, int32_t* num_tokens_per_expert,
                               int32_t* num_tokens_per_rank, uint8_t* is_token_in_rank, int32_t* local_row,
                               int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_layout_local");
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    if (rank < 0 || rank >= d.num_ranks) return EP_ERR_INVALID;
    if (!active || !num_tokens_per_expert || !num_tokens_per_rank) return EP_ERR_INVALID;
    if (d.num_tokens > 0 && (!topk_idx || !is_token_in_rank || !local_row)) return EP_ERR_INVALID;
    const LayoutGeom lg = layout_geom(d, 1, cfg.max_ctas);
    const size_t base = layout_ws_bytes(d, lg);
    if (!workspace || workspace_bytes < ep_layout_local_workspace_bytes(d) || !aligned16(workspace) ||
        workspace_bytes < base + 2 * round_up16(size_t(d.num_experts) * 4))
        return EP_ERR_INVALID;
    char* ws = static_cast<char*>(workspace);
    int32_t* offset_scratch = reinterpret_cast<int32_t*>(ws + base);
    int32_t* count_scratch = reinterpret_cast<int32_t*>(ws + base + round_up16(size_t(d.num_experts) * 4));
    return layout_run(d, 1, rank, topk_idx, active, workspace, base, num_tokens_per_expert, num_tokens_per_rank,
                      is_token_in_rank, count_scratch, offset_scratch, local_row, status, cfg,
                      static_cast<cudaStream_t>(stream));
}

namespace ep {
namespace {

int layout_run(const ep_dims_t& d, int Rs, int r0, const int32_t* topk_idx, const uint8_t* active, void* workspace,
               size_t workspace_bytes, int32_t* num_tokens_per_expert, int32_t* num_tokens_per_rank,
               uint8_t* is_token_in_rank, int32_t* recv_count, int32_t* expert_rank_offset, int32_t* pair_row,
               int32_t* status, const ep_cfg_t& cfg, cudaStream_t s) {
    // cfg.max_ctas: the chunk count of the chunked, fused and look-back paths (their grids)
    const LayoutGeom lg = layout_geom(d, Rs, cfg.max_ctas);
    if (workspace_bytes < layout_ws_bytes(d, lg)) return EP_ERR_INVALID;
    LayoutArgs a;
    a.topk_idx = topk_idx;
    a.active = active;
    char* ws = static_cast<char*>(workspace);
    a.sync = reinterpret_cast<uint64_t*>(ws);
    a.chunk_hist = reinterpret_cast<int32_t*>(ws + kSyncBytes);
    a.chunk_tpr = reinterpret_cast<int32_t*>(ws + kSyncBytes + layout_ws_hist_bytes(d, lg));
    a.num_tokens_per_expert = num_tokens_per_expert;
    a.num_tokens_per_rank = num_tokens_per_rank;
    a.is_token_in_rank = is_token_in_rank;
    a.recv_count = recv_count;
    a.expert_rank_offset = expert_rank_offset;
    a.pair_row = pair_row;
    a.status = status;
    a.R = d.num_ranks;
    a.Rs = Rs;
    a.r0 = r0;
    a.T = d.num_tokens;
    a.k = d.num_topk;
    a.E = d.num_experts;
    a.E_local = d.num_experts / d.num_ranks;
    a.key_bits = 0;
    while ((1 << a.key_bits) < d.num_experts) ++a.key_bits;
    a.C = lg.C;
    a.G = lg.G;
    a.chunk_tokens = lg.chunk_tokens;
    a.cap = int64_t(d.num_ranks) * d.num_tokens;

    const int path = resolve_layout_path(d, Rs, cfg, lg);
    if (path < 0) return path;
    const int W = lg.warps;
    if (path == EP_LAYOUT_FUSED) {
        const size_t fused_smem = fused_smem_bytes(d, lg);
        void* args[] = {&a};
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(lg.G);
        lc.blockDim = dim3(32 * W);
        lc.dynamicSmemBytes = fused_smem;
        lc.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        lc.attrs = attr;
        lc.numAttrs = 1;
        if (cudaLaunchKernelExC(&lc, reinterpret_cast<const void*>(layout_fused_kernel), args) != cudaSuccess) {
            cudaGetLastError();
            return EP_ERR_CUDA;
        }
        return launch_result();
    }
    if (path == EP_LAYOUT_LOOKBACK) {
        const size_t smem = lookback_smem_bytes(d, lg);
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(layout_lookback_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
                cudaSuccess)
            return EP_ERR_CUDA;
        if (launch_pdl(layout_lookback_kernel, dim3(lg.G), dim3(32 * W), smem, s, a) != cudaSuccess)
            return EP_ERR_CUDA;
        return launch_result();
    }
    if (path == EP_LAYOUT_CLUSTER) {
        const size_t smem = cluster_smem_bytes(d);
        ep_dims_t widest = d;  // the largest shared-memory need of the path (E = kSmallMaxExperts)
        widest.num_experts = kSmallMaxExperts;
        const size_t smem_max = cluster_smem_bytes(widest);
        if (cudaFuncSetAttribute(layout_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem_max)) != cudaSuccess ||
            cudaFuncSetAttribute(layout_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess)
            return EP_ERR_CUDA;
        // one CTA per kClusterPairsPerCta pairs, 2 to kClusterMaxCtas, as many as fit at once
        const int64_t pairs = int64_t(Rs) * d.num_tokens * d.num_topk;
        const int want = int(std::min<int64_t>(kClusterMaxCtas,
                                               std::max<int64_t>(2, ceil_div(pairs, kClusterPairsPerCta))));
        const int cl = fitting_cluster(layout_cluster_kernel, want, kSmallThreads, smem_max, g_layout_cluster_fit);
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(cl);
        lc.blockDim = dim3(kSmallThreads);
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
        if (cudaLaunchKernelEx(&lc, layout_cluster_kernel, a) != cudaSuccess) return EP_ERR_CUDA;
        return launch_result();
    }
    if (path == EP_LAYOUT_SINGLE_CTA) {
        const size_t smem = size_t(kActiveSlots + kSmallMaxRanks * kSmallMaxRanks + d.num_experts +
                                   (kSmallThreads / 32) * d.num_experts) * 4;
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(layout_single_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess)
            return EP_ERR_CUDA;
        if (launch_pdl(layout_single_cta_kernel, dim3(1), dim3(kSmallThreads), smem, s, a) != cudaSuccess)
            return EP_ERR_CUDA;
        return launch_result();
    }
    const size_t count_smem = size_t(2 * kActiveSlots + 2 * d.num_experts) * 4;
    const size_t rank_smem = size_t(kActiveSlots + 2 * d.num_experts + W * d.num_experts) * 4;
    if (count_smem > 48 * 1024 &&
        cudaFuncSetAttribute(layout_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(count_smem)) !=
            cudaSuccess)
        return EP_ERR_CUDA;
    if (rank_smem > 48 * 1024 &&
        cudaFuncSetAttribute(layout_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(rank_smem)) !=
            cudaSuccess)
        return EP_ERR_CUDA;
    if (launch_pdl(layout_count_kernel, dim3(lg.G), dim3(32 * kMaxWarps), count_smem, s, a) != cudaSuccess ||
        launch_pdl(layout_scan_kernel, dim3(unsigned(ceil_div(d.num_experts, 32))), dim3(32 * kScanWarps), 0, s, a) !=
            cudaSuccess ||
        launch_pdl(layout_rank_kernel, dim3(lg.G), dim3(32 * W), rank_smem, s, a) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

}  // namespace
}  // namespace ep

extern "C" int ep_diag_wait_timeout(void* flags, int32_t* status, void* stream) {
    EP_NVTX_RANGE("ep_diag_wait_timeout");
    if (!flags || !status || (reinterpret_cast<uintptr_t>(flags) & 7u)) return EP_ERR_INVALID;
    diag_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t*>(flags), status);
    return launch_result();
}
