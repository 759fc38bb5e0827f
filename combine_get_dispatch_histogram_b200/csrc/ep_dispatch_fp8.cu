// ep_dispatch_fp8.cu -- token dispatch with the payload cast to float8 e4m3 on sm_100a.
//
// Defines Buffer.low_latency_dispatch with use_fp8=True of the NeMo AutoModel
// page "nemo_automodel.components.moe.uccl_ep.buffer" (and its round_scale /
// use_ue8m0 options): every live pair's token row arrives in its expert slab
// as e4m3 codes with one scale per 128 channels; the scales are stored
// column-major, [E][groups][CAP].  Two launches: the cast (codes to every live
// row, each token's scales once to a row-major workspace) and a scale writer
// that fills the column-major tensor with coalesced stores.
#include <algorithm>
#include <cstdint>

#include <cuda_fp8.h>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

// ---------------------------------------------------------------------------
// Both data paths cast a token row once, in pieces of 512 channels (four scale
// groups): lane l owns 16 contiguous channels, so 8 lanes hold one group and
// its amax is a shuffle-max over 8 lanes, and the same codes go to every live
// row of the token.
//
// Vector path (EP_VARIANT_VECTOR; AUTO when a bf16 row is too long for one
// bulk stage): a unit is a token x 512 channels; each warp walks a contiguous,
// balanced range of units, loads its piece through registers and stores 16
// bytes of codes per lane to every live row.
struct DispatchFp8Args {
    const uint8_t* x;
    const int32_t* topk_idx;
    const int32_t* pair_row;
    uint8_t* codes;
    uint8_t* scales;       // column-major [E][words][cap]
    uint32_t* tok_scales;  // workspace [n_tok][words]: fp32 scales, or UE8M0 words
    const int32_t* recv_count;
    int32_t* src_info;
    int32_t* status;
    int T, k, E, H, groups;
    int words;             // scale words per row: H/128 (fp32) or H/512 (UE8M0)
    int64_t cap;
    int64_t n_tok;
    int stages;            // bulk path: bf16 row stages per CTA
    // bulk path, paced reads (read_period_ns 0: off): the producer prefetches the rows it will
    // stage next into L2 only while globaltimer % read_period_ns < read_window_ns, up to
    // read_ahead rows past the one it is loading (as ep_dispatch's EP_VARIANT_PACED)
    uint64_t read_period_ns, read_window_ns;
    int read_ahead;
};

template <int FMT>
__device__ __forceinline__ float fp8_group_scale(float amax, uint32_t* ue8m0) {
    if (FMT == EP_FP8_SCALE_F32) {
        *ue8m0 = 127u;
        return amax == 0.0f ? 1.0f : amax / 448.0f;
    }
    int e = 0;
    if (amax != 0.0f) {
        int f;
        const float m = frexpf(amax / 448.0f, &f);  // amax/448 = m * 2^f, 0.5 <= m < 1
        e = m == 0.5f ? f - 1 : f;                   // smallest e with 2^e >= amax/448
        e = max(-127, min(127, e));
    }
    *ue8m0 = uint32_t(e + 127);
    return ldexpf(1.0f, e);
}

// codes of x / scale.  A power-of-two scale divides exactly as a multiplication by
// its reciprocal (also a power of two, exact), so those formats multiply.
template <int FMT>
__device__ __forceinline__ uint2 fp8_cast8(const float* f, float scale) {
    float q[8];
    if (FMT == EP_FP8_SCALE_F32) {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = f[i] / scale;
    } else {
        const float inv = 1.0f / scale;
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = f[i] * inv;
    }
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const __nv_fp8x2_storage_t lo =
            __nv_cvt_float2_to_fp8x2(make_float2(q[4 * h], q[4 * h + 1]), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi =
            __nv_cvt_float2_to_fp8x2(make_float2(q[4 * h + 2], q[4 * h + 3]), __NV_SATFINITE, __NV_E4M3);
        w[h] = uint32_t(lo) | (uint32_t(hi) << 16);
    }
    return make_uint2(w[0], w[1]);
}

// One lane's 16 channels (two 16-byte bf16 vectors, raw[0] first) cast to e4m3.
// The 8 lanes of a 128-channel group (lanes 8g .. 8g+7) share the scale: amax is
// a shuffle-max over them, so every lane of the warp must call this together.
// Lanes with valid == false contribute nothing and get zero codes.
template <int FMT>
__device__ __forceinline__ uint4 fp8_cast_lane(uint4 r0, uint4 r1, bool valid, float* scale_out, uint32_t* ue_out) {
    float f[16];
    float amax = 0.f;
    if (valid) {
        const uint32_t wds[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[2 * i] = __uint_as_float(wds[i] << 16);
            f[2 * i + 1] = __uint_as_float(wds[i] & 0xffff0000u);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    uint32_t ue = 127u;
    const float scale = fp8_group_scale<FMT>(amax, &ue);
    *scale_out = scale;
    *ue_out = ue;
    if (!valid) return make_uint4(0, 0, 0, 0);
    const uint2 lo = fp8_cast8<FMT>(f, scale);
    const uint2 hi = fp8_cast8<FMT>(f + 8, scale);
    return make_uint4(lo.x, lo.y, hi.x, hi.y);
}

// The token's scales of piece pc (512 channels, lane l owns channels 16l..16l+15),
// row-major in the workspace: one fp32 per group, or one word of four UE8M0
// bytes per piece.  Every lane of the warp calls this together.
template <int FMT>
__device__ __forceinline__ void fp8_put_token_scales(uint32_t* ts, int pc, int lane, bool valid, float scale,
                                                     uint32_t ue) {
    if (FMT == EP_FP8_SCALE_UE8M0) {
        const uint32_t b1 = __shfl_sync(0xffffffffu, ue, 8);
        const uint32_t b2 = __shfl_sync(0xffffffffu, ue, 16);
        const uint32_t b3 = __shfl_sync(0xffffffffu, ue, 24);
        if (lane == 0) ts[pc] = ue | (b1 << 8) | (b2 << 16) | (b3 << 24);
    } else if (valid && (lane & 7) == 0) {
        ts[pc * 4 + (lane >> 3)] = __float_as_uint(scale);
    }
}

template <int FMT>
__global__ void __launch_bounds__(256) dispatch_fp8_kernel(DispatchFp8Args a) {
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int nvec = a.H >> 3;     // 16-byte bf16 vectors per row
    constexpr int kPieceVec = 64;  // 512 channels per unit; lane l owns channels [16l, 16l + 16)
    const int np = (nvec + kPieceVec - 1) / kPieceVec;
    const int64_t n_units = a.n_tok * np;
    const int64_t q = n_units / warps, rem = n_units % warps;
    const int64_t u0 = gw * q + (gw < rem ? gw : rem);
    const int64_t u1 = u0 + q + (gw < rem ? 1 : 0);

    int64_t cur_tok = -1;
    uint32_t mask = 0;
    int my_e = -1, my_row = -1;
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
            if (lane < a.k && pc == 0) {
                if (row >= a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
                if (valid_row && !live) flag_status(a.status, EP_STATUS_BAD_EXPERT);
                if (live) {
                    const int src_rank = int(tok / a.T);
                    reinterpret_cast<int2*>(a.src_info)[int64_t(e) * a.cap + row] =
                        make_int2(src_rank, int(tok - int64_t(src_rank) * a.T));
                }
            }
            mask = __ballot_sync(0xffffffffu, live);
            my_e = live ? e : -1;
            my_row = row;
        }
        if (mask == 0u) continue;
        // 8 lanes x 16 channels = one 128-channel scale group: valid for all 8 lanes or none
        const int v = pc * kPieceVec + 2 * lane;
        const bool valid = v < nvec;
        const uint8_t* src = a.x + tok * int64_t(a.H) * 2;
        uint4 r0 = make_uint4(0, 0, 0, 0), r1 = r0;
        if (valid) {
            r0 = ld_stream_v4(src + int64_t(v) * 16);
            r1 = ld_stream_v4(src + int64_t(v + 1) * 16);
        }
        float scale;
        uint32_t ue;
        const uint4 code = fp8_cast_lane<FMT>(r0, r1, valid, &scale, &ue);
        fp8_put_token_scales<FMT>(a.tok_scales + tok * a.words, pc, lane, valid, scale, ue);
        for (int j = 0; j < a.k; ++j) {
            if (!((mask >> j) & 1u)) continue;
            const int e = __shfl_sync(0xffffffffu, my_e, j);
            const int row = __shfl_sync(0xffffffffu, my_row, j);
            if (valid) {
                uint8_t* dst = a.codes + (int64_t(e) * a.cap + row) * a.H;
                st_global_v4(dst + int64_t(v) * 8, code);
            }
        }
    }
}

// FP8 bulk path (EP_VARIANT_BULK; AUTO when a bf16 row fits one stage).  A CTA is
// one producer warp and W consumer warps over a persistent range of token rows
// (row i of the CTA is token blockIdx.x + i * gridDim.x):
//   - the producer parks each row's routing in shared memory and bulk-loads the
//     bf16 row into stage i % S (a row with no live pair is not loaded), reusing
//     a stage once every consumer thread has released it (mbarrier `empty`);
//   - the consumer warps cast every staged row together, warp w taking the
//     512-channel pieces w, w + W, ..., into one of two code-row buffers; after a
//     barrier among them, lane j (< k) of the first consumer warp bulk-stores the
//     code row to slot j's slab row.  A code buffer is rewritten once the stores
//     that read it two rows earlier are done reading it.
// The copy engine moves every byte; the warps only cast.  Every consumer warp
// waits for every row in order, so when it waits for row i in stage i % S it
// has itself consumed row i - S there: the parity wait (which tells phases
// apart only modulo 2) cannot mistake the stage's previous fill for row i.
// The first of the two barriers per row also ORs the consumers' wait timeouts,
// so all of them leave the loop together and no barrier is left waiting.
constexpr int kFp8MaxConsumers = 16;
constexpr int kFp8DefaultConsumers = 8;  // per CTA unless cfg.threads asks for more (up to kFp8MaxConsumers)
constexpr int kFp8MaxStages = 16;
constexpr uint32_t kFp8RowMax = 16384;  // largest bf16 row the bulk path stages whole
constexpr int kFp8Bar = 1;              // named barrier of the consumer warps
// paced reads: the schedule of ep_dispatch's EP_VARIANT_PACED
constexpr uint64_t kFp8PacePeriodNs = 40000;
constexpr uint64_t kFp8PaceWindowNs = 6000;
constexpr int64_t kFp8PaceAheadBytes = 300 * 1024;

template <int FMT>
__global__ void __launch_bounds__(32 * (1 + kFp8MaxConsumers)) dispatch_fp8_bulk_kernel(DispatchFp8Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = int(blockDim.x >> 5) - 1;
    const int S = a.stages;
    const uint32_t row_bytes = uint32_t(a.H) * 2;
    const uint32_t stage_bytes = (row_bytes + 127u) & ~127u;
    const uint32_t code_bytes = (uint32_t(a.H) + 127u) & ~127u;
    uint8_t* codes_smem = smem + size_t(S) * stage_bytes;  // [2][code_bytes]
    uint64_t* full = reinterpret_cast<uint64_t*>(codes_smem + 2 * size_t(code_bytes));
    uint64_t* empty = full + S;
    int2* meta = reinterpret_cast<int2*>(empty + S);  // [S][32] (e or -1, row) of the staged row

    if (threadIdx.x == 0) {
        // every producer lane arrives on `full` (each releasing its own routing
        // write) and every consumer thread on `empty` (after its last stage read)
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(full + s), 32);
            mbar_init(smem_u32(empty + s), 32 * W);
        }
        mbar_init_fence();
    }
    __syncthreads();
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits

    const int64_t first = blockIdx.x, step = gridDim.x;
    const int64_t my_n = first < a.n_tok ? (a.n_tok - 1 - first) / step + 1 : 0;

    if (warp == 0) {
        // ---------------- producer
        const uint64_t pol = policy_evict_first();
        auto routing = [&](int64_t i, int& e, int& row) {
            e = -1;
            row = -1;
            if (lane < a.k) {
                const int64_t p = (first + i * step) * a.k + lane;
                e = __ldg(a.topk_idx + p);
                row = __ldg(a.pair_row + p);
            }
        };
        const uint64_t pol_prefetch = policy_evict_last();
        int64_t pf = my_n < S ? my_n : S;  // rows [0, pf) are loaded straight or prefetched
        // paced reads: in the read window (or when fewer than a ring's worth of rows are
        // prefetched), prefetch rows [pf, i + read_ahead) that have a live slot, lane j row pf + j
        auto pace_reads = [&](int64_t i) {
            int go = 0;
            if (lane == 0) go = pf <= i + S || global_timer_ns() % a.read_period_ns < a.read_window_ns;
            if (!__shfl_sync(0xffffffffu, go, 0)) return;
            const int64_t want = (i + a.read_ahead) < my_n ? (i + a.read_ahead) : my_n;
            for (; pf < want; pf += 32) {
                const int64_t v = pf + lane;
                if (v >= want) continue;
                const int64_t tok = first + v * step;
                bool live = false;
                for (int j = 0; j < a.k; ++j) {
                    const int r = __ldg(a.pair_row + tok * a.k + j);
                    live |= r >= 0 && r < a.cap;
                }
                if (live) bulk_prefetch_l2(a.x + tok * int64_t(row_bytes), row_bytes, pol_prefetch);
            }
            if (pf > want) pf = want;
        };
        int e_next = -1, row_next = -1;
        if (my_n > 0) routing(0, e_next, row_next);
        for (int64_t i = 0; i < my_n; ++i) {
            const int s = int(i % S);
            const int e = e_next, row = row_next;
            if (i + 1 < my_n) routing(i + 1, e_next, row_next);  // one row ahead
            if (i >= S) {
                // every consumer thread has finished reading stage s for row i - S
                const bool freed = __all_sync(0xffffffffu, mbar_wait(smem_u32(empty + s), uint32_t((i / S - 1) & 1)));
                if (!freed) {
                    if (lane == 0) flag_status(a.status, EP_STATUS_TIMEOUT);
                    break;
                }
            }
            const bool valid_row = row >= 0 && row < a.cap;
            const bool live = valid_row && e >= 0 && e < a.E;
            if (lane < a.k) {
                if (row >= a.cap) flag_status(a.status, EP_STATUS_OVERFLOW);
                if (valid_row && !live) flag_status(a.status, EP_STATUS_BAD_EXPERT);
            }
            meta[s * 32 + lane] = make_int2(live ? e : -1, row);
            const bool any = __ballot_sync(0xffffffffu, live) != 0u;
            const uint32_t bar = smem_u32(full + s);
            if (lane == 0 && any) {
                mbar_arrive_expect_tx(bar, row_bytes);
                bulk_load(smem_u32(smem + size_t(s) * stage_bytes), a.x + (first + i * step) * int64_t(row_bytes),
                          row_bytes, bar, pol);
            } else {
                mbar_arrive(bar);
            }
            if (a.read_period_ns != 0) pace_reads(i);
        }
        return;
    }

    // ---------------- consumers
    const int w = warp - 1;
    const int nthreads = 32 * W;
    const uint64_t pol = policy_evict_first();
    const int np = (a.H + 511) / 512;  // 512-channel pieces: lane l owns channels [16l, 16l + 16)
    int used = 0;                       // code rows stored so far
    for (int64_t i = 0; i < my_n; ++i) {
        const int s = int(i % S);
        const bool landed = __all_sync(0xffffffffu, mbar_wait(smem_u32(full + s), uint32_t((i / S) & 1)));
        if (w == 0) bulk_wait_read<1>();  // the stores of two code rows ago have read the buffer
        if (named_bar_or(kFp8Bar, nthreads, !landed)) {
            if (threadIdx.x == 32) flag_status(a.status, EP_STATUS_TIMEOUT);
            break;
        }
        const int2 m = meta[s * 32 + lane];
        if (__ballot_sync(0xffffffffu, m.x >= 0) == 0u) {  // the same routing for every warp
            mbar_arrive(smem_u32(empty + s));
            continue;
        }
        const int64_t tok = first + i * step;
        uint8_t* cb = codes_smem + size_t(used & 1) * code_bytes;
        const uint8_t* stage = smem + size_t(s) * stage_bytes;
        uint32_t* ts = a.tok_scales + tok * a.words;
        for (int pc = w; pc < np; pc += W) {
            const int c0 = pc * 512 + 16 * lane;
            const bool valid = c0 < a.H;  // whole 128-channel groups: all 8 lanes of a group or none
            uint4 r0 = make_uint4(0, 0, 0, 0), r1 = r0;
            if (valid) {
                r0 = *reinterpret_cast<const uint4*>(stage + size_t(c0) * 2);
                r1 = *reinterpret_cast<const uint4*>(stage + size_t(c0) * 2 + 16);
            }
            float scale;
            uint32_t ue;
            const uint4 code = fp8_cast_lane<FMT>(r0, r1, valid, &scale, &ue);
            fp8_put_token_scales<FMT>(ts, pc, lane, valid, scale, ue);
            if (valid) *reinterpret_cast<uint4*>(cb + c0) = code;
        }
        mbar_arrive(smem_u32(empty + s));  // this thread is done with the bf16 stage
        fence_proxy_async_shared();         // its code stores, before the bulk copies read them
        named_bar_sync(kFp8Bar, nthreads);  // the whole code row is in cb
        if (w == 0) {
            // the producer parks only live routing; checked again before any address is formed
            if (m.x >= 0 && m.x < a.E && m.y >= 0 && m.y < a.cap) {
                const int64_t slab_row = int64_t(m.x) * a.cap + m.y;
                bulk_store(a.codes + slab_row * a.H, smem_u32(cb), uint32_t(a.H), pol);
                const int src_rank = int(tok / a.T);
                reinterpret_cast<int2*>(a.src_info)[slab_row] =
                    make_int2(src_rank, int(tok - int64_t(src_rank) * a.T));
            }
            bulk_commit();
        }
        ++used;
    }
    if (w == 0) bulk_wait<0>();
}

template <int FMT>
cudaError_t launch_fp8_bulk(const DispatchFp8Args& a, int64_t grid, int consumers, size_t smem, cudaStream_t stream) {
    const cudaError_t err =
        cudaFuncSetAttribute(dispatch_fp8_bulk_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    return launch_pdl(dispatch_fp8_bulk_kernel<FMT>, dim3(unsigned(grid)), dim3(32 * (1 + consumers)), smem, stream, a);
}

// Column-major scales: one 256-thread block per chunk of 256 slab rows of an
// expert; thread t owns the chunk's row t, finds its token in src_info and
// writes that token's scale words, so for each word the block's stores are
// contiguous.  With rows of at least kStageMinWords words (fp32 or power-of-two
// scales) the block first stages the chunk's tokens' scale rows in shared memory
// -- half-warps read whole rows, 16 bytes a lane where the rows allow it, all of
// a half-warp's rows in flight at once -- because each thread reading its own
// 224-byte row from global memory touched 32 rows per load and thrashed L1 (52
// against 34 us at prefill); shorter rows (UE8M0) are copied by each thread
// directly, kScaleBatch loads in flight before their stores (staging measured
// slower there: three barriers per chunk for a 56-byte row).
// A fixed grid of G blocks walks the non-empty chunks, numbered expert by expert
// (a prefix of the per-expert chunk counts, scanned in shared memory): block b
// takes chunks b, b + G, ...  (One block per possible chunk, (R*T/256) x E, was
// mostly blocks with no rows: 26 us at prefill for 15 MB of UE8M0 words.)
constexpr int kScaleRows = 256;               // rows per chunk = threads per block
constexpr int kStageRows = kScaleRows / 16;   // rows each half-warp stages
constexpr int kStageMinWords = 32;            // rows this long or longer are staged
constexpr int kScaleBatch = 16;               // words a thread loads before storing them (direct copy)

// Shared-memory words of a staged scale row: odd, so thread t reading word w of row t hits bank
// (t * stride + w) mod 32, a different bank for every lane.
__host__ __device__ __forceinline__ int scale_row_stride(int words) { return words | 1; }

size_t scale_writer_smem_bytes(int num_experts, int words, bool staged) {
    return size_t(num_experts + 1) * 4 + 32 * 4 +
           (staged ? size_t(kScaleRows) * 8 + size_t(kScaleRows) * scale_row_stride(words) * 4 : 0);
}

template <bool STAGED>
__global__ void __launch_bounds__(kScaleRows) fp8_scale_writer_kernel(DispatchFp8Args a) {
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits
    extern __shared__ __align__(16) unsigned char smem_raw[];
    int64_t* tok_of = reinterpret_cast<int64_t*>(smem_raw);                    // [kScaleRows], -1: no row
    uint32_t* staged = reinterpret_cast<uint32_t*>(tok_of + kScaleRows);       // [kScaleRows][stride]
    const int stride = scale_row_stride(a.words);
    // [E + 1] first chunk number of each expert, then [32] the warps' sums of the scan
    int32_t* first_chunk = STAGED ? reinterpret_cast<int32_t*>(staged + kScaleRows * stride)
                                  : reinterpret_cast<int32_t*>(smem_raw);
    int32_t* warp_sums = first_chunk + a.E + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // chunks per expert, scanned: thread t sums the experts [t*per, (t+1)*per), a scan over the
    // threads (warp shuffles, then the warps' sums), and each thread writes its experts' prefixes
    const int per = (a.E + kScaleRows - 1) / kScaleRows;
    const int e_begin = min(a.E, int(threadIdx.x) * per), e_end = min(a.E, e_begin + per);
    auto chunks_of = [&](int e) {
        const int64_t n = a.recv_count[e] < a.cap ? int64_t(a.recv_count[e]) : a.cap;
        return n > 0 ? int32_t((n + kScaleRows - 1) / kScaleRows) : 0;
    };
    int32_t mine = 0;
    for (int e = e_begin; e < e_end; ++e) mine += chunks_of(e);
    int32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int32_t before = 0;
    for (int w = 0; w < warp; ++w) before += warp_sums[w];
    int32_t run = before + incl - mine;
    for (int e = e_begin; e < e_end; ++e) {
        first_chunk[e] = run;
        run += chunks_of(e);
    }
    if (threadIdx.x == blockDim.x - 1) first_chunk[a.E] = run;
    __syncthreads();
    const int32_t total = first_chunk[a.E];

    for (int32_t id = int32_t(blockIdx.x); id < total; id += int32_t(gridDim.x)) {
        // the expert of chunk id: the last e with first_chunk[e] <= id
        int lo = 0, hi = a.E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (first_chunk[mid] <= id) lo = mid;
            else hi = mid - 1;
        }
        const int e = lo;
        const int64_t n = a.recv_count[e] < a.cap ? int64_t(a.recv_count[e]) : a.cap;
        const int64_t row = int64_t(id - first_chunk[e]) * kScaleRows + threadIdx.x;
        int64_t tok = -1;
        if (row < n) {
            const int2 src = reinterpret_cast<const int2*>(a.src_info)[int64_t(e) * a.cap + row];
            tok = int64_t(src.x) * a.T + src.y;
            // a recv_count that does not belong to this dispatch could point at a stale row
            if (!(src.y >= 0 && src.y < a.T && tok >= 0 && tok < a.n_tok)) {
                flag_status(a.status, EP_STATUS_BAD_EXPERT);
                tok = -1;
            }
        }
        if (!STAGED) {
            if (tok < 0) continue;
            const uint32_t* ts = a.tok_scales + tok * a.words;
            uint32_t* out = reinterpret_cast<uint32_t*>(a.scales) + int64_t(e) * a.words * a.cap + row;
            for (int w0 = 0; w0 < a.words; w0 += kScaleBatch) {
                uint32_t v[kScaleBatch];
#pragma unroll
                for (int jj = 0; jj < kScaleBatch; ++jj) v[jj] = w0 + jj < a.words ? __ldg(ts + w0 + jj) : 0u;
#pragma unroll
                for (int jj = 0; jj < kScaleBatch; ++jj)
                    if (w0 + jj < a.words) out[int64_t(w0 + jj) * a.cap] = v[jj];
            }
            continue;
        }
        tok_of[threadIdx.x] = tok;
        __syncthreads();
        // stage: half-warp h copies the scale rows of the chunk's rows h, h + 16, ..., all of its
        // kStageRows loads in flight before the shared-memory stores
        const int half = threadIdx.x >> 4, hl = threadIdx.x & 15;
        if ((a.words & 3) == 0 && (reinterpret_cast<uintptr_t>(a.tok_scales) & 15u) == 0) {
            for (int q = hl; q < (a.words >> 2); q += 16) {
                uint4 v[kStageRows];
#pragma unroll
                for (int rr = 0; rr < kStageRows; ++rr) {
                    const int64_t tr = tok_of[half + 16 * rr];
                    v[rr] = tr >= 0 ? __ldg(reinterpret_cast<const uint4*>(a.tok_scales + tr * a.words) + q)
                                    : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int rr = 0; rr < kStageRows; ++rr) {
                    uint32_t* dst = staged + (half + 16 * rr) * stride + 4 * q;
                    dst[0] = v[rr].x; dst[1] = v[rr].y; dst[2] = v[rr].z; dst[3] = v[rr].w;
                }
            }
        } else {
            for (int q = hl; q < a.words; q += 16) {
                uint32_t v[kStageRows];
#pragma unroll
                for (int rr = 0; rr < kStageRows; ++rr) {
                    const int64_t tr = tok_of[half + 16 * rr];
                    v[rr] = tr >= 0 ? __ldg(a.tok_scales + tr * a.words + q) : 0u;
                }
#pragma unroll
                for (int rr = 0; rr < kStageRows; ++rr) staged[(half + 16 * rr) * stride + q] = v[rr];
            }
        }
        __syncthreads();
        if (tok >= 0) {
            uint32_t* out = reinterpret_cast<uint32_t*>(a.scales) + int64_t(e) * a.words * a.cap + row;
            const uint32_t* src_row = staged + threadIdx.x * stride;
            for (int wd = 0; wd < a.words; ++wd) out[int64_t(wd) * a.cap] = src_row[wd];
        }
        __syncthreads();  // the staged rows are reused by the next chunk
    }
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" size_t ep_dispatch_fp8_workspace_bytes(ep_dims_t d, int32_t scale_format) {
    if (check_dims(d) != EP_OK || d.hidden % 128 != 0) return 0;
    const int words = scale_format == EP_FP8_SCALE_UE8M0 ? d.hidden / 512 : d.hidden / 128;
    return round_up16(size_t(d.num_ranks) * d.num_tokens * words * 4);
}

extern "C" int ep_dispatch_fp8(ep_dims_t d, const uint16_t* x, const int32_t* topk_idx, const int32_t* pair_row,
                               const int32_t* recv_count, int32_t scale_format, void* workspace,
                               size_t workspace_bytes, uint8_t* recv_x, void* recv_scales, int32_t* src_info,
                               int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_dispatch_fp8");
    int rc = check_dims(d);
    if (rc != EP_OK) return rc;
    if (scale_format != EP_FP8_SCALE_F32 && scale_format != EP_FP8_SCALE_POW2 && scale_format != EP_FP8_SCALE_UE8M0)
        return EP_ERR_INVALID;
    if (d.hidden % 128 != 0 || (scale_format == EP_FP8_SCALE_UE8M0 && d.hidden % 512 != 0)) return EP_ERR_INVALID;
    const int64_t RT = int64_t(d.num_ranks) * d.num_tokens;
    if (RT == 0) return EP_OK;
    if (!x || !topk_idx || !pair_row || !recv_count || !recv_x || !recv_scales || !src_info) return EP_ERR_INVALID;
    const size_t need = ep_dispatch_fp8_workspace_bytes(d, scale_format);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return EP_ERR_INVALID;
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(recv_x) & 7u) || (reinterpret_cast<uintptr_t>(recv_scales) & 3u) ||
        (reinterpret_cast<uintptr_t>(src_info) & 7u))
        return EP_ERR_INVALID;
    DispatchFp8Args a;
    a.x = reinterpret_cast<const uint8_t*>(x);
    a.topk_idx = topk_idx;
    a.pair_row = pair_row;
    a.codes = recv_x;
    a.scales = static_cast<uint8_t*>(recv_scales);
    a.src_info = src_info;
    a.status = status;
    a.T = d.num_tokens;
    a.k = d.num_topk;
    a.E = d.num_experts;
    a.H = d.hidden;
    a.groups = d.hidden / 128;
    a.words = scale_format == EP_FP8_SCALE_UE8M0 ? d.hidden / 512 : d.hidden / 128;
    a.tok_scales = static_cast<uint32_t*>(workspace);
    a.recv_count = recv_count;
    a.cap = RT;
    a.n_tok = RT;
    a.read_period_ns = 0;
    a.read_window_ns = 0;
    a.read_ahead = 0;
    const int sms = sm_count();
    if (sms <= 0) return EP_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cfg.variant != EP_VARIANT_AUTO && cfg.variant != EP_VARIANT_BULK && cfg.variant != EP_VARIANT_VECTOR &&
        cfg.variant != EP_VARIANT_PACED)
        return EP_ERR_INVALID;
    const bool bulk_fits = uint32_t(d.hidden) * 2 <= kFp8RowMax && aligned16(recv_x);
    if ((cfg.variant == EP_VARIANT_BULK || cfg.variant == EP_VARIANT_PACED) && !bulk_fits) return EP_ERR_UNSUPPORTED;
    // paced reads only when asked for: at prefill on B200 they did not pay here (UE8M0 437 against
    // 440 us; fp32 scales 605 against 491 us, the one-CTA-per-SM grid halving the casting warps)
    const bool paced = cfg.variant == EP_VARIANT_PACED;
    cudaError_t lerr;
    // AUTO: the bulk path, except fp32 scales on at most 1024 tokens, where the vector path's
    // finer units won on B200 (22.2 against 24.1 us at 8 ranks x 128 tokens; the bulk path leads
    // from 4096 tokens on: 68.6 against 77.9 us)
    const bool auto_vector = cfg.variant == EP_VARIANT_AUTO && scale_format == EP_FP8_SCALE_F32 && RT <= 1024;
    if (cfg.variant != EP_VARIANT_VECTOR && bulk_fits && !auto_vector) {
        // default 2 CTAs per SM (1 with paced reads, with a deeper ring); cfg.max_ctas sets the
        // grid.  W consumer warps split a row's 512-channel pieces evenly (7 at H = 7168, 8 at 4096).
        int64_t grid = cfg.max_ctas > 0 ? int64_t(cfg.max_ctas) : int64_t(sms) * (paced ? 1 : 2);
        grid = std::max<int64_t>(1, std::min<int64_t>(grid, RT));
        const int ctas_per_sm = int(std::max<int64_t>(1, ceil_div(grid, sms)));
        const int np = int(ceil_div(d.hidden, 512));
        // W consumer warps split a row's pieces evenly: by default at most kFp8DefaultConsumers
        // (7 at H = 7168: two pieces each); cfg.threads = 32 * (1 + W) asks for W of them
        const int want = cfg.threads >= 64 ? std::min(kFp8MaxConsumers, cfg.threads / 32 - 1) : kFp8DefaultConsumers;
        const int consumers = int(ceil_div(np, ceil_div(np, want)));
        const size_t stage_bytes = (size_t(d.hidden) * 2 + 127) & ~size_t(127);
        const size_t fixed = 2 * ((size_t(d.hidden) + 127) & ~size_t(127));  // two code rows
        const size_t per_stage = stage_bytes + 16 + 32 * 8;                    // row, two mbarriers, routing
        const long budget = long(max_smem_optin()) / ctas_per_sm - 1024 - long(fixed);
        int stages = cfg.stages > 0 ? cfg.stages : int(std::max(0L, budget) / long(per_stage));
        if (!paced && cfg.stages <= 0) stages = std::min(stages, 8);  // the unpaced path's measured ring
        if (paced && cfg.stages <= 0) stages = std::min(stages, 14);
        stages = std::max(2, std::min(kFp8MaxStages, stages));
        if (paced) {
            a.read_period_ns = kFp8PacePeriodNs;
            a.read_window_ns = kFp8PaceWindowNs;
            a.read_ahead = int(std::max<int64_t>(1, kFp8PaceAheadBytes / int64_t(stage_bytes)));
        }
        a.stages = stages;
        const size_t smem = size_t(stages) * per_stage + fixed;
        if (smem > size_t(max_smem_optin())) return EP_ERR_UNSUPPORTED;
        switch (scale_format) {
            case EP_FP8_SCALE_F32: lerr = launch_fp8_bulk<EP_FP8_SCALE_F32>(a, grid, consumers, smem, st); break;
            case EP_FP8_SCALE_POW2: lerr = launch_fp8_bulk<EP_FP8_SCALE_POW2>(a, grid, consumers, smem, st); break;
            default: lerr = launch_fp8_bulk<EP_FP8_SCALE_UE8M0>(a, grid, consumers, smem, st); break;
        }
    } else {
        const int64_t units = RT * ceil_div(d.hidden / 8, 64);
        int64_t grid = int64_t(sms) * 4;
        if (cfg.max_ctas > 0) grid = cfg.max_ctas;
        grid = std::max<int64_t>(1, std::min<int64_t>(grid, ceil_div(units, 8)));
        a.stages = 0;
        switch (scale_format) {
            case EP_FP8_SCALE_F32: lerr = launch_pdl(dispatch_fp8_kernel<EP_FP8_SCALE_F32>, dim3(unsigned(grid)), dim3(256), 0, st, a); break;
            case EP_FP8_SCALE_POW2: lerr = launch_pdl(dispatch_fp8_kernel<EP_FP8_SCALE_POW2>, dim3(unsigned(grid)), dim3(256), 0, st, a); break;
            default: lerr = launch_pdl(dispatch_fp8_kernel<EP_FP8_SCALE_UE8M0>, dim3(unsigned(grid)), dim3(256), 0, st, a); break;
        }
    }
    if (lerr != cudaSuccess) return EP_ERR_CUDA;
    // the scale writer: a fixed grid (three blocks per SM when staging, eight otherwise); the experts'
    // row counts, and the staged tokens and rows, in shared memory
    const bool staged = a.words >= kStageMinWords;
    const size_t writer_smem = scale_writer_smem_bytes(d.num_experts, a.words, staged);
    if (writer_smem > size_t(max_smem_optin())) return EP_ERR_UNSUPPORTED;
    auto writer = staged ? fp8_scale_writer_kernel<true> : fp8_scale_writer_kernel<false>;
    if (writer_smem > 48 * 1024 &&
        cudaFuncSetAttribute(writer, cudaFuncAttributeMaxDynamicSharedMemorySize, int(writer_smem)) != cudaSuccess)
        return EP_ERR_CUDA;
    const int64_t chunks = ceil_div(RT, kScaleRows) + d.num_experts;  // an upper bound on non-empty chunks
    const unsigned writer_grid =
        unsigned(std::max<int64_t>(1, std::min<int64_t>(int64_t(sms) * (staged ? 3 : 8), chunks)));
    if (launch_pdl(writer, dim3(writer_grid), dim3(kScaleRows), writer_smem, st, a) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}
