/*
 * ep.h -- C ABI of the B200 (sm_100a) expert-parallel dispatch / combine library.
 *
 * The library moves MoE tokens between R expert-parallel ranks that live as
 * R slabs of ONE GPU's memory ("emulated ranks"): rank r owns token rows
 * x[r], routing topk_idx[r] / topk_weights[r], output rows out[r], and the
 * experts [r*E_local, (r+1)*E_local) with E_local = num_experts / num_ranks.
 * Sending a row to rank d is a store into d's receive slab; there is no peer
 * access and no collective.
 *
 * Operations and where they are defined:
 *   ep_layout   -- Buffer.get_dispatch_layout of the NeMo AutoModel page
 *                  "nemo_automodel.components.moe.uccl_ep.buffer"
 *                  (num_tokens_per_rank, is_token_in_rank,
 *                  num_tokens_per_expert), plus the communication handle that
 *                  Buffer.dispatch returns and Buffer.low_latency_combine
 *                  consumes (here: pair_row, expert_rank_offset, recv_count).
 *   ep_dispatch -- Buffer.low_latency_dispatch with use_fp8=False on the same
 *                  page: bf16 rows into per-local-expert receive slabs
 *                  [num_local_experts, num_ranks * num_max_dispatch_tokens_per_rank,
 *                  hidden]; only some slab rows are valid.
 *   ep_combine  -- Buffer.low_latency_combine on the same page: reduce WITH
 *                  weights back to [num_tokens, hidden] bf16, -1 indices
 *                  supported; the active-rank mask is re-checked as in the
 *                  ai-dynamo/nixl PR "nixl_ep: Optimize low-latency NVLink
 *                  path" (combine active rank mask optimization).
 *   ep_reroute  -- load computation, placement planning and routing expansion
 *                  of the GitDiagram page "dots-infra/ultraep architecture"
 *                  (GPU operations), with the placement rule "add one replica
 *                  at a time to the expert with the largest load/replicas,
 *                  ties to the lowest id".
 *   ep_dispatch_fp8 -- Buffer.low_latency_dispatch with use_fp8=True (and its
 *                  round_scale / use_ue8m0 options) on the NeMo page.
 *   ep_normal_layout, ep_normal_dispatch, ep_normal_combine -- the normal
 *                  (high-throughput) Buffer.dispatch / Buffer.combine of the
 *                  NeMo page: one copy per destination rank, unweighted combine.
 *   ep_replica_weight_sync, ep_replica_grad_reduce -- "Replica weight sync" and
 *                  "Replica gradient reduction" of the UltraEP page.
 *   ep_layout_local, ep_dispatch_peer, ep_wait_peers, ep_signal_peers,
 *   ep_combine_peer (+ ep_peer_offsets, ep_peer_recv_count, ep_ipc_*) -- the
 *                  same low-latency dispatch / combine between processes that
 *                  each own one GPU, over NVLink peer memory (section at the end).
 *   ep_topk_idx_to_int32 -- the int64 topk_idx of the NeMo page's Buffer calls
 *                  in the int32 form of the nixl PR, saturating out-of-range ids.
 *   ep_layout_noalloc, ep_layout_path, the ep_diag_* instruments and the
 *                  *_workspace_bytes queries have
 *                  no counterpart on the pages; they serve callers of this
 *                  library (scratch without allocation, which path a call takes,
 *                  scratch sizes).
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer owned by the caller, except
 *     where noted.  The library never allocates, frees or synchronises: each
 *     call validates its arguments on the host, enqueues kernels on `stream`
 *     (a cudaStream_t, NULL = legacy default stream) and returns.
 *   - Arrays are dense, C-contiguous (row-major) with the shapes given below.
 *     bf16 tensors are passed as uint16_t bit patterns.  R = num_ranks,
 *     T = num_tokens (tokens per rank, = num_max_dispatch_tokens_per_rank),
 *     k = num_topk, E = num_experts, H = hidden, CAP = R*T (slab rows per
 *     expert).
 *   - topk_idx is int32 (the index width the nixl PR made the default);
 *     -1 means "no selection".  Routing held as int64 (the NeMo page's dtype)
 *     is converted once by ep_topk_idx_to_int32.  A pair (r,t,j) is LIVE when
 *     0 <= e = topk_idx[r,t,j] < E, active[r] != 0 and active[e/E_local] != 0:
 *     a masked rank neither sends nor receives.
 *   - Data errors never trap.  Kernels OR bits into *status (int32, device,
 *     zeroed by the caller): EP_STATUS_BAD_EXPERT (an id outside [-1, E);
 *     the pair is dropped), EP_STATUS_OVERFLOW (an expert received more than
 *     CAP rows; rows >= CAP are neither written nor read), EP_STATUS_TIMEOUT
 *     (a bounded wait gave up; outputs are incomplete).
 *   - Return value: EP_OK, or a negative EP_ERR_* code for an argument the
 *     host rejected (nothing was enqueued) or a launch the CUDA runtime
 *     refused.  ep_strerror() names every code.
 *   - Calls that share output buffers must be ordered by the caller (same
 *     stream, or events); calls on disjoint buffers may run concurrently.
 */
#ifndef EP_B200_EP_H
#define EP_B200_EP_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Host-side return codes. */
enum {
    EP_OK = 0,
    EP_ERR_INVALID = -1,      /* null/misaligned pointer, bad shape, workspace too small */
    EP_ERR_UNSUPPORTED = -2,  /* shape outside the limits below */
    EP_ERR_CUDA = -3          /* the CUDA runtime refused a launch or query */
};

/* Device status bits (OR-ed into *status). */
enum {
    EP_STATUS_BAD_EXPERT = 1,
    EP_STATUS_OVERFLOW = 2,
    EP_STATUS_TIMEOUT = 8
};

/* Limits checked on the host (EP_ERR_UNSUPPORTED beyond them). */
enum {
    EP_MAX_RANKS = 64,        /* is_token_in_rank is built from a 64-bit rank set */
    EP_MAX_TOPK = 32,         /* one lane per slot */
    EP_MAX_EXPERTS = 8192,    /* per-warp shared-memory histograms */
    EP_MAX_NORMAL_RANKS = 32  /* normal mode: one lane per destination rank */
};

/* Problem shape.  E % R == 0, H % 8 == 0 (rows move as 16-byte vectors),
 * 1 <= k <= min(E, EP_MAX_TOPK), R*T*k < 2^31.  T may be 0. */
typedef struct ep_dims {
    int32_t num_ranks;    /* R */
    int32_t num_tokens;   /* T, tokens per rank */
    int32_t num_topk;     /* k */
    int32_t num_experts;  /* E, physical experts over all ranks */
    int32_t hidden;       /* H, bf16 elements per token row */
} ep_dims_t;

/* Launch tuning (cf. Buffer.get_dispatch_config / get_combine_config and
 * num_sms on the NeMo page).  A zero field means "choose automatically". */
typedef struct ep_cfg {
    int32_t max_ctas;     /* CTAs of the row-moving kernels: the grid of dispatch (default 2
                             per SM, 1 on the paced path; ep_normal_dispatch 4 where a 4-way
                             split of shared memory leaves >= 6 staged rows or there are at most
                             32 rows per SM, else 2) and of the vector combine (default:
                             as many as fit at once); a cap for the bulk combine (default 1 per SM) */
    int32_t threads;      /* threads per CTA where the kernel allows a choice */
    int32_t stages;       /* shared-memory pipeline depth of dispatch / combine */
    int32_t variant;      /* dispatch / combine data path: EP_VARIANT_* */
} ep_cfg_t;

/* Paths of ep_layout (ep_cfg_t.variant); they compute the same result.  AUTO
 * takes, where it applies, SINGLE_CTA up to R*T*k = 2048 pairs, CLUSTER up to
 * 65536, else CHUNKED: the fastest on B200 in each range (graph replays: 8.6 us
 * at 1024 pairs; 10.6 us from 4096 to 16384 and 12.7 us at 32768 on the
 * cluster, against 16.8 us chunked). */
enum {
    EP_LAYOUT_CHUNKED = 1,    /* three launches over chunks of each rank's tokens; any shape */
    EP_LAYOUT_SINGLE_CTA = 2, /* one launch, one CTA; R <= 32, E <= 1024, R*T*k <= 32768 */
    EP_LAYOUT_FUSED = 3,      /* one cooperative launch with two grid barriers; needs the
                                 chunk grid to fit the device (else EP_ERR_UNSUPPORTED) */
    EP_LAYOUT_CLUSTER = 4,    /* one launch of a thread-block cluster of up to 16 CTAs that
                                 share their histograms through distributed shared memory;
                                 R <= 32, E <= 1024, R*T*k <= 65536 */
    EP_LAYOUT_LOOKBACK = 5    /* one ordinary launch, one CTA per chunk: each CTA publishes its
                                 chunk's histogram with a release flag and waits (bounded) only
                                 for the chunks before it; any shape whose chunk grid has at most
                                 255 chunks (every supported shape) */
};

/* Data paths of ep_dispatch / ep_combine (ep_cfg_t.variant). */
enum {
    EP_VARIANT_AUTO = 0,      /* the faster path for the shape, as measured on B200 */
    EP_VARIANT_BULK = 1,      /* rows staged in shared memory by bulk async copies */
    EP_VARIANT_VECTOR = 2,    /* rows moved through registers as 16-byte vectors */
    EP_VARIANT_PACED = 3      /* ep_dispatch, ep_normal_dispatch, ep_dispatch_fp8: the bulk path
                                 with paced reads -- one CTA per SM (two for ep_dispatch rows whose
                                 k stores add up to less than 96 KB), and the rows about to be
                                 staged are prefetched into L2 only inside a short window that
                                 recurs on the GPU-wide clock, so HBM serves reads in bursts and the
                                 row stores alone in between (the same bits).  AUTO takes it for
                                 ep_dispatch where it measured faster: a row's k stores add up to
                                 >= 96 KB and every SM has >= 32 rows (e.g. 8 x 4096 tokens, top-8,
                                 H = 7168), or 48-96 KB and >= 96 rows per SM (8 x 2048 tokens,
                                 top-6, H = 4096) */
};

/* Human-readable name of an EP_OK / EP_ERR_* code (static storage). */
EP_API const char *ep_strerror(int code);

/* Library version string (static storage). */
EP_API const char *ep_version(void);

/* Bytes of device workspace ep_layout needs for `d` (0 for an invalid shape). */
EP_API size_t ep_layout_workspace_bytes(ep_dims_t d);

/*
 * ep_layout_path -- the path (EP_LAYOUT_*) ep_layout takes for these dims and
 * cfg.variant, so a caller can tell how many kernels a call launches (CHUNKED:
 * three; SINGLE_CTA, FUSED, CLUSTER: one).  The pages have no counterpart: it only
 * reports this library's own choice.  Returns EP_ERR_INVALID for bad dims or
 * an unknown variant and EP_ERR_UNSUPPORTED when the requested path cannot take
 * the shape, exactly as ep_layout would; launches nothing.
 */
EP_API int ep_layout_path(ep_dims_t d, ep_cfg_t cfg);

/*
 * ep_diag_wait_timeout -- diagnostic of the bounded waits (the pages have no
 * counterpart).  One CTA enters the grid barrier of the fused layout path as if
 * the grid had two CTAs, so it waits for a flag that nothing sets; after the
 * library's wait limit (2 s) it gives up, ORs EP_STATUS_TIMEOUT into *status and
 * returns.  Nothing faults or hangs and the context stays usable: this shows
 * how every bounded wait of the library ends.
 * in:  flags   >= 16 bytes of device memory, 8-byte aligned, zero-filled (a
 *              nonzero second word, 1 or 2, lets the wait pass at once)
 * out: status  int32 device word
 */
EP_API int ep_diag_wait_timeout(void *flags, int32_t *status, void *stream);

/*
 * ep_diag_dispatch_ceiling -- a measurement instrument (the pages have no
 * counterpart): the paced dispatch kernel (EP_VARIANT_PACED's grid and ring)
 * with its row loads left out, to time what HBM gives the dispatch's traffic
 * when no store waits for a read.
 *   mode 0: only the row stores and src_info of every live pair, from a zeroed
 *           ring -- the ceiling of the scatter's writes alone;
 *   mode 1: those stores plus the paced L2 prefetches of the token rows -- the
 *           dispatch's own HBM traffic with no store waiting on it.
 * Arguments and checks as ep_dispatch; the slab rows it writes hold zeros, not
 * tokens, and src_info holds the true (src_rank, src_token).
 */
EP_API int ep_diag_dispatch_ceiling(ep_dims_t d, const uint16_t *x, const int32_t *topk_idx,
                                    const int32_t *pair_row, uint16_t *recv_x, int32_t *src_info, int32_t mode,
                                    int32_t *status, ep_cfg_t cfg, void *stream);


/*
 * ep_topk_idx_to_int32 -- routing ids in the page's int64 form to the int32
 * form every other entry point reads.
 *
 * Buffer.get_dispatch_layout and Buffer.dispatch on the NeMo AutoModel page
 * "nemo_automodel.components.moe.uccl_ep.buffer" take topk_idx as
 * torch.int64; the ai-dynamo/nixl PR "nixl_ep: Optimize low-latency NVLink
 * path" made 32-bit indices the default, which this library uses.
 * in:  topk_idx64 int64 [n]   8-byte aligned
 * out: topk_idx32 int32 [n]   4-byte aligned; every element written
 * Each id is converted with saturation: -1 and every id in [-2^31, 2^31) keep
 * their value, larger ids become 2^31 - 1 and smaller ones -2^31.  Both
 * saturated values lie outside [-1, E) for every supported E, so the layout,
 * dispatch, combine and reroute kernels drop those pairs and raise
 * EP_STATUS_BAD_EXPERT instead of sending a wrapped id to a real expert.
 * One launch on `stream`; n == 0 enqueues nothing.
 */
EP_API int ep_topk_idx_to_int32(const int64_t *topk_idx64, int32_t *topk_idx32, int64_t n, void *stream);

/*
 * ep_layout -- per-expert / per-rank histogram, prefix sums and stable rows.
 *
 * in:
 *   topk_idx              int32 [R,T,k]
 *   active                uint8 [R]       active-rank mask at dispatch time
 *   workspace             >= ep_layout_workspace_bytes(d) bytes, 16-byte aligned,
 *                         owned by the caller.  Zero-fill it once before its first
 *                         use (e.g. cudaMemset) and keep it for ep_layout calls
 *                         only: its first 64 KiB carry barrier state from call to
 *                         call (cf. Buffer.clean_low_latency_buffer on the NeMo
 *                         page); the rest is scratch.  Calls sharing a workspace
 *                         must be ordered on the GPU.  After a call whose status
 *                         has EP_STATUS_TIMEOUT, zero-fill those 64 KiB again
 *                         before the next call: a chunk that started after the
 *                         wait limit can leave a flag that the next call would
 *                         take for its own.
 * out (every element written):
 *   num_tokens_per_expert int32 [R,E]     live pairs of source rank r on expert e
 *   num_tokens_per_rank   int32 [R,R]     tokens of r with >= 1 live pair on rank d
 *   is_token_in_rank      uint8 [R,T,R]   0/1
 *   recv_count            int32 [E]       rows expert e receives (valid rows are
 *                                         [0, min(recv_count[e], CAP)))
 *   expert_rank_offset    int32 [E,R]     first row of source rank r inside expert e
 *                                         = sum over r' < r of num_tokens_per_expert[r'][e]
 *   pair_row              int32 [R,T,k]   slab row of each live pair, -1 if not live
 * The row of a live pair is its position among expert e's live pairs taken in
 * (source rank, token, slot) order, so each expert's rows are ordered by
 * (src_rank, token) and the result is unique (bit-exact, deterministic).
 */
EP_API int ep_layout(ep_dims_t d, const int32_t *topk_idx, const uint8_t *active,
              void *workspace, size_t workspace_bytes,
              int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
              uint8_t *is_token_in_rank, int32_t *recv_count,
              int32_t *expert_rank_offset, int32_t *pair_row,
              int32_t *status, ep_cfg_t cfg, void *stream);

/* Scratch that ep_layout_noalloc keeps inside the library: 4 MiB per GPU. */
enum { EP_LAYOUT_NOALLOC_SCRATCH_BYTES = 4 * 1024 * 1024 };

/*
 * ep_layout_noalloc -- ep_layout for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot hand ep_layout a workspace: a C or C++ host with no framework
 * allocator would need cudaMalloc, which synchronises the device and is ruled
 * out on hot paths that run under a fixed, pre-reserved memory budget.
 * Arguments, outputs and results are those of ep_layout without the
 * workspace: the scratch is a fixed array of EP_LAYOUT_NOALLOC_SCRATCH_BYTES
 * inside the library's device image, one per GPU that loads the library,
 * held until the process exits.  Nothing is allocated at call time.
 *   - Shapes whose ep_layout_workspace_bytes(d) exceeds
 *     EP_LAYOUT_NOALLOC_SCRATCH_BYTES are rejected with EP_ERR_UNSUPPORTED
 *     before anything is enqueued (prefill shape R=8, T=4096, E=256 needs
 *     1.08 MB).
 *   - The first call on a device looks up that device's scratch address
 *     (cudaGetSymbolAddress with the device current) and caches it; make
 *     that first call before any stream capture.  EP_ERR_CUDA if the lookup
 *     fails.  The cache is per context: after a cudaDeviceReset the next
 *     call looks the address up again (the new context's copy of the array
 *     starts zeroed, as the barrier state requires).
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents.  It is zero when the library is loaded, as the layout's
 *     barrier state requires, and every call leaves that state ready for the
 *     next, so nothing is cleared per call.  Calls whose kernels may overlap
 *     on the same GPU race on it: order them (one stream, or events).
 *   - After a call whose status has EP_STATUS_TIMEOUT the array's barrier
 *     state may be left for the next call to misread, and it cannot be
 *     cleared from outside: use ep_layout with a workspace on that device
 *     from then on.
 */
EP_API int ep_layout_noalloc(ep_dims_t d, const int32_t *topk_idx, const uint8_t *active,
              int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
              uint8_t *is_token_in_rank, int32_t *recv_count,
              int32_t *expert_rank_offset, int32_t *pair_row,
              int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * ep_dispatch -- scatter token rows into the experts' receive slabs.
 *
 * in:
 *   x          bf16 [R,T,H]     16-byte aligned
 *   topk_idx   int32 [R,T,k]
 *   pair_row   int32 [R,T,k]    from ep_layout on the same topk_idx / active
 * out:
 *   recv_x     bf16 [E,CAP,H]   16-byte aligned; rank d's low-latency slab
 *                               [E_local, CAP, H] is recv_x[d*E_local : (d+1)*E_local].
 *                               Row pair_row[r,t,j] of expert topk_idx[r,t,j]
 *                               receives x[r,t,:] bit for bit; other rows are
 *                               left untouched.
 *   src_info   int32 [E,CAP,2]  (src_rank, src_token) of every written row;
 *                               other rows untouched.
 * Each token row is read from HBM once however many experts it goes to.
 */
EP_API int ep_dispatch(ep_dims_t d, const uint16_t *x, const int32_t *topk_idx,
                const int32_t *pair_row, uint16_t *recv_x, int32_t *src_info,
                int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * ep_dispatch_path -- the data path (EP_VARIANT_BULK, _VECTOR or _PACED) that
 * ep_dispatch takes for these dims and cfg.variant on the current device (AUTO
 * resolved); EP_ERR_* as ep_dispatch would return for bad dims or variant.  The
 * pages have no counterpart: it reports this library's choice.  Launches nothing.
 */
EP_API int ep_dispatch_path(ep_dims_t d, ep_cfg_t cfg);

/* Scale formats of ep_dispatch_fp8 (NeMo page, Buffer.low_latency_dispatch:
 * use_fp8, round_scale, use_ue8m0). */
enum {
    EP_FP8_SCALE_F32 = 0,   /* float scale per 128 channels = amax / 448 (1 if amax == 0) */
    EP_FP8_SCALE_POW2 = 1,  /* float scale 2^ceil(log2(amax / 448)), exponent clamped to [-127, 127] */
    EP_FP8_SCALE_UE8M0 = 2  /* the POW2 scales as UE8M0 bytes (exponent + 127), four per int32 */
};

/*
 * ep_dispatch_fp8 -- ep_dispatch with the payload cast to float8 e4m3.
 *
 * Buffer.low_latency_dispatch with use_fp8=True on the NeMo page: every live
 * pair's token row arrives as e4m3 codes with one scale per 128 channels.
 * Per group of 128 channels of a token row: amax = max |x|; scale per
 * scale_format (above); code = e4m3(x / scale), the division in float32 and
 * the cast rounding to nearest even, saturating at +-448.
 * in:
 *   x, topk_idx, pair_row   as for ep_dispatch; H % 128 == 0 (H % 512 == 0 for UE8M0)
 *   recv_count   int32 [E]  from ep_layout (which slab rows are valid)
 *   workspace    >= ep_dispatch_fp8_workspace_bytes(d, scale_format) bytes, 16-byte
 *                aligned; scratch (contents ignored on entry, undefined on return)
 * out:
 *   recv_x       uint8 [E,CAP,H]   e4m3 codes of every written row (8-byte aligned;
 *                16-byte aligned for the bulk path)
 *   recv_scales  EP_FP8_SCALE_F32 / _POW2: float [E, H/128, CAP];
 *                EP_FP8_SCALE_UE8M0: int32 [E, H/512, CAP], byte j of word w is the
 *                UE8M0 scale of channel group 4w+j.  This is the [E, CAP, groups]
 *                tensor of the page stored column-major in its last two dimensions.
 *   src_info     as for ep_dispatch
 * Rows not written keep their contents.  Two launches: the cast (codes to every
 * live row, each token's scales once to the workspace), then a scale writer that
 * fills the column-major scale tensor with coalesced stores.
 * cfg.threads (bulk path): 32 * (1 + W) asks for W casting warps per CTA (1 to 16; default:
 * up to 8, split evenly over the row's 512-channel pieces).
 * cfg.variant: EP_VARIANT_BULK stages each bf16 row in shared memory with a bulk
 * copy and bulk-stores the code rows (needs 2*H <= 16384 and a 16-byte aligned
 * recv_x, else EP_ERR_UNSUPPORTED); EP_VARIANT_VECTOR moves rows through
 * registers; EP_VARIANT_AUTO takes the bulk path when it applies, except with
 * fp32 scales on at most 1024 tokens (R*T), where the vector path is faster.
 * Both give the same bits.
 */
EP_API int ep_dispatch_fp8(ep_dims_t d, const uint16_t *x, const int32_t *topk_idx,
                           const int32_t *pair_row, const int32_t *recv_count,
                           int32_t scale_format, void *workspace, size_t workspace_bytes,
                           uint8_t *recv_x, void *recv_scales, int32_t *src_info,
                           int32_t *status, ep_cfg_t cfg, void *stream);

/* Bytes of scratch ep_dispatch_fp8 needs: each token's scales, row-major. */
EP_API size_t ep_dispatch_fp8_workspace_bytes(ep_dims_t d, int32_t scale_format);

/*
 * ep_combine -- top-k weighted gather-reduce back to the source ranks.
 *
 * in:
 *   y            bf16 [E,CAP,H]  16-byte aligned expert outputs (rows as laid out
 *                                by ep_dispatch; may be recv_x itself, zero copy)
 *   topk_idx     int32 [R,T,k]
 *   topk_weights float [R,T,k]
 *   pair_row     int32 [R,T,k]   from ep_layout
 *   active       uint8 [R]       mask at combine time (may differ from dispatch)
 * out:
 *   out          bf16 [R,T,H]    16-byte aligned, every element written:
 *     out[r,t,:] = bf16_rne( sum over j = 0..k-1, in that order, of
 *                  w[r,t,j] * y[e][pair_row[r,t,j]][:] )   (float32 accumulate)
 *     taking only slots with pair_row >= 0, pair_row < CAP, e in range and
 *     active[e/E_local]; rows of a source rank with active[r] == 0 are zeros.
 */
EP_API int ep_combine(ep_dims_t d, const uint16_t *y, const int32_t *topk_idx,
               const float *topk_weights, const int32_t *pair_row,
               const uint8_t *active, uint16_t *out,
               int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * Normal (high-throughput) mode -- Buffer.dispatch / Buffer.combine of the NeMo
 * page: a token goes ONCE to every rank it has a live expert on
 * (is_token_in_rank) and combine adds the returned rows WITHOUT weights.
 * Rank d's receive buffer holds recv_capacity rows (the page's
 * num_worst_tokens; R*T can never overflow); its received tokens are ordered
 * by (source rank, token).  R <= EP_MAX_NORMAL_RANKS.
 *
 * ep_normal_layout -- receive rows from ep_layout's outputs.
 * in:  is_token_in_rank uint8 [R,T,R], num_tokens_per_rank int32 [R,R],
 *      recv_count int32 [E] (all from ep_layout), expert_alignment >= 1
 * out: token_recv_row int32 [R,T,R]  row of (r,t) in rank d's buffer, -1 if not sent
 *      recv_tokens    int32 [R]      tokens rank d receives (rows >= recv_capacity are
 *                                    flagged EP_STATUS_OVERFLOW and never written)
 *      num_recv_tokens_per_expert int32 [E]  recv_count rounded up to a multiple of
 *                                    expert_alignment (the page's per-expert list)
 */
EP_API int ep_normal_layout(ep_dims_t d, int32_t recv_capacity, int32_t expert_alignment,
                            const uint8_t *is_token_in_rank, const int32_t *num_tokens_per_rank,
                            const int32_t *recv_count, int32_t *token_recv_row,
                            int32_t *recv_tokens, int32_t *num_recv_tokens_per_expert,
                            int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * ep_normal_dispatch -- send each token row once per destination rank (the bulk data path;
 * cfg.variant EP_VARIANT_PACED paces its reads, AUTO does so for long dispatches, any other
 * value runs it unpaced).
 * in:  x bf16 [R,T,H], topk_idx int32 [R,T,k], topk_weights float [R,T,k], active uint8 [R]
 *      (the mask ep_layout used), token_recv_row from ep_normal_layout
 * out (rows [0, min(recv_tokens[d], recv_capacity)) of every rank d; others untouched):
 *      recv_x            bf16 [R, recv_capacity, H]
 *      recv_topk_idx     int32 [R, recv_capacity, k]  local expert id (e - d*E_local) where the
 *                                                     slot's live expert is on rank d, else -1
 *      recv_topk_weights float [R, recv_capacity, k]  the slot's weight there, else 0
 *      src_info          int32 [R, recv_capacity, 2]  (src_rank, src_token)
 */
EP_API int ep_normal_dispatch(ep_dims_t d, int32_t recv_capacity, const uint16_t *x,
                              const int32_t *topk_idx, const float *topk_weights,
                              const uint8_t *active, const int32_t *token_recv_row,
                              uint16_t *recv_x, int32_t *recv_topk_idx, float *recv_topk_weights,
                              int32_t *src_info, int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * ep_normal_combine -- unweighted reduce of the returned rows.
 * in:  y bf16 [R, recv_capacity, H] (rank d's processed received tokens), token_recv_row,
 *      active uint8 [R] (mask at combine time)
 * out: out bf16 [R,T,H]: out[r,t] = bf16_rne(sum over d = 0..R-1, in that order, of
 *      y[d][token_recv_row[r,t,d]]) in float32, over rows >= 0 and < recv_capacity with
 *      active[d]; zeros for a source rank with active[r] == 0.
 */
EP_API int ep_normal_combine(ep_dims_t d, int32_t recv_capacity, const uint16_t *y,
                             const int32_t *token_recv_row, const uint8_t *active, uint16_t *out,
                             int32_t *status, ep_cfg_t cfg, void *stream);

/* Paths of ep_reroute (ep_cfg_t.variant); they compute the same result.  AUTO
 * takes CLUSTER. */
enum {
    EP_REROUTE_TWO_LAUNCH = 1, /* count per CTA into the workspace, then sum, plan and expand */
    EP_REROUTE_CLUSTER = 2     /* one launch of a thread-block cluster of up to 16 CTAs that
                                  read each other's counts through distributed shared memory */
};

/* Bytes of device workspace ep_reroute needs (the two-launch path uses it; the
 * cluster path does not, but every call is checked against this size). */
EP_API size_t ep_reroute_workspace_bytes(int32_t num_ranks, int32_t num_tokens, int32_t num_topk,
                                  int32_t num_logical);

/*
 * ep_reroute -- logical expert load, greedy replica placement, routing expansion.
 *
 * in:
 *   topk_idx_logical int32 [R,T,k]   logical ids in [0, num_logical), or -1
 *   workspace        >= ep_reroute_workspace_bytes(...) bytes, 16-byte aligned
 * out:
 *   load           int32 [num_logical]      (token, slot) pairs per logical expert
 *   num_replicas   int32 [num_logical]      starts at 1; num_extra times, +1 for the
 *                                           expert with the largest load/replicas
 *                                           (exact integer compare, ties -> lowest id)
 *   phys_base      int32 [num_logical + 1]  exclusive prefix sum of num_replicas
 *   topk_idx_phys  int32 [R,T,k]            phys_base[e] + ((r*T + t) mod num_replicas[e]),
 *                                           -1 where the logical id is -1 or out of range
 * num_logical + num_extra physical experts result; ep_layout / ep_dispatch /
 * ep_combine then run with num_experts = num_logical + num_extra.
 */
EP_API int ep_reroute(int32_t num_ranks, int32_t num_tokens, int32_t num_topk,
               int32_t num_logical, int32_t num_extra,
               const int32_t *topk_idx_logical, void *workspace, size_t workspace_bytes,
               int32_t *load, int32_t *num_replicas, int32_t *phys_base,
               int32_t *topk_idx_phys, int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * Replica weight sync and replica gradient reduction -- the GPU operations of
 * the GitDiagram page "dots-infra/ultraep architecture" around routing
 * expansion.  Replica i of logical expert e is physical expert phys_base[e] + i
 * (phys_base int32 [num_logical + 1], device, from ep_reroute).
 *
 * ep_replica_weight_sync: replicas[phys_base[e] + i] = master[e] for every
 *   replica, as raw bytes.  master [num_logical, param_bytes], replicas
 *   [num_physical, param_bytes]; param_bytes % 16 == 0, 16-byte aligned.
 * ep_replica_grad_reduce: master_grads[e][j] = sum over the replicas of e, in
 *   replica order, of replica_grads[p][j], accumulated in float32.
 *   replica_grads float [num_physical, num_params], master_grads float
 *   [num_logical, num_params]; num_params % 4 == 0, 16-byte aligned.
 */
EP_API int ep_replica_weight_sync(int32_t num_logical, int32_t num_physical, const int32_t *phys_base,
                                  int64_t param_bytes, const void *master, void *replicas,
                                  int32_t *status, ep_cfg_t cfg, void *stream);

EP_API int ep_replica_grad_reduce(int32_t num_logical, int32_t num_physical, const int32_t *phys_base,
                                  int64_t num_params, const float *replica_grads, float *master_grads,
                                  int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * ---------------------------------------------------------------------------
 * Expert parallelism across GPUs: one process per GPU, rank r of R.
 *
 * The low-latency dispatch / combine of the NeMo AutoModel page
 * "nemo_automodel.components.moe.uccl_ep.buffer" (Buffer.low_latency_dispatch,
 * Buffer.low_latency_combine; intranode NVLink) store token rows straight into
 * the destination rank's receive buffer and signal arrival with flags; the
 * ai-dynamo/nixl PR "nixl_ep: Optimize low-latency NVLink path" keeps a table of
 * peer pointers and an active-rank mask that lets the ranks that are still up
 * carry on.  The entry points below are that transport over NVLink / NVSwitch
 * peer memory.  One step, in stream order on every rank:
 *   1. ep_layout_local on the rank's own routing; the caller all-gathers the
 *      [E] num_tokens_per_expert of every rank into counts [R, E] (a collective
 *      of R * E int32, e.g. NCCL all_gather);
 *   2. ep_dispatch_peer: rows into every destination's slab, then a release flag;
 *   3. ep_wait_peers on the rank's arrival flags (bounded), ep_peer_recv_count;
 *   4. the experts run on the local slab and write their outputs;
 *   5. ep_signal_peers into every rank's "ready" flags, ep_wait_peers on the
 *      rank's own ready flags;
 *   6. ep_combine_peer gathers the weighted outputs back into the rank's tokens.
 * Receive layout: expert e (on rank d = e / E_local, local expert le) keeps its
 * rows in (source rank, token, slot) order in d's slab [E_local, CAP, H],
 * CAP = R * T: the row of source r's pair is expert_rank_offset[e][r] (from the
 * count matrix) + local_row, exactly the single-GPU layout of ep_layout.
 * Peer memory is touched only by plain 16-byte loads / stores and 8-byte
 * release / acquire flag accesses (no bulk copy, no multicast).  A masked rank
 * (active[d] == 0) is neither written, read, signalled nor waited for.  Signals
 * are 64-bit values that grow from step to step (a wait passes when the flag is
 * >= the value), so flag words never need clearing; zero them once.
 * ---------------------------------------------------------------------------
 */

/* Addresses, valid in the calling process, of every rank's buffers: device
 * arrays of num_ranks uint64 each (entry d = rank d's buffer; the caller's own
 * rank included).  Map peers' buffers with ep_ipc_export / ep_ipc_import. */
typedef struct ep_peer_table {
    const uint64_t *slab;      /* rank d's receive slab, bf16 [E_local, CAP, H], 16-byte aligned */
    const uint64_t *src_info;  /* rank d's src_info, int32 [E_local, CAP, 2] */
    const uint64_t *flags;     /* rank d's arrival flag words, uint64 [R]; word s is written by source s */
} ep_peer_table_t;

/* Bytes of the workspace ep_layout_local needs for `d` (0 for an invalid shape). */
EP_API size_t ep_layout_local_workspace_bytes(ep_dims_t d);

/*
 * ep_layout_local -- ep_layout over ONE source rank's routing (Buffer.get_dispatch_layout
 * as each rank of a real EP world runs it on its own tokens).
 * in:  rank                 this process's rank r
 *      topk_idx   int32 [T,k] rank r's routing
 *      active     uint8 [R]   the world's active-rank mask (pairs of a masked source or
 *                             destination are not live)
 *      workspace  >= ep_layout_local_workspace_bytes(d), 16-byte aligned, zeroed once
 *                 before first use, reserved for ep_layout_local calls (as for ep_layout)
 * out: num_tokens_per_expert int32 [E]   r's live pairs per expert (the row to all-gather)
 *      num_tokens_per_rank   int32 [R]   r's tokens with >= 1 live pair on rank d
 *      is_token_in_rank      uint8 [T,R]
 *      local_row             int32 [T,k] row of each live pair among r's live pairs of its
 *                                        expert, in (token, slot) order; -1 if not live
 */
EP_API int ep_layout_local(ep_dims_t d, int32_t rank, const int32_t *topk_idx, const uint8_t *active,
                           void *workspace, size_t workspace_bytes, int32_t *num_tokens_per_expert,
                           int32_t *num_tokens_per_rank, uint8_t *is_token_in_rank, int32_t *local_row,
                           int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * ep_peer_offsets -- HOST function (no GPU): from the all-gathered count matrix,
 * counts int32 [R,E] (host), the first row of source `rank` inside every expert,
 * expert_rank_offset int32 [E] (host) = sum over r' < rank of counts[r'][e], and
 * the rows each of `rank`'s experts receives, recv_count int32 [E/R] (host) =
 * sum over r' of counts[r'][rank * E/R + le].  For callers that bring the counts
 * to the host; the device path derives the same values inside its kernels.
 * EP_ERR_INVALID for bad arguments or a sum beyond int32.
 */
EP_API int ep_peer_offsets(int32_t num_ranks, int32_t num_experts, int32_t rank, const int32_t *counts,
                           int32_t *expert_rank_offset, int32_t *recv_count);

/* Bytes of workspace ep_dispatch_peer needs (a CTA-completion counter). */
EP_API size_t ep_dispatch_peer_workspace_bytes(void);

/*
 * ep_dispatch_peer -- send rank r's token rows to the experts' slabs on every rank.
 * in:  peers      the table above
 *      x          bf16 [T,H]   rank r's tokens, 16-byte aligned
 *      topk_idx   int32 [T,k], local_row int32 [T,k] (ep_layout_local on the same routing)
 *      counts     int32 [R,E]  device, every rank's num_tokens_per_expert (all-gathered)
 *      active     uint8 [R]    mask at dispatch time (masked destinations are skipped)
 *      signal     value released into word r of every active destination's flags after
 *                 the last row (use a value larger than every earlier step's)
 *      workspace  >= ep_dispatch_peer_workspace_bytes(), 8-byte aligned, zeroed once,
 *                 reserved for this rank's ep_dispatch_peer calls (ordered on the GPU)
 * out (in the destination ranks' memory): slab rows and src_info (src_rank, src_token)
 *      of every live pair; rows >= CAP are flagged EP_STATUS_OVERFLOW and not written.
 * A masked source (active[r] == 0) sends and signals nothing.  The call launches even
 * with T = 0, so the flags still go out.  cfg.max_ctas caps the grid (default: the CTAs
 * that fit at once); the other cfg fields are ignored.
 */
EP_API int ep_dispatch_peer(ep_dims_t d, int32_t rank, ep_peer_table_t peers, const uint16_t *x,
                            const int32_t *topk_idx, const int32_t *local_row, const int32_t *counts,
                            const uint8_t *active, uint64_t signal, void *workspace, size_t workspace_bytes,
                            int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * ep_wait_peers -- bounded wait until flags[s] >= signal for every active rank s.
 * flags uint64 [R] in this rank's memory (8-byte aligned).  Each wait gives up
 * after the library's wait limit (2 s): EP_STATUS_TIMEOUT is OR-ed into *status
 * and the kernel returns, so the context stays usable; kernels after it in the
 * stream then see the peers' writes only if no timeout was reported.
 * wait_ns int64 [R] (device, may be NULL): the nanoseconds spent waiting for each
 * source are ADDED to wait_ns[s] -- the page's dispatch_wait_recv_cost_stats (a
 * cumulative per-source wait time that localises a slow rank); masked sources add 0.
 */
EP_API int ep_wait_peers(int32_t num_ranks, const uint64_t *flags, uint64_t signal, const uint8_t *active,
                         int64_t *wait_ns, int32_t *status, void *stream);

/*
 * ep_signal_peers -- after the kernels before it in the stream, release `signal`
 * into word `rank` of every active rank d's flags; peer_flags is a device array of
 * R addresses (rank d's flag words).  Nothing is sent when rank itself is masked.
 */
EP_API int ep_signal_peers(int32_t num_ranks, int32_t rank, const uint64_t *peer_flags, const uint8_t *active,
                           uint64_t signal, void *stream);

/* recv_count int32 [E/R] (device) = rows each local expert of `rank` receives,
 * summed over the count matrix counts int32 [R,E] (device). */
EP_API int ep_peer_recv_count(int32_t num_ranks, int32_t num_experts, int32_t rank, const int32_t *counts,
                              int32_t *recv_count, void *stream);

/*
 * ep_combine_peer -- rank r's weighted gather of its tokens' expert outputs.
 * in:  y_slabs   device [R] addresses of every rank's expert outputs, bf16 [E_local, CAP, H]
 *                (rows as ep_dispatch_peer placed them)
 *      topk_idx, topk_weights float [T,k], local_row, counts, active (mask at combine time)
 * out: out bf16 [T,H] = bf16_rne(sum over j = 0..k-1 of w[t,j] * y[row of (t,j)]) in
 *      float32 from +0, over live slots whose destination is active; zeros if active[r] == 0.
 * cfg.threads = 2 gives each lane two 16-byte columns per unit (default one); cfg.max_ctas caps
 * the grid.  The bits are the same either way.
 */
EP_API int ep_combine_peer(ep_dims_t d, int32_t rank, const uint64_t *y_slabs, const int32_t *topk_idx,
                           const float *topk_weights, const int32_t *local_row, const int32_t *counts,
                           const uint8_t *active, uint16_t *out, int32_t *status, ep_cfg_t cfg, void *stream);

/*
 * ep_recv_stats_accumulate -- stats[i] += recv_count[i] for i < num (int32, device):
 * the page's cumulative_local_expert_recv_stats of Buffer.low_latency_dispatch, a
 * running per-expert receive count for EP load-balance monitoring.  Pass ep_layout's
 * recv_count (num = E) or ep_peer_recv_count's (num = E / R).
 */
EP_API int ep_recv_stats_accumulate(int32_t num, const int32_t *recv_count, int32_t *stats, void *stream);

/* CUDA IPC handles for the peer table: a handle is EP_IPC_HANDLE_BYTES of host memory. */
enum { EP_IPC_HANDLE_BYTES = 64 };

/* The IPC handle of the allocation that holds device pointer `ptr` and ptr's byte
 * offset inside it (host outputs), to send to the other ranks.  The allocation must be
 * an ordinary device allocation (cudaMalloc, or PyTorch's caching allocator without
 * expandable segments); virtual-memory-managed ones have no IPC handle (EP_ERR_CUDA). */
EP_API int ep_ipc_export(const void *ptr, void *handle, uint64_t *offset);

/* Map another process's exported buffer: *ptr = its address here, *base = the mapping
 * to pass to ep_ipc_close.  A process cannot import its own handles (CUDA refuses). */
EP_API int ep_ipc_import(const void *handle, uint64_t offset, void **ptr, void **base);

/* Unmap a buffer mapped by ep_ipc_import. */
EP_API int ep_ipc_close(void *base);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_EP_H */
