// ep_layout_noalloc.cu -- ep_layout for callers that cannot allocate device memory.
//
// ep_layout needs a few megabytes of scratch (per-chunk expert histograms and
// per-chunk rank counts) that its caller normally allocates and passes in.
// Some callers have no way to do that: a plain C or C++ host without a
// framework allocator would have to call cudaMalloc, which synchronises the
// device and is not allowed on a hot path that runs under a fixed memory
// budget (for example a serving loop whose memory is all reserved up front).
// This entry point serves them: the scratch is a fixed-size array that is part
// of this library's device image, so the caller passes only inputs and
// outputs and nothing is allocated at call time.
//
// The array is reserved on every GPU that loads the library and stays
// reserved until the process exits.  All calls on one device share it and it
// keeps whatever the last call left there.  Like ep_layout's workspace, it
// must start zeroed (its first words carry the layout's barrier state from
// call to call): a static device array is zero when the library is loaded, and
// every call leaves that state ready for the next one, so nothing is cleared
// per call; the rest is scratch that each call writes before reading.  Two
// calls whose kernels overlap on the same GPU (different streams without
// ordering between them) would overwrite each other's scratch, so such calls
// must be ordered by the caller.
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "ep.h"
#include "ep_host.h"

namespace {

// Layout scratch, one copy per device (EP_LAYOUT_NOALLOC_SCRATCH_BYTES each).
static __device__ __align__(256) unsigned char g_layout_scratch[EP_LAYOUT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchAddress {
    unsigned long long context_id;  // context the address belongs to; 0 = not known
    void* address;
};
ScratchAddress g_scratch[kMaxDevices] = {};
std::mutex g_setup_mutex;

// Unique id of the calling thread's current CUDA context, or 0 when there is
// none or the driver cannot say.  The driver functions are reached through the
// runtime's entry-point query, so the library needs no link against libcuda.
// Caller holds g_setup_mutex.
unsigned long long current_context_id() {
    static bool looked_up = false;
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    if (!looked_up) {
        looked_up = true;
        cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", reinterpret_cast<void**>(&get_current), cudaEnableDefault,
                                    &q1) != cudaSuccess || q1 != cudaDriverEntryPointSuccess)
            get_current = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", reinterpret_cast<void**>(&get_id), cudaEnableDefault, &q2) !=
                cudaSuccess || q2 != cudaDriverEntryPointSuccess)
            get_id = nullptr;
        cudaGetLastError();
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the current device's copy of g_layout_scratch.  In host
// code the array's name only stands for the symbol; the address a kernel may
// use comes from cudaGetSymbolAddress, looked up with the device current on the
// first call and cached.  The cache is keyed by the context as well: after a
// cudaDeviceReset the device's next context holds a new, zeroed copy of the
// array at a new address, so the address is looked up again.
int current_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return EP_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchAddress& c = g_scratch[dev];
    const unsigned long long ctx = current_context_id();
    if (c.address == nullptr || (ctx != 0 && ctx != c.context_id)) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();  // leave no error behind for the caller's next launch check
            return EP_ERR_CUDA;
        }
        c.address = p;
        c.context_id = current_context_id();  // the lookup may have created the primary context
    }
    *out = c.address;
    return EP_OK;
}

}  // namespace

extern "C" int ep_layout_noalloc(ep_dims_t d, const int32_t* topk_idx, const uint8_t* active,
                                 int32_t* num_tokens_per_expert, int32_t* num_tokens_per_rank,
                                 uint8_t* is_token_in_rank, int32_t* recv_count, int32_t* expert_rank_offset,
                                 int32_t* pair_row, int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_layout_noalloc");
    const int rc = ep::check_dims(d);
    if (rc != EP_OK) return rc;
    const size_t need = ep_layout_workspace_bytes(d);
    if (need > size_t(EP_LAYOUT_NOALLOC_SCRATCH_BYTES)) return EP_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (need > 0) {
        const int src = current_scratch(&scratch);
        if (src != EP_OK) return src;
    }
    return ep_layout(d, topk_idx, active, scratch, need > 0 ? size_t(EP_LAYOUT_NOALLOC_SCRATCH_BYTES) : 0,
                     num_tokens_per_expert, num_tokens_per_rank, is_token_in_rank, recv_count,
                     expert_rank_offset, pair_row, status, cfg, stream);
}
