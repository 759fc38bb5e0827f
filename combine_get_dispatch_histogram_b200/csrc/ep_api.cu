// ep_api.cu -- library-wide entry points (error names, version) and the host
// helpers the launchers share (device queries, launch-error mapping).
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "ep.h"
#include "ep_host.h"

namespace ep {

namespace {
constexpr int kMaxDevices = 64;
// per-device caches; 0 = not asked yet (a race only repeats the same query)
std::atomic<int> g_sms[kMaxDevices] = {};
std::atomic<int> g_smem[kMaxDevices] = {};

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}
}  // namespace

int sm_count() {
    const int dev = current_device();
    if (dev < 0) return -1;
    int v = g_sms[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        g_sms[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

int max_smem_optin() {
    const int dev = current_device();
    if (dev < 0) return 48 * 1024;
    int v = g_smem[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return 48 * 1024;
        g_smem[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

int launch_result() { return cudaGetLastError() == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

}  // namespace ep

extern "C" const char* ep_strerror(int code) {
    switch (code) {
        case EP_OK: return "ok";
        case EP_ERR_INVALID: return "invalid argument (null or misaligned pointer, bad shape, small workspace)";
        case EP_ERR_UNSUPPORTED: return "shape outside the library limits";
        case EP_ERR_CUDA: return "CUDA runtime error";
        default: return "unknown error code";
    }
}

extern "C" const char* ep_version(void) { return "ep-b200 0.1.0 (sm_100a)"; }
