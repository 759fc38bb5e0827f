// ep_replica.cu -- replica weight sync and replica gradient reduction on sm_100a.
//
// The GPU operations of the GitDiagram page "dots-infra/ultraep architecture"
// around routing expansion: "Replica weight sync" copies each logical expert's
// master weights to its replicas before expert compute, and "Replica gradient
// reduction" sums the replicas' gradients into the master gradients in the
// backward pass.  Replica i of logical expert e is physical expert
// phys_base[e] + i, the numbering ep_reroute produces.
//
// Both are streaming kernels: block (x, e) owns a slice of expert e's
// parameters; weight sync reads each master vector once and stores it to every
// replica, gradient reduction reads the replicas' vectors and adds them in
// float32 in replica order.
#include <algorithm>
#include <cstdint>

#include "ep.h"
#include "ep_device.cuh"
#include "ep_host.h"

namespace ep {
namespace {

constexpr int kReplicaThreads = 256;
constexpr int kVecPerThread = 4;

__global__ void __launch_bounds__(kReplicaThreads)
    replica_weight_sync_kernel(const int32_t* phys_base, int32_t num_physical, int64_t nvec,
                               int32_t* status, const uint4* master, uint4* replicas) {
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits
    const int e = blockIdx.y;
    int32_t p0 = phys_base[e], p1 = phys_base[e + 1];
    if (p0 < 0 || p1 > num_physical || p0 > p1) {  // a malformed phys_base: touch nothing
        if (threadIdx.x == 0 && blockIdx.x == 0) flag_status(status, EP_STATUS_BAD_EXPERT);
        p0 = p1 = 0;
    }
    const int64_t v0 = (int64_t(blockIdx.x) * kReplicaThreads * kVecPerThread) + threadIdx.x;
    uint4 v[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
        const int64_t i = v0 + int64_t(u) * kReplicaThreads;
        if (i < nvec) v[u] = ld_stream_v4(master + int64_t(e) * nvec + i);
    }
    for (int32_t p = p0; p < p1; ++p) {
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
            const int64_t i = v0 + int64_t(u) * kReplicaThreads;
            if (i < nvec) st_global_v4(replicas + int64_t(p) * nvec + i, v[u]);
        }
    }
}

__global__ void __launch_bounds__(kReplicaThreads)
    replica_grad_reduce_kernel(const int32_t* phys_base, int32_t num_physical, int64_t nvec,
                               int32_t* status, const float4* grads, float4* master) {
    pdl_wait();  // nothing upstream is read before this
    // no early trigger: a streaming grid lets its dependent launch only as it exits
    const int e = blockIdx.y;
    int32_t p0 = phys_base[e], p1 = phys_base[e + 1];
    if (p0 < 0 || p1 > num_physical || p0 > p1) {  // a malformed phys_base: touch nothing
        if (threadIdx.x == 0 && blockIdx.x == 0) flag_status(status, EP_STATUS_BAD_EXPERT);
        p0 = p1 = 0;
    }
    const int64_t v0 = (int64_t(blockIdx.x) * kReplicaThreads * kVecPerThread) + threadIdx.x;
    float4 acc[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int32_t p = p0; p < p1; ++p) {
        float4 g[kVecPerThread];
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
            const int64_t i = v0 + int64_t(u) * kReplicaThreads;
            if (i < nvec) {
                const uint4 r = ld_stream_v4(grads + int64_t(p) * nvec + i);
                g[u] = make_float4(__uint_as_float(r.x), __uint_as_float(r.y), __uint_as_float(r.z),
                                   __uint_as_float(r.w));
            }
        }
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
            acc[u].x += g[u].x;
            acc[u].y += g[u].y;
            acc[u].z += g[u].z;
            acc[u].w += g[u].w;
        }
    }
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
        const int64_t i = v0 + int64_t(u) * kReplicaThreads;
        if (i < nvec) master[int64_t(e) * nvec + i] = acc[u];
    }
}

int check_replica_args(int32_t num_logical, int32_t num_physical, const int32_t* phys_base, int64_t bytes,
                       const void* src, const void* dst) {
    if (num_logical <= 0 || num_physical < num_logical || bytes < 0 || !phys_base) return EP_ERR_INVALID;
    if (num_logical > 65535) return EP_ERR_UNSUPPORTED;
    if (bytes % 16 != 0) return EP_ERR_INVALID;
    if (bytes > 0 && (!src || !dst || !aligned16(src) || !aligned16(dst))) return EP_ERR_INVALID;
    return EP_OK;
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" int ep_replica_weight_sync(int32_t num_logical, int32_t num_physical, const int32_t* phys_base,
                                      int64_t param_bytes, const void* master, void* replicas, int32_t* status,
                                      ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_replica_weight_sync");
    (void)cfg;
    const int rc = check_replica_args(num_logical, num_physical, phys_base, param_bytes, master, replicas);
    if (rc != EP_OK || param_bytes == 0) return rc;
    const int64_t nvec = param_bytes / 16;
    const int64_t blocks = ceil_div(nvec, int64_t(kReplicaThreads) * kVecPerThread);
    if (blocks > 0x7fffffff) return EP_ERR_UNSUPPORTED;
    if (launch_pdl(replica_weight_sync_kernel, dim3(unsigned(blocks), unsigned(num_logical)), dim3(kReplicaThreads), 0,
                   static_cast<cudaStream_t>(stream), phys_base, num_physical, nvec, status,
                   static_cast<const uint4*>(master), static_cast<uint4*>(replicas)) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}

extern "C" int ep_replica_grad_reduce(int32_t num_logical, int32_t num_physical, const int32_t* phys_base,
                                      int64_t num_params, const float* replica_grads, float* master_grads,
                                      int32_t* status, ep_cfg_t cfg, void* stream) {
    EP_NVTX_RANGE("ep_replica_grad_reduce");
    (void)cfg;
    if (num_params < 0) return EP_ERR_INVALID;
    const int rc = check_replica_args(num_logical, num_physical, phys_base, num_params * 4, replica_grads, master_grads);
    if (rc != EP_OK || num_params == 0) return rc;
    const int64_t nvec = num_params / 4;
    const int64_t blocks = ceil_div(nvec, int64_t(kReplicaThreads) * kVecPerThread);
    if (blocks > 0x7fffffff) return EP_ERR_UNSUPPORTED;
    if (launch_pdl(replica_grad_reduce_kernel, dim3(unsigned(blocks), unsigned(num_logical)), dim3(kReplicaThreads), 0,
                   static_cast<cudaStream_t>(stream), phys_base, num_physical, nvec, status,
                   reinterpret_cast<const float4*>(replica_grads), reinterpret_cast<float4*>(master_grads)) !=
        cudaSuccess)
        return EP_ERR_CUDA;
    return launch_result();
}
