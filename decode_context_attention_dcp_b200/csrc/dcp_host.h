// dcp_host.h -- host-side helpers shared by the library's translation units: the
// per-thread error text, launch-error reporting, occupancy queries, the dynamic
// shared-memory opt-in of each kernel instance, and the per-element-type combine
// dispatchers (one translation unit each, so that they compile in parallel).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "dcp_combine.h"
#include "dcp_kernels.cuh"

namespace dcp_host {

// Records the message as the calling thread's error text and returns status.
int32_t fail(int32_t status, const char *fmt, ...);

// Clears the calling thread's error text and returns DCP_OK.
int32_t ok();

// The calling thread's error text ("" after a successful call).
const char *last_error();

// DCP_OK, or DCP_ERR_CUDA with the launch error of the last kernel launch.
int32_t launch_status(const char *what);

// Multiprocessor count of the current device (cached per device).
int sm_count();

// Resident CTAs per SM of one kernel instance on the current device.
template <class K>
int resident_ctas(K kernel, int threads, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess || n <= 0) n = 1;
    return n;
}

// Per kernel instance and device: the dynamic shared-memory opt-in (once) and the
// resident-CTA count for the last shared-memory size seen.
struct InstanceCache {
    std::atomic<int> opted[64];
    std::atomic<uint64_t> occupancy[64];  // (smem << 16) | ctas
};

template <class K>
bool reserve_smem(K kernel, InstanceCache &ic, size_t max_bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (dev < 64 && ic.opted[dev].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_bytes) != cudaSuccess)
        return false;
    if (dev < 64) ic.opted[dev].store(1, std::memory_order_release);
    return true;
}

template <class K>
int cached_resident_ctas(K kernel, InstanceCache &ic, int threads, size_t smem) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return resident_ctas(kernel, threads, smem);
    const uint64_t c = ic.occupancy[dev].load(std::memory_order_relaxed);
    if (c && (c >> 16) == smem) return (int)(c & 0xffff);
    const int n = resident_ctas(kernel, threads, smem);
    ic.occupancy[dev].store(((uint64_t)smem << 16) | (uint64_t)n, std::memory_order_relaxed);
    return n;
}

// The combine of each element type: host-side shape choice and launch.  `packed`
// selects the packed-buffer kernels, else the split-layout ones (plain, per request
// or with packed output, as `a` asks).
int32_t dispatch_combine_bf16(const dcp::CombineArgs &a, bool packed, cudaStream_t stream);
int32_t dispatch_combine_fp16(const dcp::CombineArgs &a, bool packed, cudaStream_t stream);
int32_t dispatch_combine_fp32(const dcp::CombineArgs &a, bool packed, cudaStream_t stream);
// The split-layout half of each (its own translation unit).
int32_t dispatch_split_bf16(const dcp::CombineArgs &a, cudaStream_t stream);
int32_t dispatch_split_fp16(const dcp::CombineArgs &a, cudaStream_t stream);
int32_t dispatch_split_fp32(const dcp::CombineArgs &a, cudaStream_t stream);

}  // namespace dcp_host
