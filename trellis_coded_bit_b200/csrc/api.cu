// api.cu -- status strings, version, workspace status word and the wait-bound
// test hook of the EXL3 B200 library.
#include <atomic>

#include <cuda_runtime.h>

#include "../../include/exl3.h"
#include "../../include/exl3_debug.h"
#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

static std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
static std::atomic<unsigned> g_launch_flags{0u};

unsigned launch_flags()
{
    return g_launch_flags.load(std::memory_order_relaxed);
}

uint64_t wait_limit_ns()
{
    return g_wait_ns.load(std::memory_order_relaxed);
}

// SM count of the current device, looked up once per device (a read-only
// property of the hardware, so the cache never goes stale).
int num_sms()
{
    constexpr int kDevs = 64;
    static std::atomic<int> cache[kDevs];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    if (dev >= 0 && dev < kDevs) {
        const int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0)
            return v;
    }
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
        cudaGetLastError();
        v = 148;
    }
    if (dev >= 0 && dev < kDevs)
        cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

}  // namespace exl3

extern "C" const char *exl3_status_string(int status)
{
    switch (status) {
    case EXL3_OK: return "EXL3_OK";
    case EXL3_ERR_INVALID_ARG: return "EXL3_ERR_INVALID_ARG: null or misaligned pointer, or bad size/K";
    case EXL3_ERR_UNSUPPORTED: return "EXL3_ERR_UNSUPPORTED: request outside what this entry point handles";
    case EXL3_ERR_WORKSPACE: return "EXL3_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case EXL3_ERR_CUDA: return "EXL3_ERR_CUDA: a CUDA call or kernel launch failed";
    case EXL3_ERR_TIMEOUT: return "EXL3_ERR_TIMEOUT: a bounded device wait ran out";
    default: return "EXL3_ERR_UNKNOWN";
    }
}

extern "C" const char *exl3_version(void)
{
    return "exl3-b200 0.1 sm_100a";
}

extern "C" exl3_status exl3_workspace_status(void *workspace, size_t workspace_bytes, int clear,
                                             void *stream)
{
    if (!workspace || workspace_bytes < 4 || !exl3::aligned16(workspace))
        return EXL3_ERR_WORKSPACE;
    uint32_t word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return EXL3_ERR_CUDA;
    // the sync area every gemv/gemm workspace starts with (status word,
    // arrival counters)
    const size_t sync = workspace_bytes < 65536 ? workspace_bytes : 65536;
    if (clear && cudaMemsetAsync(workspace, 0, sync, s) != cudaSuccess)
        return EXL3_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return EXL3_ERR_CUDA;
    return word == exl3::kStatusOk ? EXL3_OK : (exl3_status)word;
}

extern "C" void exl3_debug_set_wait_limit_ns(uint64_t ns)
{
    exl3::g_wait_ns.store(ns ? ns : exl3::kDefaultWaitNs, std::memory_order_relaxed);
}

extern "C" uint64_t exl3_debug_wait_limit_ns(void)
{
    return exl3::wait_limit_ns();
}

extern "C" void exl3_set_launch_flags(unsigned flags)
{
    exl3::g_launch_flags.store(flags & EXL3_LAUNCH_PDL, std::memory_order_relaxed);
}

extern "C" unsigned exl3_launch_flags(void)
{
    return exl3::launch_flags();
}
