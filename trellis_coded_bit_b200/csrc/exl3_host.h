// exl3_host.h -- host-side helpers shared by the library's entry points:
// argument checks (all done before any launch) and launch error mapping.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/exl3.h"

namespace exl3 {

inline bool aligned16(const void *p)
{
    return ((uintptr_t)p & 15u) == 0;
}

inline bool ranges_overlap(const void *a, size_t an, const void *b, size_t bn)
{
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + bn && b0 < a0 + an;
}

// Bound of device-side waits in nanoseconds (see exl3_debug.h).
uint64_t wait_limit_ns();

// Process-wide launch options (EXL3_LAUNCH_PDL).
unsigned launch_flags();

// Streaming multiprocessors of the current device (looked up once).
int num_sms();

// Launches `kernel` with the library's launch options: with EXL3_LAUNCH_PDL
// the launch allows programmatic dependent launch (the kernel itself calls
// griddepcontrol.wait before touching anything but weights).
template <typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (launch_flags() & EXL3_LAUNCH_PDL) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

inline exl3_status launch_status()
{
    return cudaPeekAtLastError() == cudaSuccess ? EXL3_OK : EXL3_ERR_CUDA;
}

// Checks shared by gemv and gemm.  `max_m` <= 0 means unbounded.
inline exl3_status check_linear_args(const void *x, const uint16_t *trellis, const void *suh,
                                     const void *svh, const void *y, int64_t m, int64_t k,
                                     int64_t n, int K)
{
    if (!x || !trellis || !suh || !svh || !y)
        return EXL3_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(trellis) || !aligned16(suh) || !aligned16(svh) || !aligned16(y))
        return EXL3_ERR_INVALID_ARG;
    if (m < 1 || k < 128 || n < 128 || (k % 128) || (n % 128) || K < 1 || K > 8)
        return EXL3_ERR_INVALID_ARG;
    if (k > (int64_t)1 << 22 || n > (int64_t)1 << 22 || m > (int64_t)1 << 24)
        return EXL3_ERR_INVALID_ARG;
    if (ranges_overlap(x, (size_t)(m * k * 2), y, (size_t)(m * n * 2)))
        return EXL3_ERR_INVALID_ARG;
    return EXL3_OK;
}

}  // namespace exl3
