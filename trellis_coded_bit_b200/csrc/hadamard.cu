// hadamard.cu -- exl3_hadamard: blockwise 128-point Hadamard rotation with
// optional sign/scale vectors before and after (EXL3 GEMM kernel article,
// section GEMM内核: the input is rotated by a 128-point Hadamard transform
// before the dequantising matmul).
//
// One warp per (row, 128-column block): each lane loads 4 consecutive fp16
// (8 bytes, fully coalesced 256 B per warp), the butterflies run in fp32 in
// registers and through warp shuffles, the result is rounded once to fp16.
// HBM-bound: 4 bytes moved per element (+ the small pre/post vectors).
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

// x and y may be the same buffer (in place): each warp reads its block before
// writing it, so the pointers are deliberately not __restrict__.
__global__ void __launch_bounds__(256) hadamard_kernel(const __half *x, __half *y, int64_t rows,
                                                       int64_t cols, const __half *__restrict__ pre,
                                                       const __half *__restrict__ post)
{
    const int lane = threadIdx.x & 31;
    const int64_t blocks_per_row = cols >> 7;
    const int64_t total = rows * blocks_per_row;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total;
         w += warps) {
        const int64_t r = w / blocks_per_row;
        const int64_t c0 = (w - r * blocks_per_row) * 128 + lane * 4;
        const uint2 raw = *reinterpret_cast<const uint2 *>(x + r * cols + c0);
        const __half2 x01 = *reinterpret_cast<const __half2 *>(&raw.x);
        const __half2 x23 = *reinterpret_cast<const __half2 *>(&raw.y);
        float v[4] = {__low2float(x01), __high2float(x01), __low2float(x23), __high2float(x23)};
        if (pre) {
            const uint2 pr = *reinterpret_cast<const uint2 *>(pre + c0);
            const __half2 p01 = *reinterpret_cast<const __half2 *>(&pr.x);
            const __half2 p23 = *reinterpret_cast<const __half2 *>(&pr.y);
            v[0] *= __low2float(p01);
            v[1] *= __high2float(p01);
            v[2] *= __low2float(p23);
            v[3] *= __high2float(p23);
        }
        warp_fwht128(v);
        const float s = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            v[e] *= s;
        if (post) {
            const uint2 po = *reinterpret_cast<const uint2 *>(post + c0);
            const __half2 q01 = *reinterpret_cast<const __half2 *>(&po.x);
            const __half2 q23 = *reinterpret_cast<const __half2 *>(&po.y);
            v[0] *= __low2float(q01);
            v[1] *= __high2float(q01);
            v[2] *= __low2float(q23);
            v[3] *= __high2float(q23);
        }
        __half2 o01 = __floats2half2_rn(v[0], v[1]);
        __half2 o23 = __floats2half2_rn(v[2], v[3]);
        uint2 out;
        out.x = *reinterpret_cast<uint32_t *>(&o01);
        out.y = *reinterpret_cast<uint32_t *>(&o23);
        *reinterpret_cast<uint2 *>(y + r * cols + c0) = out;
    }
}

exl3_status launch_hadamard(const __half *x, __half *y, int64_t rows, int64_t cols,
                            const __half *pre, const __half *post, cudaStream_t stream)
{
    const int64_t work = rows * (cols / 128);
    if (work == 0)
        return EXL3_OK;
    int64_t grid = (work + 7) / 8;
    if (grid > 148 * 16)
        grid = 148 * 16;
    hadamard_kernel<<<(unsigned)grid, 256, 0, stream>>>(x, y, rows, cols, pre, post);
    return launch_status();
}

}  // namespace exl3

extern "C" exl3_status exl3_hadamard(const void *x, void *y, int64_t rows, int64_t cols,
                                     const void *pre, const void *post, void *stream)
{
    using namespace exl3;
    if (rows < 0 || cols <= 0 || (cols % 128))
        return EXL3_ERR_INVALID_ARG;
    if (rows == 0)
        return EXL3_OK;
    if (!x || !y || !aligned16(x) || !aligned16(y))
        return EXL3_ERR_INVALID_ARG;
    if ((pre && !aligned16(pre)) || (post && !aligned16(post)))
        return EXL3_ERR_INVALID_ARG;
    const size_t bytes = (size_t)(rows * cols * 2);
    if (x != y && ranges_overlap(x, bytes, y, bytes))
        return EXL3_ERR_INVALID_ARG;
    return launch_hadamard((const __half *)x, (__half *)y, rows, cols, (const __half *)pre,
                           (const __half *)post, (cudaStream_t)stream);
}
