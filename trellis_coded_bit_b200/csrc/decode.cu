// decode.cu -- exl3_decode_tiles: trellis -> dense fp16 weights (the checking
// path).  Sources: EXL3 GEMM kernel article, sections 先看结论 / GEMM内核
// (procedural codebook) and Viterbi编码内核剖析 (16x16 tail-biting tiles
// packed as a 16-bit sequence).
//
// It runs the same row decoder as the GEMM's decoder warps (row_weights_f16:
// compile-time bit windows, codebook, fp16 RNE sum), so its bit-exact parity
// also pins the hot paths' window arithmetic.  A warp takes 4 tiles; in two
// passes (even rows, then odd rows, so that a pass's lanes share the row
// parity) lane l decodes row 2(l%8)+pass of tile l/8: 16 weights written as
// two 16-byte stores.
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

template <int K, int PAR>
__device__ __forceinline__ void decode_one_row(const uint32_t *tile, int row, const Codebook &cb, __half *dst)
{
    uint32_t raw[RowSpan<K, PAR>::N32];
    load_row<K, PAR>(tile, row, raw);
    uint32_t w[8];
    row_weights_f16<K, RowSpan<K, PAR>::P>(raw, cb, w);
    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

template <int K>
__global__ void __launch_bounds__(256) decode_tiles_kernel(const uint16_t *__restrict__ trellis,
                                                           __half *__restrict__ w, int64_t k,
                                                           int64_t n, const Codebook cb)
{
    const int lane = threadIdx.x & 31;
    const int64_t tn_count = n >> 4;
    const int64_t tiles = (k >> 4) * tn_count;
    const int64_t groups = (tiles + 3) >> 2;  // 4 tiles per warp
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t gi = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); gi < groups;
         gi += warps) {
        const int64_t t = gi * 4 + (lane >> 3);
        if (t >= tiles)
            continue;
        const uint32_t *tile = reinterpret_cast<const uint32_t *>(trellis + t * 16 * K);
        const int64_t tk = t / tn_count, tn = t - tk * tn_count;
        const int row0 = 2 * (lane & 7);
        __half *base = w + (tk * 16) * n + tn * 16;
        decode_one_row<K, 0>(tile, row0, cb, base + (int64_t)row0 * n);
        decode_one_row<K, 1>(tile, row0 + 1, cb, base + (int64_t)(row0 + 1) * n);
    }
}

typedef void (*decode_fn)(const uint16_t *, __half *, int64_t, int64_t, const Codebook);

static decode_fn decode_table(int K)
{
    switch (K) {
    case 1: return decode_tiles_kernel<1>;
    case 2: return decode_tiles_kernel<2>;
    case 3: return decode_tiles_kernel<3>;
    case 4: return decode_tiles_kernel<4>;
    case 5: return decode_tiles_kernel<5>;
    case 6: return decode_tiles_kernel<6>;
    case 7: return decode_tiles_kernel<7>;
    default: return decode_tiles_kernel<8>;
    }
}

}  // namespace exl3

extern "C" exl3_status exl3_decode_tiles(const uint16_t *trellis, void *w, int64_t k, int64_t n,
                                         int K, void *stream)
{
    using namespace exl3;
    if (!trellis || !w || !aligned16(trellis) || !aligned16(w))
        return EXL3_ERR_INVALID_ARG;
    if (k < 16 || n < 16 || (k % 16) || (n % 16) || K < 1 || K > 8)
        return EXL3_ERR_INVALID_ARG;
    if (ranges_overlap(trellis, (size_t)(k * n * K / 8), w, (size_t)(k * n * 2)))
        return EXL3_ERR_INVALID_ARG;
    const int64_t groups = ((k / 16) * (n / 16) + 3) / 4;
    int64_t grid = (groups + 7) / 8;
    if (grid > 148 * 16)
        grid = 148 * 16;
    decode_table(K)<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(trellis, (__half *)w, k, n,
                                                                    codebook_constants());
    return launch_status();
}
