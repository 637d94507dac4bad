// decode.cu -- exl3_decode_tiles: trellis -> dense fp16 weights (the checking
// path).  Each warp decodes one 16x16 tile; lane u decodes the run of 8
// consecutive weights of tile row u/2, columns 8(u%2) .. 8(u%2)+7, i.e. the
// stream bits [64uK/8 ... ) -- every run starts on a byte.  The 8 weights are
// written as one 16-byte store.  Sources: EXL3 GEMM kernel article, sections
// 先看结论 / GEMM内核 (procedural codebook) and Viterbi编码内核剖析 (16x16
// tail-biting tiles packed as a 16-bit sequence).
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

template <int K>
__global__ void __launch_bounds__(256) decode_tiles_kernel(const uint16_t *__restrict__ trellis,
                                                           __half *__restrict__ w, int64_t k,
                                                           int64_t n)
{
    const int lane = threadIdx.x & 31;
    const int64_t tn_count = n >> 4;
    const int64_t tiles = (k >> 4) * tn_count;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < tiles;
         t += warps) {
        const uint32_t *tile = reinterpret_cast<const uint32_t *>(trellis + t * 16 * K);
        const int row = lane >> 1, half = lane & 1;
        uint32_t s[8];
        if constexpr (K <= 6) {
            run_states<K, 8>(tile, lane * 8 * K, s);
        } else {
            uint32_t a[4], b[4];
            run_states<K, 4>(tile, lane * 8 * K, a);
            run_states<K, 4>(tile, lane * 8 * K + 4 * K, b);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                s[j] = a[j];
                s[4 + j] = b[j];
            }
        }
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __half2 h2 = __halves2half2(codebook_weight(s[2 * j]), codebook_weight(s[2 * j + 1]));
            out[j] = *reinterpret_cast<uint32_t *>(&h2);
        }
        const int64_t tk = t / tn_count, tn = t - tk * tn_count;
        __half *dst = w + (tk * 16 + row) * n + tn * 16 + half * 8;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

typedef void (*decode_fn)(const uint16_t *, __half *, int64_t, int64_t);

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
    const int64_t tiles = (k / 16) * (n / 16);
    int64_t grid = (tiles + 7) / 8;
    if (grid > 148 * 16)
        grid = 148 * 16;
    decode_table(K)<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(trellis, (__half *)w, k, n);
    return launch_status();
}
