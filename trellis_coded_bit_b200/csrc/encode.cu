// encode.cu -- exl3_encode: tail-biting trellis encoding of a weight matrix,
// the write side of the format the GEMV/GEMM decode (EXL3 GEMM kernel
// article, section Viterbi编码内核剖析: a 16x16 weight block is encoded by a
// Viterbi forward pass over the trellis that keeps the accumulated cost of
// every path and takes the cheapest, and the tail-biting boundary is closed by
// enumerating start states).
//
// The search.  A weight's state is s_i = ((s_{i-1} << K) | c_i) mod 2^16 with
// c_i its K new bits, and the code is tail-biting (s_{-1} = s_255).  M_i[m] is
// the cheapest cost of a path through weight i whose state has low 16-K bits
// m -- exactly the states that can precede a state whose high 16-K bits are
// m -- so one step is
//     M_i[m] = min over h of  (w_i - cb(s))^2 + M_{i-1}[s >> K],
//              s = (h << (16-K)) | m,
// with the choice of h recorded for the trace-back.  Pass 1 lets every state
// start (M_{-1} = 0) and takes the cheapest end's low 16-K bits as the
// overlap o; pass 2 allows only starts whose high bits are o (M_{-1} = 0 at o,
// +inf elsewhere), ends in the cheapest state with low bits o and traces the
// path back, so its head and tail agree.  Costs are fp32, each weight's term
// added with one fused multiply-add, ties to the smallest index: the oracle
// takes the same decisions in the same precision, so the codes are bit-exact.
//
// B200 mapping (the pages' 512-thread block per tile is prior art):
//   * one CTA of 256 threads per tile, grid-stride over tiles; thread j owns
//     the entries m = j + 256q, so every min over h is thread-local;
//   * M ping-pongs in shared memory (2 x 2^(16-K) fp32, up to 128 KB at K = 2,
//     so smaller K leave room for more CTAs per SM); for K = 1 it would need
//     256 KB and lives in the CTA's workspace slot instead (L2);
//   * the codebook value of a state is computed on the fly, as in the decode
//     (the multiply stepped by one add across an entry's states, one LOP3,
//     an fp16 add);
//   * the recorded choices (one byte per entry and weight) go to the CTA's
//     workspace slot; one thread traces back, then the CTA packs the 16K
//     words in parallel.
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

constexpr int kEncThreads = 256;

template <int K>
struct EncShape {
    static constexpr int NM = 1 << (16 - K);          // entries of M
    static constexpr int PER = NM / kEncThreads;      // entries per thread
    static constexpr bool kGlobalM = K == 1;          // M in the workspace
    static constexpr size_t kChoiceBytes = (size_t)256 * NM;
    static constexpr size_t kSlotBytes = kChoiceBytes + (kGlobalM ? (size_t)2 * NM * 4 : 0);
    static constexpr size_t kSmem = (kGlobalM ? 0 : (size_t)2 * NM * 4) + 256 * 4 + 256 + 2 * 32 * 8;
};

// One step of the recursion over the thread's entries: prev -> next, choices
// to `choice` (a row of NM bytes) when RECORD.  The states of an entry m are
// s_h = (h << (16-K)) | m = m + h 2^(16-K), so their codebook products are
// v_h = v_0 + h (C1 << (16-K)) (mod 2^32), one add per state, and their
// predecessor costs sit at prev[(m >> K) + h 2^(16-2K)]: a per-m base plus a
// per-h constant offset.  The integer values are the same as in the plain
// formula, so the decisions are unchanged.
template <int K, bool RECORD>
__device__ __forceinline__ void enc_step(float wi, const float *prev, float *next, unsigned char *choice,
                                         const Codebook &cb, uint32_t dv)
{
    using Sh = EncShape<K>;
    const int j = threadIdx.x;
#pragma unroll 2
    for (int q = 0; q < Sh::PER; ++q) {
        const uint32_t m = (uint32_t)(j + kEncThreads * q);
        const float *pm = prev + (m >> K);
        uint32_t v = m * cb.mul + cb.add;
        float best = 0.f;
        int best_h = 0;
#pragma unroll(K <= 4 ? (1 << K) : 4)
        for (int h = 0; h < (1 << K); ++h) {
            const uint32_t w = (v & cb.mask) ^ cb.xr;
            const __half2 hw = *reinterpret_cast<const __half2 *>(&w);
            const float d = wi - __half2float(__hadd(__low2half(hw), __high2half(hw)));
            const float val = __fmaf_rn(d, d, pm[h << (16 - 2 * K)]);
            if (h == 0 || val < best) {
                best = val;
                best_h = h;
            }
            v += dv;
        }
        next[m] = best;
        if (RECORD)
            choice[m] = (unsigned char)best_h;
    }
}

template <int K>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(const float *__restrict__ w, uint16_t *trellis,
                                                             float *cost, int64_t k, int64_t n,
                                                             unsigned char *ws, Codebook cb)
{
    using Sh = EncShape<K>;
    constexpr int NM = Sh::NM;
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char *slot = ws + (size_t)blockIdx.x * Sh::kSlotBytes;
    unsigned char *choices = slot;
    float *bufA, *bufB;
    if constexpr (Sh::kGlobalM) {
        bufA = reinterpret_cast<float *>(slot + Sh::kChoiceBytes);
        bufB = bufA + NM;
    } else {
        bufA = reinterpret_cast<float *>(smem);
        bufB = bufA + NM;
    }
    float *target = reinterpret_cast<float *>(smem + (Sh::kGlobalM ? 0 : (size_t)2 * NM * 4));
    unsigned char *chunks = reinterpret_cast<unsigned char *>(target + 256);
    float *red_v = reinterpret_cast<float *>(chunks + 256);
    int *red_i = reinterpret_cast<int *>(red_v + 32);
    const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
    const int64_t tn_count = n / 16, tiles = (k / 16) * tn_count;
    const uint32_t dv = cb.mul << (16 - K);  // codebook-product step from state s to s + 2^(16-K)

    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t tk = tile / tn_count, tn = tile - tk * tn_count;
        target[j] = w[(tk * 16 + j / 16) * n + tn * 16 + (j & 15)];  // weight order i = 16 r + c
        int o = 0;
        for (int pass = 1; pass <= 2; ++pass) {
            float *prev = bufA, *next = bufB;
            for (int q = 0; q < Sh::PER; ++q) {
                const int m = j + kEncThreads * q;
                prev[m] = (pass == 1 || m == o) ? 0.f : __int_as_float(0x7f800000);
            }
            __syncthreads();
            for (int i = 0; i < 256; ++i) {
                if (pass == 1)
                    enc_step<K, false>(target[i], prev, next, nullptr, cb, dv);
                else
                    enc_step<K, true>(target[i], prev, next, choices + (size_t)i * NM, cb, dv);
                __syncthreads();
                float *t = prev;
                prev = next;
                next = t;
            }
            // 256 steps: the result is back in bufA
            if (pass == 1) {
                // o = argmin_m M_255[m], smallest m on ties
                float bv = prev[j];
                int bi = j;
                for (int q = 1; q < Sh::PER; ++q) {
                    const int m = j + kEncThreads * q;
                    if (prev[m] < bv) {
                        bv = prev[m];
                        bi = m;
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float ov = __shfl_down_sync(0xffffffffu, bv, off);
                    const int oi = __shfl_down_sync(0xffffffffu, bi, off);
                    if (ov < bv || (ov == bv && oi < bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
                if (lane == 0) {
                    red_v[warp] = bv;
                    red_i[warp] = bi;
                }
                __syncthreads();
                if (j == 0) {
                    for (int q = 1; q < kEncThreads / 32; ++q)
                        if (red_v[q] < bv || (red_v[q] == bv && red_i[q] < bi)) {
                            bv = red_v[q];
                            bi = red_i[q];
                        }
                    red_i[0] = bi;
                }
                __syncthreads();
                o = red_i[0];
                __syncthreads();
            }
        }
        // trace back from the cheapest last state with low bits o
        if (j == 0) {
            uint32_t s = ((uint32_t)choices[(size_t)255 * NM + o] << (16 - K)) | (uint32_t)o;
            chunks[255] = (unsigned char)(s & ((1u << K) - 1));
            for (int i = 255; i > 0; --i) {
                const uint32_t m = s >> K;
                s = ((uint32_t)choices[(size_t)(i - 1) * NM + m] << (16 - K)) | m;
                chunks[i - 1] = (unsigned char)(s & ((1u << K) - 1));
            }
            if (cost)
                cost[tile] = bufA[o];
        }
        __syncthreads();
        // pack: chunk c_i fills stream positions [iK, iK + K), most
        // significant bit first; word p / 16 holds position p at bit 15 - p % 16
        if (j < 16 * K) {
            uint32_t word = 0;
#pragma unroll
            for (int b = 0; b < 16; ++b) {
                const int p = 16 * j + b;
                word |= (uint32_t)((chunks[p / K] >> (K - 1 - p % K)) & 1) << (15 - b);
            }
            trellis[tile * 16 * K + j] = (uint16_t)word;
        }
        __syncthreads();  // target, chunks and the buffers are reused by the next tile
    }
}

struct EncPlan {
    int ctas;
    size_t smem, slot, total;
};

// Grid: resident CTAs per SM from the shared memory (228 KB per SM, 1 KB
// reserved per CTA), at most 4 (the kernel's registers allow that many at 256
// threads); at most ~1 GiB of workspace; no more CTAs than tiles.
template <int K>
static void enc_plan_t(int64_t tiles, EncPlan &pl)
{
    using Sh = EncShape<K>;
    pl.smem = Sh::kSmem;
    pl.slot = Sh::kSlotBytes;
    int64_t per_sm = (int64_t)(228 * 1024) / (int64_t)(pl.smem + 1024);
    per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
    int64_t G = per_sm * num_sms();
    const int64_t cap = ((int64_t)1 << 30) / (int64_t)pl.slot;
    if (G > cap)
        G = cap;
    if (G > tiles)
        G = tiles;
    if (G < 1)
        G = 1;
    pl.ctas = (int)G;
    pl.total = 256 + (size_t)G * pl.slot;
}

static void enc_plan(int K, int64_t tiles, EncPlan &pl)
{
    switch (K) {
    case 1: enc_plan_t<1>(tiles, pl); break;
    case 2: enc_plan_t<2>(tiles, pl); break;
    case 3: enc_plan_t<3>(tiles, pl); break;
    case 4: enc_plan_t<4>(tiles, pl); break;
    case 5: enc_plan_t<5>(tiles, pl); break;
    case 6: enc_plan_t<6>(tiles, pl); break;
    case 7: enc_plan_t<7>(tiles, pl); break;
    default: enc_plan_t<8>(tiles, pl); break;
    }
}

template <int K>
static cudaError_t enc_launch(const float *w, uint16_t *trellis, float *cost, int64_t k, int64_t n,
                              unsigned char *ws, const EncPlan &pl, cudaStream_t s)
{
    if (pl.smem > 48 * 1024) {
        const cudaError_t e =
            cudaFuncSetAttribute(encode_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
        if (e != cudaSuccess)
            return e;
    }
    encode_kernel<K><<<pl.ctas, kEncThreads, pl.smem, s>>>(w, trellis, cost, k, n, ws + 256, codebook_constants());
    return cudaGetLastError();
}

static bool enc_args_ok(int64_t k, int64_t n, int K)
{
    return k >= 16 && n >= 16 && k % 16 == 0 && n % 16 == 0 && K >= 1 && K <= 8 && k <= ((int64_t)1 << 22) &&
           n <= ((int64_t)1 << 22);
}

}  // namespace exl3

extern "C" size_t exl3_encode_workspace_size(int64_t k, int64_t n, int K)
{
    using namespace exl3;
    if (!enc_args_ok(k, n, K))
        return 0;
    EncPlan pl;
    enc_plan(K, (k / 16) * (n / 16), pl);
    return pl.total;
}

extern "C" exl3_status exl3_encode(const float *w, uint16_t *trellis, float *cost, int64_t k, int64_t n, int K,
                                   void *workspace, size_t workspace_bytes, void *stream)
{
    using namespace exl3;
    if (!w || !trellis || !aligned16(w) || !aligned16(trellis) || (cost && ((uintptr_t)cost & 3u)))
        return EXL3_ERR_INVALID_ARG;
    if (!enc_args_ok(k, n, K))
        return EXL3_ERR_INVALID_ARG;
    const size_t cost_bytes = (size_t)((k / 16) * (n / 16)) * 4;
    if (ranges_overlap(w, (size_t)(k * n * 4), trellis, (size_t)(k * n * K / 8)) ||
        (cost && (ranges_overlap(cost, cost_bytes, w, (size_t)(k * n * 4)) ||
                  ranges_overlap(cost, cost_bytes, trellis, (size_t)(k * n * K / 8)))))
        return EXL3_ERR_INVALID_ARG;
    EncPlan pl;
    enc_plan(K, (k / 16) * (n / 16), pl);
    if (!workspace || !aligned16(workspace) || workspace_bytes < pl.total)
        return EXL3_ERR_WORKSPACE;
    unsigned char *ws = (unsigned char *)workspace;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    switch (K) {
    case 1: e = enc_launch<1>(w, trellis, cost, k, n, ws, pl, s); break;
    case 2: e = enc_launch<2>(w, trellis, cost, k, n, ws, pl, s); break;
    case 3: e = enc_launch<3>(w, trellis, cost, k, n, ws, pl, s); break;
    case 4: e = enc_launch<4>(w, trellis, cost, k, n, ws, pl, s); break;
    case 5: e = enc_launch<5>(w, trellis, cost, k, n, ws, pl, s); break;
    case 6: e = enc_launch<6>(w, trellis, cost, k, n, ws, pl, s); break;
    case 7: e = enc_launch<7>(w, trellis, cost, k, n, ws, pl, s); break;
    default: e = enc_launch<8>(w, trellis, cost, k, n, ws, pl, s); break;
    }
    return e == cudaSuccess ? EXL3_OK : EXL3_ERR_CUDA;
}
