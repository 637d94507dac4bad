// exl3_device.cuh -- device building blocks shared by the library's kernels:
// trellis bit reading, the procedural codebook, the 128-point Hadamard on a
// warp, tensor-core MMA wrappers, mbarriers and bulk async copies.
//
// Format (this library's convention; the pages fix the mechanisms but not the
// bit order): a 16x16 tile's 16K uint16 words form one big-endian bit string;
// weight i = 16 r + c owns bits [iK, iK + K) and its state is the 16-bit
// window ending there, cyclic over the tile (tail-biting: weight 0 continues
// from the stream's end).  "EXL3 GEMM kernel article" below is the page
// "ExLlamaV3推理快的秘密: EXL3 GEMM内核与融合Viterbi编码CUDA实现剖析".
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace exl3 {

// ---------------------------------------------------------------- status ---

// Layout of the status word every gemv/gemm workspace starts with.
enum : uint32_t { kStatusOk = 0u, kStatusTimeout = 5u };

// Bounded waits are limited in wall time, read from the global nanosecond
// timer: a legitimate wait lasts microseconds, the default limit is 1 s.
constexpr uint64_t kDefaultWaitNs = 1000000000ull;

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------ bit stream ---

// Words are stored little-endian, the bit string is big-endian per word: the
// stream order of the bytes of an aligned 32-bit load b0 b1 b2 b3 is
// b1 b0 b3 b2.  Returns the 32 stream bits with the earliest bit at bit 31.
__device__ __forceinline__ uint32_t be32(uint32_t raw)
{
    return __byte_perm(raw, 0u, 0x1032);
}

// 64 stream bits starting at bit position `pos` (earliest bit = bit 63) of a
// tile held as 8K 32-bit words at `tile`.  pos may be in [-32, 256K); the read
// wraps cyclically (tail-biting).
template <int K>
__device__ __forceinline__ uint64_t read_bits64(const uint32_t *tile, int pos)
{
    constexpr int kWords32 = 8 * K;  // 32-bit words per tile
    constexpr int kBits = 256 * K;
    if (pos < 0)
        pos += kBits;
    int q0 = pos >> 5;
    const int o = pos & 31;
    int q1 = q0 + 1;
    if (q1 >= kWords32)
        q1 -= kWords32;
    int q2 = q1 + 1;
    if (q2 >= kWords32)
        q2 -= kWords32;
    const uint32_t a = be32(tile[q0]);
    const uint32_t b = be32(tile[q1]);
    const uint32_t c = be32(tile[q2]);
    const uint32_t hi = __funnelshift_l(b, a, o);
    const uint32_t lo = __funnelshift_l(c, b, o);
    return ((uint64_t)hi << 32) | lo;
}

// States of N consecutive weights of one tile row, the first of which starts
// its own K bits at stream bit `start` (a multiple of 8: every run of 8
// weights starts on a byte).  N * K + 16 - K must fit the 64 bits read.
template <int K, int N>
__device__ __forceinline__ void run_states(const uint32_t *tile, int start, uint32_t (&s)[N])
{
    static_assert((N - 1) * K + 16 <= 64, "run does not fit one 64-bit read");
    const uint64_t r = read_bits64<K>(tile, start - (16 - K));
#pragma unroll
    for (int j = 0; j < N; ++j)
        s[j] = (uint32_t)(r >> (48 - j * K)) & 0xffffu;
}

// ------------------------------------------------------------- codebook ---

// The procedural codebook's 32-bit word for a state: one multiply-add and one
// mask/xor (EXL3 GEMM kernel article, sections 先看结论 and GEMM内核: "one
// integer multiply + one lop3, no table lookup").  Its two 16-bit halves are
// fp16 bit patterns whose sum is the weight.
__device__ __forceinline__ uint32_t codebook_word(uint32_t state)
{
    uint32_t v = state * 89226354u + 64248484u;
    return (v & 0x8fff8fffu) ^ 0x3b603b60u;
}

// The weight itself: the two halves added in fp16, round-to-nearest-even.
__device__ __forceinline__ __half codebook_weight(uint32_t state)
{
    const uint32_t v = codebook_word(state);
    const __half2 h = *reinterpret_cast<const __half2 *>(&v);
    return __hadd(__low2half(h), __high2half(h));
}

// ------------------------------------------------------------ hadamard ----

// In-warp 128-point Sylvester Hadamard: lane l holds elements 4l .. 4l+3 of
// the block.  H[i][j] = (-1)^popcount(i & j); unnormalised.
__device__ __forceinline__ void warp_fwht128(float (&v)[4])
{
    float a = v[0] + v[1], b = v[0] - v[1], c = v[2] + v[3], d = v[2] - v[3];
    v[0] = a + c;
    v[1] = b + d;
    v[2] = a - c;
    v[3] = b - d;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (threadIdx.x & m) != 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float o = __shfl_xor_sync(0xffffffffu, v[e], m);
            v[e] = upper ? (o - v[e]) : (v[e] + o);
        }
    }
}

// ------------------------------------------------------------------ MMA ---

// D += A (16x16 fp16, row) * B (16x8 fp16, col), fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// -------------------------------------------------------------- mbarrier ---

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(
                     smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns
// false (and the caller must bail out) once `limit_ns` has passed.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > limit_ns)
            return false;
    return true;
}

// Warp-uniform bounded wait: lane 0 decides (so a timeout cannot split the
// warp), then the other lanes observe the completed phase themselves, which
// cannot move on before this warp releases the stage.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    const int lane = threadIdx.x & 31;
    bool ok = true;
    if (lane == 0)
        ok = mbar_wait(bar, parity, limit_ns);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (ok && lane != 0)
        mbar_wait(bar, parity, kDefaultWaitNs);
    return ok;
}

// 1-D bulk async copy global -> shared, completing on an mbarrier (no
// multicast).  Addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                         uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void record_timeout(uint32_t *status)
{
    if (status)
        atomicExch(status, kStatusTimeout);
}

}  // namespace exl3
