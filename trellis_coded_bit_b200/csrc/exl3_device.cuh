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

// Programmatic dependent launch: wait for the preceding grid in the stream
// to complete (no-op when the launch did not allow overlap) / let the next
// grid start launching.
__device__ __forceinline__ void grid_dep_wait()
{
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

__device__ __forceinline__ void grid_dep_launch()
{
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ------------------------------------------------------------ tile rows ---
//
// A tile row holds 16 weights = 16K bits = exactly K words, so row r starts at
// word rK.  Its states need the row's K words plus the word before (the
// prefix; for row 0 the tile's last word -- the tail-biting wrap).  The
// 32-bit loads covering those K + 1 words start on a half-word position P:
// P = 1 when the prefix word is the upper half of the first load, P = 0 when
// it is the lower half.  P depends only on K and the row's parity, so callers
// that process rows of one parity at a time get compile-time layouts.

template <int K, int PAR>
struct RowSpan {
    static constexpr int P = (PAR == 0) ? 1 : ((K & 1) ? 0 : 1);
    static constexpr int N32 = (P + K + 2) / 2;  // 32-bit loads covering K + 1 words
};

// Loads the words of tile row `row` (of parity PAR) from a tile of 8K 32-bit
// words.  raw[0] holds the prefix word; the loads are read-only (nc) and as
// wide as the row's alignment allows.
template <int K, int PAR, int N>
__device__ __forceinline__ void load_row(const uint32_t *__restrict__ tile, int row, uint32_t (&raw)[N])
{
    constexpr int P = RowSpan<K, PAR>::P;
    constexpr int N32 = RowSpan<K, PAR>::N32;
    static_assert(N >= N32, "raw buffer too small");
    const int first = (row * K - 1) >> 1;  // floor; -1 for row 0
    raw[0] = __ldg(tile + (first < 0 ? 8 * K - 1 : first));
    if constexpr (K == 4 && P == 1) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(tile + first + 1));
        raw[1] = v.x;
        raw[2] = v.y;
    } else if constexpr (K == 8 && P == 1) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(tile + first + 1));
        raw[1] = v.x;
        raw[2] = v.y;
        raw[3] = v.z;
        raw[4] = v.w;
    } else {
#pragma unroll
        for (int i = 1; i < N32; ++i)
            raw[i] = __ldg(tile + first + i);
    }
}

// The 16 states of a tile row from its loaded words.  Word W[-1] (prefix) is
// at half-word position P, W[i] at P + 1 + i.  Weight j's window ends at row
// bit e = (j + 1) K: it lies in V = W[a-1]:W[a] (a = e / 16) shifted right by
// c = 16 - e % 16; c = 16 is the word W[a-1] itself.  Every window is one
// byte permute (with zero fill), from V or from V pre-shifted by c % 8 bits;
// all selectors are compile-time constants.
template <int K, int P, int N>
__device__ __forceinline__ void row_states(const uint32_t (&raw)[N], uint32_t (&s)[16])
{
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int e = (j + 1) * K;
        const int a = e >> 4;
        const int c = 16 - (e & 15);
        const int pos = P + a;  // half-word position of W[a-1]
        if (c == 16) {
            s[j] = __byte_perm(raw[pos >> 1], 0u, (pos & 1) ? 0x4432u : 0x4410u);
        } else {
            const uint32_t v = (pos & 1) ? __byte_perm(raw[pos >> 1], raw[(pos >> 1) + 1], 0x3254u)
                                         : __byte_perm(raw[pos >> 1], 0u, 0x1032u);
            const int r = c & 7, cb = c >> 3;
            const uint32_t sel = 0x4400u | ((uint32_t)(cb + 1) << 4) | (uint32_t)cb;
            s[j] = __byte_perm(r ? (v >> r) : v, 0u, sel);
        }
    }
}

// Same as load_row for a tile held in shared memory (plain loads).
template <int K, int PAR, int N>
__device__ __forceinline__ void load_row_plain(const uint32_t *tile, int row, uint32_t (&raw)[N])
{
    constexpr int N32 = RowSpan<K, PAR>::N32;
    static_assert(N >= N32, "raw buffer too small");
    const int first = (row * K - 1) >> 1;
    raw[0] = tile[first < 0 ? 8 * K - 1 : first];
#pragma unroll
    for (int i = 1; i < N32; ++i)
        raw[i] = tile[first + i];
}

// ------------------------------------------------------------- codebook ---

// The procedural codebook's constants.  Kernels receive them as launch
// parameters and keep them in registers: a SASS instruction encodes at most
// one 32-bit immediate, so with literal constants the mask/xor would split
// into two logic ops; from registers it is one IMAD plus one LOP3 per weight,
// the "one integer multiply + one lop3" of the EXL3 GEMM kernel article
// (sections 先看结论 and GEMM内核).
constexpr uint32_t kCbMul = 89226354u;
constexpr uint32_t kCbAdd = 64248484u;
constexpr uint32_t kCbMask = 0x8fff8fffu;
constexpr uint32_t kCbXor = 0x3b603b60u;

struct Codebook {
    uint32_t mul, add, mask, xr;
};

__host__ __device__ inline Codebook codebook_constants()
{
    return Codebook{kCbMul, kCbAdd, kCbMask, kCbXor};
}

// The codebook's 32-bit word for a state; its two 16-bit halves are fp16 bit
// patterns whose sum is the weight.
__device__ __forceinline__ uint32_t codebook_word(uint32_t state, const Codebook &cb)
{
    const uint32_t v = state * cb.mul + cb.add;
    return (v & cb.mask) ^ cb.xr;
}


// The exact fp16 weights of one tile row (row_states + codebook, the halves
// added in fp16 with round-to-nearest-even), packed as 8 half2: out[j] holds
// the weights of columns 2j and 2j+1.
template <int K, int P, int N>
__device__ __forceinline__ void row_weights_f16(const uint32_t (&raw)[N], const Codebook &cb,
                                                uint32_t (&out)[8])
{
    uint32_t s[16];
    row_states<K, P>(raw, s);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t v0 = codebook_word(s[2 * j], cb);
        const uint32_t v1 = codebook_word(s[2 * j + 1], cb);
        const __half2 h0 = *reinterpret_cast<const __half2 *>(&v0);
        const __half2 h1 = *reinterpret_cast<const __half2 *>(&v1);
        // lo + hi of each word in both lanes (one add with half selects), then
        // one byte permute packs the two weights
        __half2 w0 = __hadd2(__low2half2(h0), __high2half2(h0));
        __half2 w1 = __hadd2(__low2half2(h1), __high2half2(h1));
        out[j] = __byte_perm(*reinterpret_cast<uint32_t *>(&w0), *reinterpret_cast<uint32_t *>(&w1), 0x5410u);
    }
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

// Bounded wait for a role that is not on the critical path at that moment (a
// producer running ahead, an epilogue waiting out a whole k loop): it sleeps
// between polls so that its waiting takes no issue slots from the warps doing
// the work.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity, uint64_t limit_ns,
                                                unsigned sleep_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        __nanosleep(sleep_ns);
        if (global_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}

// Warp-uniform bounded wait for warps that wait often and briefly: every
// lane polls (one try_wait per poll for the whole warp) and a vote keeps the
// outcome uniform; the timer is read only every 16 polls.
__device__ __forceinline__ bool warp_wait_uniform(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity)))
        return true;
    const uint64_t t0 = global_ns();
    for (;;) {
#pragma unroll 1
        for (int j = 0; j < 16; ++j)
            if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity)))
                return true;
        if (global_ns() - t0 > limit_ns)
            return false;
    }
}

// Warp-uniform bounded wait: lane 0 decides (so a timeout cannot split the
// warp), then the other lanes observe the completed phase themselves, which
// cannot move on before this warp releases the stage.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns,
                                          unsigned sleep_ns = 0)
{
    const int lane = threadIdx.x & 31;
    bool ok = true;
    if (lane == 0)
        ok = sleep_ns ? mbar_wait_sleep(bar, parity, limit_ns, sleep_ns) : mbar_wait(bar, parity, limit_ns);
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
