// gemm.cu -- exl3_gemm: y = svh .* H(H(x .* suh) . W_hat) on the fifth-
// generation tensor cores (tcgen05.mma, accumulators in TMEM), with W_hat
// decoded from the trellis into shared memory on the fly (EXL3 GEMM kernel
// article, section GEMM内核: the input is Hadamard-rotated, then the kernel
// reads the quantised weights, decodes them with the procedural codebook and
// multiplies, in one pass; the kernel map picks tile shapes).
//
// B200 design (the pages' consumer-GPU kernel is prior art, not a blueprint):
//   1. A rotation pass computes x' = H(x .* suh)/sqrt(128) in fp32 and writes
//      it as fp16 directly in the tensor core's canonical K-major, 128-byte
//      swizzled tile layout ([m/128][k/64] tiles of 128 rows x 64 channels,
//      16 KB each), so one 1-D bulk copy moves one A tile into shared memory.
//      A launch may serve up to 8 layers with the same m, k and K
//      (exl3_gemm_multi: q/k/v, gate/up): each has its own x' region, and the
//      GEMM's output tile columns are all the layers' columns in order (a
//      small table gives each layer's x', trellis, svh, y, n and first tile
//      column), so the stream-K split below balances them together.
//   2. The main kernel is persistent and "stream-K" balanced: the work units
//      are (256 x 256 output tile, 64-channel k block) pairs in tile order,
//      and CTA c of G (G <= one per SM) owns units [cU/G, (c+1)U/G), so every
//      CTA gets the same work whatever the tile count (no last partial
//      wave).  A CTA's range splits at tile boundaries into segments.  A
//      segment that covers a whole tile is finished directly; one that covers
//      part of a tile writes its fp32 accumulators to the workspace, and the
//      last segment to arrive on the tile's counter (atomic ticket, no
//      spinning) sums every segment's partials in segment order
//      (deterministic) and finishes the tile.  23 warps:
//        warp 0   A producer: bulk-copies the two A tiles of each unit into a
//                 3-stage ring (no multicast; it sleeps between polls);
//        warp 2   trellis producer: bulk-copies each unit's 4 trellis tile
//                 rows (16 tiles each) into a ring as deep as the shared
//                 memory left allows (12 stages at K = 1 .. 2 at K = 8),
//                 so the decoders never wait for HBM (sleeps between polls);
//        warp 1   allocates 512 TMEM columns (two 128 x 256 fp32
//                 accumulators); one lane issues
//                 tcgen05.mma.cta_group::1.kind::f16 (M=128, N=256, K=16,
//                 A K-major, B MN-major) and commits to mbarriers that free
//                 the A and B stages and, at a segment end, hand the
//                 accumulators to the epilogue;
//        warps 3..18 decode: lane u of a warp decodes two rows of one trellis
//                 tile, sums the codebook halves in fp16 (RNE, the exact
//                 W_hat) and stores them into the MN-major 128-byte-swizzled
//                 B stage (3-stage ring); fence.proxy.async, mbarrier arrive;
//        warps 19..22 epilogue (one TMEM lane quarter each): tcgen05.ld of the
//                 accumulators, the 128-point output rotation as
//                 H4 (x) H32 (32-point butterflies in registers, a TMEM round
//                 trip, then the 4-point stage), svh/sqrt(128), fp16 y; or the
//                 partial-sum write and the ticket.
//   For m <= 64 the same kernel runs with the operands swapped (template
//   flag WA): the decoded stage is the A operand (M = 128 output channels per
//   MMA, two per 16-channel step), x' rows 0 .. N-1 the B operand (N = m
//   rounded up to 32), and the epilogue transposes the accumulators (channels
//   in TMEM lanes, batches in columns) through shared memory for the output
//   rotation.
//   Shared memory is addressed from the dynamic shared array (the 1024-byte
//   alignment the swizzled tiles need is an offset, not an integer cast), so
//   the decoders' loads and stores stay shared-space instructions.
//   All waits are bounded; a timeout is recorded in the workspace status word
//   and every role drains its in-flight copies / MMAs before the CTA exits.
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

constexpr int kBM = 128;             // rows per MMA tile (TMEM lanes)
constexpr int kMT = 2;               // M tiles per CTA sharing one decoded B
constexpr int kBN = 256;             // output channels per tile (MMA N)
constexpr int kBK = 64;              // input channels per unit
constexpr int kDecWarps = 16;
// 23 warps: the decoders carry no epilogue state, and the epilogue warps do
// not hold up decoding while they drain the accumulators
constexpr int kWarpProducerA = 0, kWarpMma = 1, kWarpProducerT = 2, kWarpDec0 = 3;
constexpr int kWarpEpi0 = kWarpDec0 + kDecWarps;                   // 19..22
constexpr int kGemmThreads = 32 * (kWarpEpi0 + 4);                 // 736
constexpr int kATileBytes = kBM * kBK * 2;                  // 16 KB
constexpr int kAStageBytes = kMT * kATileBytes;             // 32 KB
constexpr int kBStageBytes = kBK * kBN * 2;                 // 32 KB
constexpr int kAStages = 3;
constexpr int kBStages = 3;
constexpr int kMaxTStages = 12;
constexpr int kTmemCols = kMT * kBN;                        // 512
constexpr int kPartialFloats = kMT * kBM * kBN;             // one split segment: 256 KB

__host__ __device__ constexpr int gemm_trellis_stage_bytes(int K)
{
    return (kBK / 16) * (kBN / 16) * 32 * K;  // 4 tile rows x 16 tiles
}

// Small m (m <= kWaMaxM, one M tile): the decoded weight stage is the A
// operand instead (M = 128 output channels, MN-major, the same bytes the
// decoders write for B) and x' the B operand (N = m rounded up to 32,
// K-major: the first N rows of the x' tile).  Each unit is then two
// M = 128 x N x 16 MMAs per 16 channels instead of one M = 128 x 256 x 16 of
// which only m rows are wanted.  The accumulators hold output channels in
// TMEM lanes and batches in columns, so the epilogue transposes them through
// a 16 KB shared buffer (32 batches x 128 channels) for the output rotation.
constexpr int kWaMaxM = 64;
constexpr int kWaEpiBytes = 32 * 128 * 4;

__host__ __device__ constexpr int gemm_a_stage_bytes(bool wa)
{
    return wa ? kWaMaxM * 128 : kAStageBytes;
}

// Trellis ring depth: whatever shared memory the A and B rings (and the
// small-m epilogue buffer) leave (up to 227 KB per CTA), at most kMaxTStages
// stages.
constexpr int kSmemLimit = 232448;

__host__ __device__ constexpr int gemm_fixed_bytes(bool wa)
{
    return 1024 /* alignment slack */ + 1024 /* barriers */ + kAStages * gemm_a_stage_bytes(wa) +
           kBStages * kBStageBytes + (wa ? kWaEpiBytes : 0);
}

__host__ __device__ constexpr int gemm_t_stages(int K, bool wa)
{
    return (kSmemLimit - gemm_fixed_bytes(wa)) / gemm_trellis_stage_bytes(K) > kMaxTStages
               ? kMaxTStages
               : (kSmemLimit - gemm_fixed_bytes(wa)) / gemm_trellis_stage_bytes(K);
}

__host__ __device__ constexpr int gemm_smem_bytes(int K, bool wa)
{
    return gemm_fixed_bytes(wa) + gemm_t_stages(K, wa) * gemm_trellis_stage_bytes(K);
}

static_assert(gemm_t_stages(8, false) >= 2 && gemm_smem_bytes(8, false) <= kSmemLimit &&
                  gemm_smem_bytes(1, false) <= kSmemLimit && gemm_smem_bytes(8, true) <= kSmemLimit &&
                  gemm_smem_bytes(1, true) <= kSmemLimit,
              "shared memory per CTA");
static_assert(kWaMaxM % 32 == 0 && kWaMaxM <= kBM && 2 * kWaMaxM * 128 <= kPartialFloats &&
                  (gemm_a_stage_bytes(true) & 1023) == 0,
              "small-m tiles");

// ----------------------------------------------------- tcgen05 wrappers ---

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

#define EXL3_TMEM_ST32(taddr, v)                                                                          \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13," \
                 "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(   \
                     taddr),                                                                               \
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),   \
                 "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),          \
                 "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),        \
                 "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),        \
                 "r"(v[29]), "r"(v[30]), "r"(v[31])                                                        \
                 : "memory")

// A TMEM load and its wait in one statement: PTX leaves the destination
// registers of tcgen05.ld undefined until tcgen05.wait::ld, so the compiler
// must not be able to touch them (a spill, say) in between.
#define EXL3_TMEM_LD32(taddr, v)                                                                          \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
                 "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"          \
                 "tcgen05.wait::ld.sync.aligned;\n"                                                       \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), \
                   "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), \
                   "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), \
                   "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), \
                   "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), \
                   "=r"(v[31]) \
                 : "r"(taddr)                                                                              \
                 : "memory")

// Four 8-column loads at taddr, taddr + 32, + 64, + 96 into v[0..31], then the wait.
#define EXL3_TMEM_LD8X4(taddr, v)                                                                         \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%32];\n"               \
                 "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%8,%9,%10,%11,%12,%13,%14,%15}, [%33];\n"         \
                 "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%16,%17,%18,%19,%20,%21,%22,%23}, [%34];\n"       \
                 "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%24,%25,%26,%27,%28,%29,%30,%31}, [%35];\n"       \
                 "tcgen05.wait::ld.sync.aligned;\n"                                                       \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), \
                   "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), \
                   "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), \
                   "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), \
                   "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), \
                   "=r"(v[31]) \
                 : "r"(taddr), "r"((taddr) + 32u), "r"((taddr) + 64u), "r"((taddr) + 96u)                  \
                 : "memory")

// Four 8-column stores of v[0..31] at taddr, taddr + 32, + 64, + 96 (no wait).
#define EXL3_TMEM_ST8X4(taddr, v)                                                                         \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%4,%5,%6,%7,%8,%9,%10,%11};\n"              \
                 "tcgen05.st.sync.aligned.32x32b.x8.b32 [%1], {%12,%13,%14,%15,%16,%17,%18,%19};\n"        \
                 "tcgen05.st.sync.aligned.32x32b.x8.b32 [%2], {%20,%21,%22,%23,%24,%25,%26,%27};\n"        \
                 "tcgen05.st.sync.aligned.32x32b.x8.b32 [%3], {%28,%29,%30,%31,%32,%33,%34,%35};\n"        \
                 ::"r"(taddr), "r"((taddr) + 32u), "r"((taddr) + 64u), "r"((taddr) + 96u),                \
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),   \
                 "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),          \
                 "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),        \
                 "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),        \
                 "r"(v[29]), "r"(v[30]), "r"(v[31])                                                        \
                 : "memory")

__device__ __forceinline__ void tmem_wait_st()
{
    asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// Shared-memory matrix descriptor: 128-byte swizzle, sm_100 format.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)((lbo >> 4) & 0x3fffu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: D f32, A f16 K-major, B f16 MN-major.
__host__ __device__ constexpr uint32_t gemm_idesc()
{
    return (1u << 4) | (0u << 7) | (0u << 10) | (0u << 15) | (1u << 16) | ((uint32_t)(kBN >> 3) << 17) |
           ((uint32_t)(kBM >> 4) << 24);
}

// Small-m form: D f32, A (weights) f16 MN-major, B (x') f16 K-major, M = 128,
// N = nb.
__host__ __device__ constexpr uint32_t gemm_idesc_wa(int nb)
{
    return (1u << 4) | (0u << 7) | (0u << 10) | (1u << 15) | (0u << 16) | ((uint32_t)(nb >> 3) << 17) |
           ((uint32_t)(kBM >> 4) << 24);
}

// 32-point Sylvester Hadamard on 32 fp32 values held by one thread.
__device__ __forceinline__ void fwht32(float (&v)[32])
{
#pragma unroll
    for (int h = 1; h < 32; h <<= 1)
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

// -------------------------------------------------------- rotation pass ---

constexpr int kGemmMaxLayers = 8;  // layers per launch

// The layers of one rotation launch (same m and k): x, suh and the tiled x'.
struct GemmRotParams {
    const __half *x[kGemmMaxLayers];
    const __half *suh[kGemmMaxLayers];
    unsigned char *xt[kGemmMaxLayers];
    int nlayers, m, k;
};

// x'[r, :] = H(x[r, :] .* suh)/sqrt(128) of each layer written in the tiled,
// swizzled A layout: tile (r/128, c/64), 128-byte row r%128, 16-byte chunk
// ((c%64)/8) ^ (r%8).  A warp per (layer, row, 128-channel block).
__global__ void __launch_bounds__(256) rotate_tiled_kernel(const GemmRotParams rp)
{
    const int lane = threadIdx.x & 31;
    grid_dep_wait();    // x is produced by the preceding kernel
    grid_dep_launch();  // the GEMM kernel may set up (barriers, TMEM) meanwhile
    const int m = rp.m, k = rp.k;
    const int64_t per_layer = (int64_t)m * (k / 128);
    const int64_t blocks = per_layer * rp.nlayers;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t wj = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); wj < blocks; wj += warps) {
        const int l = (int)(wj / per_layer);
        const int64_t w = wj - (int64_t)l * per_layer;
        const __half *__restrict__ x = rp.x[l];
        const __half *__restrict__ suh = rp.suh[l];
        unsigned char *__restrict__ xt = rp.xt[l];
        const int r = (int)(w / (k / 128));
        const int blk = (int)(w - (int64_t)r * (k / 128));
        const int c = blk * 128 + lane * 4;
        const uint2 raw = *reinterpret_cast<const uint2 *>(x + (int64_t)r * k + c);
        const uint2 sr = *reinterpret_cast<const uint2 *>(suh + c);
        const __half2 *xv = reinterpret_cast<const __half2 *>(&raw);
        const __half2 *sv = reinterpret_cast<const __half2 *>(&sr);
        float v[4] = {__low2float(xv[0]) * __low2float(sv[0]), __high2float(xv[0]) * __high2float(sv[0]),
                      __low2float(xv[1]) * __low2float(sv[1]), __high2float(xv[1]) * __high2float(sv[1])};
        warp_fwht128(v);
        const float s = 0.08838834764831845f;
        __half2 o0 = __floats2half2_rn(v[0] * s, v[1] * s);
        __half2 o1 = __floats2half2_rn(v[2] * s, v[3] * s);
        const int kb = c >> 6, chunk = (c & 63) >> 3, within = c & 7;
        const int64_t tile = (int64_t)(r >> 7) * (k >> 6) + kb;
        const int row = r & 127;
        unsigned char *dst = xt + tile * kATileBytes + row * 128 + ((chunk ^ (row & 7)) << 4) + within * 2;
        uint2 out;
        out.x = *reinterpret_cast<uint32_t *>(&o0);
        out.y = *reinterpret_cast<uint32_t *>(&o1);
        *reinterpret_cast<uint2 *>(dst) = out;
    }
}

// Decodes tile row `row` of a shared-memory tile (stage tile row trow, column
// tcol) to exact fp16 weights and stores its 16 values as two 16-byte chunks of
// the MN-major, 128-byte-swizzled B stage: input channel kr is a row of an
// 8-row x 64-column atom (atoms of 8 k rows at 1024 B, 64-column groups at
// 8192 B), chunk (n % 64) / 8 lands at chunk position ((n % 64) / 8) ^ (kr % 8).
template <int K, int PAR>
__device__ __forceinline__ void decode_row_to_b(const uint32_t *tile, int row, const Codebook &cb,
                                                unsigned char *bt, int trow, int tcol)
{
    uint32_t raw[RowSpan<K, PAR>::N32];
    load_row_plain<K, PAR>(tile, row, raw);
    uint32_t w[8];
    row_weights_f16<K, RowSpan<K, PAR>::P>(raw, cb, w);
    const int kr = trow * 16 + row;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int n0 = tcol * 16 + h * 8;
        unsigned char *dst = bt + ((n0 >> 6) * (kBK / 8) + (kr >> 3)) * 1024 + (kr & 7) * 128 +
                             ((((n0 & 63) >> 3) ^ (kr & 7)) << 4);
        *reinterpret_cast<uint4 *>(dst) = make_uint4(w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]);
    }
}

// ------------------------------------------------------------ main kernel ---

// One layer of a launch: its output columns are the launch's tile columns
// [tn_begin, tn_begin + ceil(n / 256)); every layer has the launch's m, k, K.
struct GemmLayer {
    const unsigned char *xt;   // the layer's tiled x'
    const uint16_t *trellis;
    const __half *svh;
    __half *y;
    int n, tn_begin;
};

struct GemmParams {
    GemmLayer L[kGemmMaxLayers];
    int nlayers;
    float *partials;           // [2 G][kPartialFloats] split-segment accumulators
    uint32_t *counters;        // [tiles] arrival tickets (return to zero)
    uint32_t *status;
    int m, k;
    int tiles_n;               // tile columns of all layers
    int kb_count;              // k / 64 units per tile
    uint32_t units;            // tiles * kb_count (units * ctas < 2^32)
    int ctas;                  // grid size G
    int nb;                    // small-m form: MMA N (m rounded up to 32); 0 otherwise
    uint64_t wait_ns;
    Codebook cb;
};

struct GemmBars {
    uint64_t afull[kAStages], aempty[kAStages];
    uint64_t bfull[kBStages], bempty[kBStages];
    uint64_t tfull[kMaxTStages], tempty[kMaxTStages];
    uint64_t acc_full, acc_empty, drain;
    uint32_t tmem_slot;
    int abort;
    int ticket;
};
static_assert(sizeof(GemmBars) <= 1024, "barrier block");

// The layer that owns tile column tn.
__device__ __forceinline__ int gemm_layer_of(const GemmParams &p, int tn)
{
    int l = 0;
    while (l + 1 < p.nlayers && tn >= p.L[l + 1].tn_begin)
        ++l;
    return l;
}

// CTA owning unit u: the largest c with floor(c U / G) <= u.  (32-bit: the
// host guarantees U * G < 2^32.)
__device__ __forceinline__ int gemm_owner(uint32_t u, uint32_t U, uint32_t G)
{
    return (int)(((u + 1) * G - 1) / U);
}

// Partial-sum slot of CTA c's segment in the tile starting at unit tb: its
// first segment (the one holding its first unit) uses slot 2c, its last 2c+1.
__device__ __forceinline__ int gemm_slot(uint32_t c, uint32_t tb, uint32_t U, uint32_t G)
{
    return (int)((c * U / G >= tb) ? 2 * c : 2 * c + 1);
}

// Named barrier over the four epilogue warps.
__device__ __forceinline__ void epi_sync()
{
    asm volatile("bar.sync 1, 128;\n" ::: "memory");
}

// Epilogue of one segment [u, se) (units of one tile), run by the four
// epilogue warps (one TMEM lane quarter each): waits for the accumulators, then either finishes the tile (output
// rotation, svh, fp16 y) or writes the segment's partial sums and takes a
// ticket -- the last segment of the tile to arrive sums all partials and
// finishes it.  Releases the accumulators to the MMA issuer at the end.
// Returns false if the wait ran out (the caller stops).
__device__ __forceinline__ bool gemm_epilogue(const GemmParams &p, GemmBars &bars, uint32_t tmem, int seg,
                                              uint32_t u, uint32_t se, uint32_t U, uint32_t G, uint32_t KB)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int erow = quarter * 32 + lane;  // row within an M tile
    float4 *const parts = reinterpret_cast<float4 *>(p.partials);
    volatile int *abort_flag = &bars.abort;
    const uint32_t t = u / KB;
    const uint32_t tb = t * KB, te = tb + KB;
    const bool whole = u == tb && se == te;
    const int tm = (int)(t / p.tiles_n), tn = (int)(t - (t / p.tiles_n) * p.tiles_n);
    const int mt_count = (p.m - tm * kBM * kMT) > kBM ? kMT : 1;
    // a whole k loop can pass before the accumulators are ready: sleep between polls
    if (!warp_wait(&bars.acc_full, (uint32_t)seg & 1u, p.wait_ns, 1000)) {
        if (lane == 0) {
            record_timeout(p.status);
            *abort_flag = 1;
        }
        return false;
    }
    tc_fence_after();
    if (*abort_flag)
        return false;
    int nseg = 1, c_lo = 0;
    bool finish = true;
    if (!whole) {
        // this segment's fp32 accumulators -> its slot, 16-byte chunk
        // (mt, 4-column group g, row): consecutive lanes, consecutive chunks
        c_lo = gemm_owner(tb, U, G);
        nseg = gemm_owner(te - 1, U, G) - c_lo + 1;
        float4 *slot = parts + (size_t)gemm_slot(blockIdx.x, tb, U, G) * (kPartialFloats / 4);
        for (int mt = 0; mt < mt_count; ++mt) {
#pragma unroll 1
            for (int cc = 0; cc < kBN / 32; ++cc) {
                uint32_t r[32];
                EXL3_TMEM_LD32(tmem + lane_base + (uint32_t)(mt * kBN + 32 * cc), r);
#pragma unroll
                for (int g = 0; g < 8; ++g)
                    __stcg(slot + ((mt * 64 + cc * 8 + g) * kBM + erow),
                           make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                       __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3])));
            }
        }
        __threadfence();
        epi_sync();
        if (warp == kWarpEpi0 && lane == 0) {
            const uint32_t prev = atomicAdd(&p.counters[t], 1u);
            const int last = prev == (uint32_t)(nseg - 1) ? 1 : 0;
            if (last) {
                __threadfence();
                p.counters[t] = 0u;  // every segment has arrived: re-arm for the next call
            }
            bars.ticket = last;
        }
        epi_sync();
        finish = bars.ticket != 0;
    }
    if (finish && !whole) {
        // every segment's partials, summed in segment order, accumulated in
        // TMEM (s = p0; s += p1; ...): 32 columns (8 loads in flight) a step
        for (int mt = 0; mt < mt_count; ++mt) {
#pragma unroll 1
            for (int j = 0; j < nseg; ++j) {
                const float4 *src = parts + (size_t)gemm_slot((uint32_t)(c_lo + j), tb, U, G) * (kPartialFloats / 4) +
                                    (mt * 64 * kBM + erow);
#pragma unroll 1
                for (int cc = 0; cc < kBN / 32; ++cc) {
                    float4 q[8];
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        q[g] = __ldcg(src + (cc * 8 + g) * kBM);
                    const uint32_t ta = tmem + lane_base + (uint32_t)(mt * kBN + 32 * cc);
                    uint32_t r[32];
                    if (j == 0) {
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            r[4 * g] = __float_as_uint(q[g].x);
                            r[4 * g + 1] = __float_as_uint(q[g].y);
                            r[4 * g + 2] = __float_as_uint(q[g].z);
                            r[4 * g + 3] = __float_as_uint(q[g].w);
                        }
                    } else {
                        EXL3_TMEM_LD32(ta, r);
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            r[4 * g] = __float_as_uint(__uint_as_float(r[4 * g]) + q[g].x);
                            r[4 * g + 1] = __float_as_uint(__uint_as_float(r[4 * g + 1]) + q[g].y);
                            r[4 * g + 2] = __float_as_uint(__uint_as_float(r[4 * g + 2]) + q[g].z);
                            r[4 * g + 3] = __float_as_uint(__uint_as_float(r[4 * g + 3]) + q[g].w);
                        }
                    }
                    EXL3_TMEM_ST32(ta, r);
                }
                tmem_wait_st();
            }
        }
    }
    if (finish) {
        // H128 = H4 (x) H32 on each 128-column half: first the 4-point stage
        // across the four 32-column chunks (eight columns of each per TMEM
        // round trip), then per chunk the 32-point butterflies in registers,
        // svh/sqrt(128) and fp16.  A chunk is 64 contiguous bytes of the row
        // the lane holds; a 4 x 4 exchange of 16-byte pieces within each group
        // of four lanes then lets the group store 64 contiguous bytes of one
        // row per instruction (8 rows per warp store instead of 32).
        // The last tile of n = 256j + 128 carries 128 columns: its other half
        // holds results of stale weights and is not stored.
        const GemmLayer &L = p.L[gemm_layer_of(p, tn)];
        const int tnl = tn - L.tn_begin;         // tile column within the layer
        const int halves = (tnl + 1) * kBN > L.n ? 1 : kBN / 128;
        const int gi = lane & 3;                 // piece this lane stores
        const int grow = erow - gi;              // first row of the lane's group
        for (int mt = 0; mt < mt_count; ++mt) {
            const int row0 = tm * kBM * kMT + mt * kBM + grow;
            for (int hb = 0; hb < halves; ++hb) {
                const uint32_t col0 = (uint32_t)(mt * kBN + hb * 128);
#pragma unroll 1
                for (int o = 0; o < 4; ++o) {
                    uint32_t w[32];  // [chunk c][8 columns]
                    const uint32_t ta = tmem + lane_base + col0 + 8 * o;
                    EXL3_TMEM_LD8X4(ta, w);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float a0 = __uint_as_float(w[e]), a1 = __uint_as_float(w[8 + e]);
                        const float a2 = __uint_as_float(w[16 + e]), a3 = __uint_as_float(w[24 + e]);
                        const float s01 = a0 + a1, d01 = a0 - a1, s23 = a2 + a3, d23 = a2 - a3;
                        w[e] = __float_as_uint(s01 + s23);
                        w[8 + e] = __float_as_uint(d01 + d23);
                        w[16 + e] = __float_as_uint(s01 - s23);
                        w[24 + e] = __float_as_uint(d01 - d23);
                    }
                    EXL3_TMEM_ST8X4(ta, w);
                }
                tmem_wait_st();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    EXL3_TMEM_LD32(tmem + lane_base + col0 + 32 * c, r);
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        v[i] = __uint_as_float(r[i]);
                    fwht32(v);
                    const int ncol0 = tnl * kBN + hb * 128 + 32 * c;
                    // piece q (columns 8q .. 8q + 7 of the chunk) as 4 words
                    uint32_t pc[4][4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 sv4 = *reinterpret_cast<const uint4 *>(L.svh + ncol0 + 8 * q);
                        const __half2 *sv = reinterpret_cast<const __half2 *>(&sv4);
                        const float sc = 0.08838834764831845f;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __half2 h = __floats2half2_rn(v[8 * q + 2 * e] * sc * __low2float(sv[e]),
                                                          v[8 * q + 2 * e + 1] * sc * __high2float(sv[e]));
                            pc[q][e] = *reinterpret_cast<uint32_t *>(&h);
                        }
                    }
                    // 4 x 4 exchange: afterwards slot s of lane 4g + i holds
                    // piece i of row 4g + s
#pragma unroll
                    for (int b = 2; b >= 1; b >>= 1) {
                        const bool hi = (lane & b) != 0;
#pragma unroll
                        for (int q0 = 0; q0 < 4; ++q0) {
                            if (q0 & b)
                                continue;
                            const int q1 = q0 ^ b;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const uint32_t send = hi ? pc[q0][e] : pc[q1][e];
                                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, b);
                                if (hi)
                                    pc[q0][e] = recv;
                                else
                                    pc[q1][e] = recv;
                            }
                        }
                    }
#pragma unroll
                    for (int sr = 0; sr < 4; ++sr)
                        if (row0 + sr < p.m)
                            *reinterpret_cast<uint4 *>(L.y + (int64_t)(row0 + sr) * L.n + ncol0 + 8 * gi) =
                                make_uint4(pc[sr][0], pc[sr][1], pc[sr][2], pc[sr][3]);
                }
            }
        }
    }
    // hand the accumulators back to the MMA issuer
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
        mbar_arrive(&bars.acc_empty);
    return true;
}


// Small-m epilogue of one segment [u, se): the accumulators hold output
// channel tn*256 + 128h + lane in TMEM lane `lane` of half h (columns
// [h nb, h nb + nb), batch b at column h nb + b).  Partial sums go to the slot
// as [column][lane] (coalesced over the lanes), the finishing segment sums
// them in segment order in TMEM, and the output rotation runs per batch row:
// 32 columns at a time pass through `ebuf` (32 x 128 fp32) so that each warp
// holds a 128-channel row (4 per lane) for the in-warp Hadamard.
__device__ __forceinline__ bool gemm_epilogue_wa(const GemmParams &p, GemmBars &bars, uint32_t tmem, float *ebuf,
                                                 int seg, uint32_t u, uint32_t se, uint32_t U, uint32_t G,
                                                 uint32_t KB)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int nrow = quarter * 32 + lane;  // output channel within a 128-channel half
    const int nb = p.nb;
    const int nchunks = (2 * nb) >> 5;  // 32-column chunks over both halves
    volatile int *abort_flag = &bars.abort;
    const uint32_t t = u / KB;  // one tile row: tile t is column block t
    const uint32_t tb = t * KB, te = tb + KB;
    const bool whole = u == tb && se == te;
    const int tn = (int)t;
    if (!warp_wait(&bars.acc_full, (uint32_t)seg & 1u, p.wait_ns, 1000)) {
        if (lane == 0) {
            record_timeout(p.status);
            *abort_flag = 1;
        }
        return false;
    }
    tc_fence_after();
    if (*abort_flag)
        return false;
    int nseg = 1, c_lo = 0;
    bool finish = true;
    if (!whole) {
        c_lo = gemm_owner(tb, U, G);
        nseg = gemm_owner(te - 1, U, G) - c_lo + 1;
        float *slot = p.partials + (size_t)gemm_slot(blockIdx.x, tb, U, G) * kPartialFloats;
#pragma unroll 1
        for (int cc = 0; cc < nchunks; ++cc) {
            uint32_t r[32];
            EXL3_TMEM_LD32(tmem + lane_base + (uint32_t)(32 * cc), r);
#pragma unroll
            for (int j = 0; j < 32; ++j)
                __stcg(slot + (32 * cc + j) * 128 + nrow, __uint_as_float(r[j]));
        }
        __threadfence();
        epi_sync();
        if (warp == kWarpEpi0 && lane == 0) {
            const uint32_t prev = atomicAdd(&p.counters[t], 1u);
            const int last = prev == (uint32_t)(nseg - 1) ? 1 : 0;
            if (last) {
                __threadfence();
                p.counters[t] = 0u;  // every segment has arrived: re-arm for the next call
            }
            bars.ticket = last;
        }
        epi_sync();
        finish = bars.ticket != 0;
    }
    if (finish && !whole) {
        // every segment's partials, summed in segment order in TMEM
#pragma unroll 1
        for (int j = 0; j < nseg; ++j) {
            const float *src = p.partials + (size_t)gemm_slot((uint32_t)(c_lo + j), tb, U, G) * kPartialFloats + nrow;
#pragma unroll 1
            for (int cc = 0; cc < nchunks; ++cc) {
                float q[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    q[i] = __ldcg(src + (32 * cc + i) * 128);
                const uint32_t ta = tmem + lane_base + (uint32_t)(32 * cc);
                uint32_t r[32];
                if (j == 0) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r[i] = __float_as_uint(q[i]);
                } else {
                    EXL3_TMEM_LD32(ta, r);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r[i] = __float_as_uint(__uint_as_float(r[i]) + q[i]);
                }
                EXL3_TMEM_ST32(ta, r);
            }
            tmem_wait_st();
        }
    }
    if (finish) {
        // the last tile of n = 256j + 128 carries only channel half 0
        const GemmLayer &L = p.L[gemm_layer_of(p, tn)];
        const int tnl = tn - L.tn_begin;  // tile column within the layer
        const int fchunks = (tnl + 1) * kBN > L.n ? nchunks / 2 : nchunks;
#pragma unroll 1
        for (int cc = 0; cc < fchunks; ++cc) {
            const int h = (32 * cc) / nb, b0 = 32 * cc - h * nb;
            uint32_t r[32];
            EXL3_TMEM_LD32(tmem + lane_base + (uint32_t)(32 * cc), r);
#pragma unroll
            for (int j = 0; j < 32; ++j)
                ebuf[j * 128 + nrow] = __uint_as_float(r[j]);
            epi_sync();
            const int ncol = tnl * kBN + h * 128 + 4 * lane;
            const uint2 sv2 = *reinterpret_cast<const uint2 *>(L.svh + ncol);
            const __half2 *sv = reinterpret_cast<const __half2 *>(&sv2);
#pragma unroll 1
            for (int i = 0; i < 8; ++i) {
                const int j = quarter * 8 + i;
                if (b0 + j < p.m) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(ebuf + j * 128 + 4 * lane);
                    float v[4] = {v4.x, v4.y, v4.z, v4.w};
                    warp_fwht128(v);
                    const float sc = 0.08838834764831845f;
                    __half2 o0 = __floats2half2_rn(v[0] * sc * __low2float(sv[0]), v[1] * sc * __high2float(sv[0]));
                    __half2 o1 = __floats2half2_rn(v[2] * sc * __low2float(sv[1]), v[3] * sc * __high2float(sv[1]));
                    uint2 out;
                    out.x = *reinterpret_cast<uint32_t *>(&o0);
                    out.y = *reinterpret_cast<uint32_t *>(&o1);
                    *reinterpret_cast<uint2 *>(L.y + (int64_t)(b0 + j) * L.n + ncol) = out;
                }
            }
            epi_sync();  // ebuf is refilled by the next chunk
        }
    }
    // hand the accumulators back to the MMA issuer
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
        mbar_arrive(&bars.acc_empty);
    return true;
}

template <int K, bool WA>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const GemmParams p)
{
    constexpr int TS = gemm_t_stages(K, WA);
    constexpr int kTrBytes = gemm_trellis_stage_bytes(K);
    constexpr int kTileRowBytes = (kBN / 16) * 32 * K;
    constexpr int AS = gemm_a_stage_bytes(WA);
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    GemmBars &bars = *reinterpret_cast<GemmBars *>(smem);
    unsigned char *aring = smem + 1024;
    unsigned char *bring = aring + kAStages * AS;
    float *ebuf = reinterpret_cast<float *>(bring + kBStages * kBStageBytes);  // small-m epilogue only
    unsigned char *tring = bring + kBStages * kBStageBytes + (WA ? kWaEpiBytes : 0);
    volatile int *abort_flag = &bars.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t U = p.units;
    const uint32_t G = (uint32_t)p.ctas;
    const uint32_t u0 = blockIdx.x * U / G, u1 = (blockIdx.x + 1) * U / G;
    const int nu = (int)(u1 - u0);
    const uint32_t KB = (uint32_t)p.kb_count;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&bars.afull[s], 1);
            mbar_init(&bars.aempty[s], 1);
        }
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(&bars.bfull[s], kDecWarps);
            mbar_init(&bars.bempty[s], 1);
        }
        for (int s = 0; s < TS; ++s) {
            mbar_init(&bars.tfull[s], 1);
            mbar_init(&bars.tempty[s], kDecWarps);
        }
        mbar_init(&bars.acc_full, 1);
        mbar_init(&bars.acc_empty, 4);
        mbar_init(&bars.drain, 1);
        bars.abort = 0;
        bars.ticket = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma)
        tmem_alloc(&bars.tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_slot;
    // weights (trellis) may stream at once; everything else waits for the
    // preceding kernel (x' comes from the rotation kernel just before)
    if (warp != kWarpProducerT)
        grid_dep_wait();

    if (warp == kWarpProducerA) {
        // ---------------------------------------------------- A producer ---
        if (lane == 0) {
            uint32_t t = u0 / KB;
            int kb = (int)(u0 - t * KB);
            int tm = (int)(t / p.tiles_n);
            int mt_count = (p.m - tm * kBM * kMT) > kBM ? kMT : 1;  // skip an all-padding M tile
            const unsigned char *xt = p.L[gemm_layer_of(p, (int)(t - (uint32_t)tm * p.tiles_n))].xt;
            int issued = 0;
            for (int i = 0; i < nu; ++i) {
                const int s = i % kAStages;
                if (!mbar_wait_sleep(&bars.aempty[s], ((uint32_t)(i / kAStages) & 1u) ^ 1u, p.wait_ns, 100)) {
                    record_timeout(p.status);
                    *abort_flag = 1;
                    break;
                }
                unsigned char *dst = aring + s * AS;
                if constexpr (WA) {
                    // the first nb rows (batches) of x' tile (0, kb): nb x 128 contiguous bytes
                    mbar_arrive_expect_tx(&bars.afull[s], (uint32_t)(p.nb * 128));
                    bulk_g2s(dst, xt + (int64_t)kb * kATileBytes, (uint32_t)(p.nb * 128), &bars.afull[s]);
                } else {
                    mbar_arrive_expect_tx(&bars.afull[s], (uint32_t)(mt_count * kATileBytes));
                    for (int mt = 0; mt < mt_count; ++mt) {
                        const int64_t tile = (int64_t)(tm * kMT + mt) * (p.k / kBK) + kb;
                        bulk_g2s(dst + mt * kATileBytes, xt + tile * kATileBytes, kATileBytes, &bars.afull[s]);
                    }
                }
                issued = i + 1;
                if (++kb == (int)KB) {
                    kb = 0;
                    ++t;
                    tm = (int)(t / p.tiles_n);
                    mt_count = (p.m - tm * kBM * kMT) > kBM ? kMT : 1;
                    xt = p.L[gemm_layer_of(p, (int)(t - (uint32_t)tm * p.tiles_n))].xt;
                }
            }
            for (int i = (issued > kAStages ? issued - kAStages : 0); i < issued; ++i)
                if (!mbar_wait(&bars.afull[i % kAStages], (uint32_t)(i / kAStages) & 1u, kDefaultWaitNs))
                    record_timeout(p.status);
        }
    } else if (warp == kWarpProducerT) {
        // ---------------------------------------------- trellis producer ---
        if (lane == 0) {
            uint32_t t = u0 / KB;
            int kb = (int)(u0 - t * KB);
            int tn = (int)(t % p.tiles_n);
            // the tile column's layer: its trellis, a tile row of its matrix
            // (row_words), the column within it and whether it is half width
            const uint16_t *trel = nullptr;
            int64_t row_words = 0;
            int tnl = 0, row_bytes = kTileRowBytes;
            auto enter_column = [&]() {
                const GemmLayer &L = p.L[gemm_layer_of(p, tn)];
                trel = L.trellis;
                row_words = (int64_t)(L.n / 16) * 16 * K;
                tnl = tn - L.tn_begin;
                // the last tile of n = 256j + 128 has 8 trellis tiles per tile
                // row, not 16; the decoders decode stale bytes for the rest
                row_bytes = (tnl + 1) * kBN > L.n ? kTileRowBytes / 2 : kTileRowBytes;
            };
            enter_column();
            int issued = 0;
            for (int i = 0; i < nu; ++i) {
                const int s = i % TS;
                if (!mbar_wait_sleep(&bars.tempty[s], ((uint32_t)(i / TS) & 1u) ^ 1u, p.wait_ns, 200)) {
                    record_timeout(p.status);
                    *abort_flag = 1;
                    break;
                }
                unsigned char *dst = tring + s * kTrBytes;
                mbar_arrive_expect_tx(&bars.tfull[s], (uint32_t)((kBK / 16) * row_bytes));
                const uint16_t *src = trel + (int64_t)kb * (kBK / 16) * row_words + (int64_t)tnl * 16 * 16 * K;
#pragma unroll
                for (int r = 0; r < kBK / 16; ++r)
                    bulk_g2s(dst + r * kTileRowBytes, src + r * row_words, (uint32_t)row_bytes, &bars.tfull[s]);
                issued = i + 1;
                if (++kb == (int)KB) {
                    kb = 0;
                    ++t;
                    tn = (int)(t % p.tiles_n);
                    enter_column();
                }
            }
            for (int i = (issued > TS ? issued - TS : 0); i < issued; ++i)
                if (!mbar_wait(&bars.tfull[i % TS], (uint32_t)(i / TS) & 1u, kDefaultWaitNs))
                    record_timeout(p.status);
        }
    } else if (warp == kWarpMma) {
        // ----------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            const uint32_t idesc = WA ? gemm_idesc_wa(p.nb) : gemm_idesc();
            uint32_t t = u0 / KB;
            int kb = (int)(u0 - t * KB);
            int mt_count = (p.m - (int)(t / p.tiles_n) * kBM * kMT) > kBM ? kMT : 1;
            int seg = 0;
            bool ok = true;
            for (int i = 0; i < nu; ++i) {
                const bool seg_start = i == 0 || kb == 0;
                const bool seg_end = i == nu - 1 || kb == (int)KB - 1;
                if (seg_start && seg > 0) {
                    // the epilogue has read (and released) the previous accumulators
                    if (!mbar_wait(&bars.acc_empty, (uint32_t)(seg - 1) & 1u, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                const int sa = i % kAStages, sb = i % kBStages;
                if (!mbar_wait(&bars.afull[sa], (uint32_t)(i / kAStages) & 1u, p.wait_ns) ||
                    !mbar_wait(&bars.bfull[sb], (uint32_t)(i / kBStages) & 1u, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = smem_addr(aring + sa * AS);
                const uint32_t b0 = smem_addr(bring + sb * kBStageBytes);
                if constexpr (WA) {
                    // weights (the decoded stage, MN-major: 64-channel groups at
                    // 8192 B, 8-row k atoms at 1024 B) as A, one MMA per
                    // 128-channel half h into TMEM columns [h nb, h nb + nb)
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t xdesc = smem_desc(a0 + kk * 32, 16, 1024);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint64_t wdesc = smem_desc(b0 + h * 16384 + kk * 2048, 8192, 1024);
                            mma_f16_ss(tmem + (uint32_t)(h * p.nb), wdesc, xdesc, idesc,
                                       (!seg_start || kk) ? 1u : 0u);
                        }
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t bdesc = smem_desc(b0 + kk * 2048, 8192, 1024);
                        for (int mt = 0; mt < mt_count; ++mt) {
                            const uint64_t adesc = smem_desc(a0 + mt * kATileBytes + kk * 32, 16, 1024);
                            mma_f16_ss(tmem + (uint32_t)(mt * kBN), adesc, bdesc, idesc,
                                       (!seg_start || kk) ? 1u : 0u);
                        }
                    }
                }
                mma_commit(&bars.aempty[sa]);
                mma_commit(&bars.bempty[sb]);
                if (seg_end) {
                    mma_commit(&bars.acc_full);
                    ++seg;
                }
                if (++kb == (int)KB) {
                    kb = 0;
                    ++t;
                    mt_count = (p.m - (int)(t / p.tiles_n) * kBM * kMT) > kBM ? kMT : 1;
                }
            }
            if (!ok) {
                record_timeout(p.status);
                *abort_flag = 1;
            }
            // make sure no MMA is still writing TMEM when the CTA tears down
            mma_commit(&bars.drain);
            if (!mbar_wait(&bars.drain, 0, kDefaultWaitNs))
                record_timeout(p.status);
        }
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
        // ---------------------------------------------- epilogue warps ---
        uint32_t seg_u = u0;
        for (int seg = 0; seg_u < u1; ++seg) {
            const uint32_t te = (seg_u / KB + 1) * KB;
            const uint32_t seg_e = te < u1 ? te : u1;
            const bool ok = WA ? gemm_epilogue_wa(p, bars, tmem, ebuf, seg, seg_u, seg_e, U, G, KB)
                               : gemm_epilogue(p, bars, tmem, seg, seg_u, seg_e, U, G, KB);
            if (!ok)
                break;
            seg_u = seg_e;
        }
    } else if (warp >= kWarpDec0 && warp < kWarpDec0 + kDecWarps) {
        // ------------------------------------------------------- decoders ---
        // 4 tiles per warp; lane l decodes rows 2(l%8) and 2(l%8)+1 of tile
        // l/8 (one parity per call: compile-time bit windows)
        static_assert((kBK / 16) * (kBN / 16) == 4 * kDecWarps, "tiles per unit");
        const int dw = warp - kWarpDec0;
        const int T = dw * 4 + (lane >> 3);
        const int trow = T / (kBN / 16), tcol = T - (T / (kBN / 16)) * (kBN / 16);
        const int toff = trow * kTileRowBytes + tcol * 32 * K;
        const int r0 = 2 * (lane & 7);
        for (int i = 0; i < nu; ++i) {
            const int st = i % TS, sb = i % kBStages;
            if (!warp_wait_uniform(&bars.tfull[st], (uint32_t)(i / TS) & 1u, p.wait_ns) ||
                !warp_wait_uniform(&bars.bempty[sb], ((uint32_t)(i / kBStages) & 1u) ^ 1u, p.wait_ns)) {
                if (lane == 0) {
                    record_timeout(p.status);
                    *abort_flag = 1;
                }
                break;
            }
            const uint32_t *tw = reinterpret_cast<const uint32_t *>(tring + st * kTrBytes + toff);
            unsigned char *bt = bring + sb * kBStageBytes;
            decode_row_to_b<K, 0>(tw, r0, p.cb, bt, trow, tcol);
            decode_row_to_b<K, 1>(tw, r0 + 1, p.cb, bt, trow, tcol);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.bfull[sb]);
                mbar_arrive(&bars.tempty[st]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------- dispatch ---

constexpr size_t kGemmSyncArea = 64 * 1024;

struct GemmPlan {
    int64_t tiles, units;
    int tiles_n, kb_count, ctas;
    size_t counters, xt, xt_bytes, partials, total;  // workspace layout (byte offsets, sizes)
};

// Plan of one launch over `count` layers with the same m, k and K and output
// widths n[0..count): tile columns are the layers' in order (each n = 256j or
// 256j + 128, whose last tile is half width).  Workspace: [0, 64 KB) status
// word and one ticket per tile; then each layer's tiled x'; then two fp32
// partial slots per CTA.
static GemmPlan gemm_plan(int64_t m, int64_t k, const int64_t *n, int count, int sms)
{
    GemmPlan pl;
    const int64_t tiles_m = (m + kBM * kMT - 1) / (kBM * kMT);
    pl.tiles_n = 0;
    for (int l = 0; l < count; ++l)
        pl.tiles_n += (int)((n[l] + kBN - 1) / kBN);
    pl.tiles = tiles_m * pl.tiles_n;
    pl.kb_count = (int)(k / kBK);
    pl.units = pl.tiles * pl.kb_count;
    // at least a quarter of a tile's k blocks per CTA: a tile is then split
    // over at most ~5 CTAs, which bounds the finishing CTA's partial-sum reads
    const int64_t min_units = pl.kb_count / 4 > 1 ? pl.kb_count / 4 : 1;
    const int64_t cap = (pl.units + min_units - 1) / min_units;
    pl.ctas = (int)(cap < sms ? cap : sms);
    pl.counters = 256;
    pl.xt = (pl.counters + (size_t)pl.tiles * 4 + 1023) / 1024 * 1024;
    // data only from 64 KB on: the words below (status, counters) are zero
    // after every call of either kind, so one workspace can serve GEMV and
    // GEMM calls of any shapes in turn
    pl.xt = pl.xt > kGemmSyncArea ? pl.xt : kGemmSyncArea;
    pl.xt_bytes = ((size_t)(tiles_m * kBM * kMT) * (size_t)k * 2 + 1023) / 1024 * 1024;
    pl.partials = pl.xt + (size_t)count * pl.xt_bytes;
    pl.total = pl.partials + (size_t)2 * pl.ctas * kPartialFloats * 4;
    return pl;
}

template <int K, bool WA>
static exl3_status launch_gemm_t(const GemmParams &p, cudaStream_t stream)
{
    constexpr int smem = gemm_smem_bytes(K, WA);
    auto kern = gemm_kernel<K, WA>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return EXL3_ERR_CUDA;
    if (launch_kernel(kern, dim3(p.ctas), dim3(kGemmThreads), (size_t)smem, stream, p) != cudaSuccess)
        return EXL3_ERR_CUDA;
    return launch_status();
}

}  // namespace exl3

namespace exl3 {

// One rotation launch and one GEMM launch over `count` (1 .. kGemmMaxLayers)
// layers with the same m, k and K, with the workspace laid out by gemm_plan.
static exl3_status run_gemm_group(const exl3_linear *layers, int count, int64_t m, unsigned char *ws,
                                  size_t ws_bytes, cudaStream_t s)
{
    const int64_t k = layers[0].k;
    const int K = layers[0].K;
    int64_t n[kGemmMaxLayers];
    for (int l = 0; l < count; ++l)
        n[l] = layers[l].n;
    const GemmPlan pl = gemm_plan(m, k, n, count, num_sms());
    if (pl.units * (int64_t)pl.ctas >= ((int64_t)1 << 32))
        return EXL3_ERR_UNSUPPORTED;  // split the call along m (about 10^14 multiply-adds per call)
    if (!ws || !aligned16(ws) || ws_bytes < pl.total)
        return EXL3_ERR_WORKSPACE;
    GemmRotParams rp;
    rp.nlayers = count;
    rp.m = (int)m;
    rp.k = (int)k;
    GemmParams p;
    p.nlayers = count;
    int tn = 0;
    for (int l = 0; l < count; ++l) {
        unsigned char *xt = ws + pl.xt + (size_t)l * pl.xt_bytes;  // 1024-byte offsets from an aligned base
        rp.x[l] = (const __half *)layers[l].x;
        rp.suh[l] = (const __half *)layers[l].suh;
        rp.xt[l] = xt;
        GemmLayer &L = p.L[l];
        L.xt = xt;
        L.trellis = layers[l].trellis;
        L.svh = (const __half *)layers[l].svh;
        L.y = (__half *)layers[l].y;
        L.n = (int)n[l];
        L.tn_begin = tn;
        tn += (int)((n[l] + kBN - 1) / kBN);
    }
    int64_t rot_grid = (count * m * (k / 128) + 7) / 8;
    if (rot_grid > 148 * 16)
        rot_grid = 148 * 16;
    if (launch_kernel(rotate_tiled_kernel, dim3((unsigned)rot_grid), dim3(256), 0, s, rp) != cudaSuccess ||
        launch_status() != EXL3_OK)
        return EXL3_ERR_CUDA;
    p.partials = reinterpret_cast<float *>(ws + pl.partials);
    p.counters = reinterpret_cast<uint32_t *>(ws + pl.counters);
    p.status = (uint32_t *)ws;
    p.m = (int)m;
    p.k = (int)k;
    p.tiles_n = pl.tiles_n;
    p.kb_count = pl.kb_count;
    p.units = (uint32_t)pl.units;
    p.ctas = pl.ctas;
    p.wait_ns = wait_limit_ns();
    p.cb = codebook_constants();
    const bool wa = m <= kWaMaxM;
    p.nb = wa ? (int)((m + 31) & ~(int64_t)31) : 0;
    if (wa) {
        switch (K) {
        case 1: return launch_gemm_t<1, true>(p, s);
        case 2: return launch_gemm_t<2, true>(p, s);
        case 3: return launch_gemm_t<3, true>(p, s);
        case 4: return launch_gemm_t<4, true>(p, s);
        case 5: return launch_gemm_t<5, true>(p, s);
        case 6: return launch_gemm_t<6, true>(p, s);
        case 7: return launch_gemm_t<7, true>(p, s);
        default: return launch_gemm_t<8, true>(p, s);
        }
    }
    switch (K) {
    case 1: return launch_gemm_t<1, false>(p, s);
    case 2: return launch_gemm_t<2, false>(p, s);
    case 3: return launch_gemm_t<3, false>(p, s);
    case 4: return launch_gemm_t<4, false>(p, s);
    case 5: return launch_gemm_t<5, false>(p, s);
    case 6: return launch_gemm_t<6, false>(p, s);
    case 7: return launch_gemm_t<7, false>(p, s);
    default: return launch_gemm_t<8, false>(p, s);
    }
}

// Argument checks of a multi call: every layer valid, and all with the first
// layer's k and K (they share one launch's k loop and decode).
static exl3_status check_gemm_multi(const exl3_linear *layers, int count, int64_t m)
{
    if (!layers || count < 1)
        return EXL3_ERR_INVALID_ARG;
    for (int l = 0; l < count; ++l) {
        const exl3_linear &d = layers[l];
        const exl3_status st = check_linear_args(d.x, d.trellis, d.suh, d.svh, d.y, m, d.k, d.n, d.K);
        if (st != EXL3_OK)
            return st;
        if (d.k != layers[0].k || d.K != layers[0].K)
            return EXL3_ERR_UNSUPPORTED;
    }
    return EXL3_OK;
}

}  // namespace exl3

extern "C" size_t exl3_gemm_workspace_size(int64_t m, int64_t k, int64_t n, int K)
{
    if (m < 1 || k < 128 || n < 128 || (k % 128) || (n % 128) || K < 1 || K > 8)
        return 0;
    return exl3::gemm_plan(m, k, &n, 1, exl3::num_sms()).total;
}

extern "C" exl3_status exl3_gemm(const void *x, const uint16_t *trellis, const void *suh,
                                 const void *svh, void *y, int64_t m, int64_t k, int64_t n, int K,
                                 void *workspace, size_t workspace_bytes, void *stream)
{
    using namespace exl3;
    const exl3_status st = check_linear_args(x, trellis, suh, svh, y, m, k, n, K);
    if (st != EXL3_OK)
        return st;
    exl3_linear d;
    d.x = x;
    d.trellis = trellis;
    d.suh = suh;
    d.svh = svh;
    d.y = y;
    d.k = k;
    d.n = n;
    d.K = K;
    return run_gemm_group(&d, 1, m, (unsigned char *)workspace, workspace_bytes, (cudaStream_t)stream);
}

extern "C" size_t exl3_gemm_multi_workspace_size(const exl3_linear *layers, int count, int64_t m)
{
    using namespace exl3;
    if (check_gemm_multi(layers, count, m) != EXL3_OK)
        return 0;
    size_t most = 0;
    for (int l0 = 0; l0 < count; l0 += kGemmMaxLayers) {
        const int c = count - l0 < kGemmMaxLayers ? count - l0 : kGemmMaxLayers;
        int64_t n[kGemmMaxLayers];
        for (int l = 0; l < c; ++l)
            n[l] = layers[l0 + l].n;
        const size_t b = gemm_plan(m, layers[0].k, n, c, num_sms()).total;
        most = b > most ? b : most;
    }
    return most;
}

extern "C" exl3_status exl3_gemm_multi(const exl3_linear *layers, int count, int64_t m, void *workspace,
                                       size_t workspace_bytes, void *stream)
{
    using namespace exl3;
    const exl3_status st = check_gemm_multi(layers, count, m);
    if (st != EXL3_OK)
        return st;
    for (int l0 = 0; l0 < count; l0 += kGemmMaxLayers) {
        const int c = count - l0 < kGemmMaxLayers ? count - l0 : kGemmMaxLayers;
        const exl3_status rs =
            run_gemm_group(layers + l0, c, m, (unsigned char *)workspace, workspace_bytes, (cudaStream_t)stream);
        if (rs != EXL3_OK)
            return rs;
    }
    return EXL3_OK;
}
