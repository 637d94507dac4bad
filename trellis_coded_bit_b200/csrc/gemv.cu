// gemv.cu -- exl3_gemv: y = svh .* H(H(x .* suh) . W_hat) for 1 <= m <= 16,
// with W_hat decoded on the fly from the trellis (EXL3 GEMM kernel article,
// section 小批量GEMV: in decoding the bottleneck moves from compute to memory
// bandwidth, so a dedicated GEMV path streams the quantised weights once).
//
// B200 design (the pages' consumer-GPU GEMV is prior art, not copied):
//   * grid = (n/128 column blocks) x (k splits); one CTA = 1 producer warp +
//     8 consumer warps, all on the same 128 output columns.
//   * The producer warp streams the CTA's tile rows (8 tiles = 128 columns x
//     16 input channels, 2K*128 bytes, contiguous in the trellis) into a ring
//     of shared-memory stages with cp.async.bulk (no multicast), signalled on
//     mbarriers; consumers release stages on a second set of mbarriers.  All
//     waits are bounded (timeout -> status word, early exit).
//   * Consumer warp w takes tile row w of every stage.  Lane (g, t) decodes,
//     for each of 4 row groups q and 2 column halves, the run of 8
//     consecutive weights of tile row 4q+t, columns 8(g&1).. of tile
//     (4*half + g/2): one 64-bit read of the bit string, 8 windows, 8
//     codebook words -- everything stays in registers.
//   * The MAC runs on the tensor cores (mma.sync m16n8k16, fp32 accumulate).
//     A codebook word's two fp16 halves are placed as a pair of k slots in B
//     and the activation is duplicated across that pair in A, so the tensor
//     core forms x*(hi + lo) exactly in fp32; the fp16 rounding of hi + lo
//     that defines W_hat is skipped (the difference is at most half an fp16
//     ulp of each weight, far inside the output tolerance).  The 8 weights of
//     a run go to 4 MMAs (2 per MMA: k-pairs t and t+4 of output column
//     parity 0 and 1); A rows are (batch, column parity) and zero elsewhere,
//     so column parity never mixes.  Batch rows 0..7 per group, 2 groups for
//     m > 8.
//   * x' = H(x .* suh)/sqrt(128) for the CTA's k range is computed once into
//     shared memory (fp32 butterflies, rounded to fp16, stored duplicated).
//   * Split-k: every CTA writes fp32 partials; the last CTA to arrive on the
//     column block's counter (atomic ticket, no spinning) sums them in split
//     order (deterministic), applies H/sqrt(128) and svh, writes fp16 y and
//     re-arms the counter.
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

constexpr int kGemvWarpsK = 8;        // consumer warps per CTA (one tile row each per stage)
constexpr int kGemvThreads = 32 * (kGemvWarpsK + 1);
constexpr int kGemvStages = 4;
constexpr int kGemvRowsPerStage = kGemvWarpsK;  // tile rows per stage

struct GemvParams {
    const __half *x;
    const uint16_t *trellis;
    const __half *suh;
    const __half *svh;
    __half *y;
    int m, k, n;
    int splits;
    int rows_per_split;  // tile rows (of 16 input channels) per split, last may be shorter
    float *partials;     // [splits][m][n]
    uint32_t *counters;  // [n / 128]
    uint32_t *status;
    uint64_t wait_ns;    // bound of every device wait
};

// Shared memory carve-up (bytes), all 16-byte aligned.
struct GemvSmem {
    int bars;      // 2 * stages mbarriers
    int flag;      // last-CTA flag
    int xs;        // dup'd x' [k_local][m] u32
    int stage;     // stages of tile rows
    int red;       // [warps][m][128] f32 reduction buffer (aliases stages)
    int total;
};

template <int K>
__host__ __device__ constexpr int gemv_stage_bytes()
{
    return kGemvRowsPerStage * 8 * 32 * K;  // 8 tiles of 32K bytes per tile row
}

__host__ __device__ inline GemvSmem gemv_smem_layout(int K, int m, int rows_per_split)
{
    GemvSmem s;
    s.bars = 0;
    s.flag = 2 * kGemvStages * 8;
    s.xs = (s.flag + 16 + 15) & ~15;
    const int xs_bytes = rows_per_split * 16 * m * 4;
    s.stage = (s.xs + xs_bytes + 127) & ~127;
    const int stage_bytes = kGemvRowsPerStage * 8 * 32 * K;
    const int red_bytes = kGemvWarpsK * m * 128 * 4;
    s.red = s.stage;
    const int body = kGemvStages * stage_bytes > red_bytes ? kGemvStages * stage_bytes : red_bytes;
    s.total = s.stage + body;
    return s;
}

template <int K, int MG>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvParams p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const GemvSmem L = gemv_smem_layout(K, p.m, p.rows_per_split);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + kGemvStages;
    volatile int *flag = reinterpret_cast<volatile int *>(smem + L.flag);
    uint32_t *xs = reinterpret_cast<uint32_t *>(smem + L.xs);
    unsigned char *stage_base = smem + L.stage;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = blockIdx.x, split = blockIdx.y;
    const int m = p.m, n = p.n;
    const int tn_count = n >> 4;
    const int row_begin = split * p.rows_per_split;
    int row_end = row_begin + p.rows_per_split;
    const int tr_total = p.k >> 4;
    if (row_end > tr_total)
        row_end = tr_total;
    const int rows = row_end - row_begin;
    const int n_stage_iters = (rows + kGemvRowsPerStage - 1) / kGemvRowsPerStage;
    constexpr int kStageBytes = gemv_stage_bytes<K>();
    constexpr int kRowBytes = 8 * 32 * K;  // one tile row of 8 tiles

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemvStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kGemvWarpsK);
        }
        *flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kGemvWarpsK) {
        // ------------------------------------------------------ producer ---
        if (lane == 0) {
            bool ok = true;
            int issued = 0;
            for (int it = 0; it < n_stage_iters; ++it) {
                const int s = it % kGemvStages;
                const uint32_t ph = (uint32_t)(it / kGemvStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, p.wait_ns)) {
                    ok = false;
                    break;
                }
                const int r0 = row_begin + it * kGemvRowsPerStage;
                int nr = row_end - r0;
                if (nr > kGemvRowsPerStage)
                    nr = kGemvRowsPerStage;
                mbar_arrive_expect_tx(&full[s], (uint32_t)(nr * kRowBytes));
                for (int r = 0; r < nr; ++r) {
                    const uint16_t *src =
                        p.trellis + ((int64_t)(r0 + r) * tn_count + (int64_t)nb * 8) * 16 * K;
                    bulk_g2s(stage_base + s * kStageBytes + r * kRowBytes, src, kRowBytes, &full[s]);
                }
                issued = it + 1;
            }
            if (!ok)
                record_timeout(p.status);
            // never leave while copies into this CTA's shared memory are in flight
            for (int it = (issued > kGemvStages ? issued - kGemvStages : 0); it < issued; ++it) {
                const int s = it % kGemvStages;
                if (!mbar_wait(&full[s], (uint32_t)(it / kGemvStages) & 1u, kDefaultWaitNs))
                    record_timeout(p.status);
            }
        }
        return;
    }

    // ----------------------------------------------------------- consumers ---
    // x' for this split's k range: warp w rotates 128-channel blocks w, w+8, ...
    {
        const int k0 = row_begin * 16;
        const int nblk = rows * 16 / 128;
        for (int job = warp; job < nblk * m; job += kGemvWarpsK) {
            const int b = job / nblk, blk = job - (job / nblk) * nblk;
            const int c = k0 + blk * 128 + lane * 4;
            const uint2 raw = *reinterpret_cast<const uint2 *>(p.x + (int64_t)b * p.k + c);
            const uint2 sr = *reinterpret_cast<const uint2 *>(p.suh + c);
            const __half2 *xv = reinterpret_cast<const __half2 *>(&raw);
            const __half2 *sv = reinterpret_cast<const __half2 *>(&sr);
            float v[4] = {__low2float(xv[0]) * __low2float(sv[0]), __high2float(xv[0]) * __high2float(sv[0]),
                          __low2float(xv[1]) * __low2float(sv[1]), __high2float(xv[1]) * __high2float(sv[1])};
            warp_fwht128(v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __half h = __float2half_rn(v[e] * 0.08838834764831845f);
                const uint32_t hb = (uint32_t)__half_as_ushort(h);
                xs[(blk * 128 + lane * 4 + e) * m + b] = hb | (hb << 16);
            }
        }
    }
    asm volatile("bar.sync 1, %0;\n" ::"r"(32 * kGemvWarpsK));

    const int g = lane >> 2, t = lane & 3;
    const bool odd = (g & 1) != 0;
    float acc[MG][2][4][4];
#pragma unroll
    for (int a = 0; a < MG; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int d = 0; d < 4; ++d)
                    acc[a][b][c][d] = 0.f;

    bool ok = true;
    for (int it = 0; it < n_stage_iters; ++it) {
        const int s = it % kGemvStages;
        if (!warp_wait(&full[s], (uint32_t)(it / kGemvStages) & 1u, p.wait_ns)) {
            ok = false;
            break;
        }
        const int rl = it * kGemvRowsPerStage + warp;  // local tile row of this warp
        if (rl < rows) {
            const uint32_t *row_tiles =
                reinterpret_cast<const uint32_t *>(stage_base + s * kStageBytes + warp * kRowBytes);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int kl = rl * 16 + 4 * q + t;
                uint32_t A[MG][4];
#pragma unroll
                for (int mg = 0; mg < MG; ++mg) {
                    const int ba = 8 * mg + (g >> 1), bb = ba + 4;
                    const uint32_t xa = ba < m ? xs[kl * m + ba] : 0u;
                    const uint32_t xb = bb < m ? xs[kl * m + bb] : 0u;
                    A[mg][0] = odd ? 0u : xa;
                    A[mg][1] = odd ? 0u : xb;
                    A[mg][2] = odd ? xa : 0u;
                    A[mg][3] = odd ? xb : 0u;
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t *tile = row_tiles + (4 * h + (g >> 1)) * 8 * K;
                    const int start = (16 * (4 * q + t) + 8 * (g & 1)) * K;
                    uint32_t st[8];
                    if constexpr (K <= 6) {
                        run_states<K, 8>(tile, start, st);
                    } else {
                        uint32_t lo[4], hi[4];
                        run_states<K, 4>(tile, start, lo);
                        run_states<K, 4>(tile, start + 4 * K, hi);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            st[j] = lo[j];
                            st[4 + j] = hi[j];
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t b0 = codebook_word(st[2 * j]);
                        const uint32_t b1 = codebook_word(st[2 * j + 1]);
#pragma unroll
                        for (int mg = 0; mg < MG; ++mg)
                            mma_16816(acc[mg][h][j], A[mg], b0, b1);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);
    }
    if (!ok) {
        record_timeout(p.status);
        *flag = -1;
    }

    // ------------------------------------------------- reduce across warps ---
    asm volatile("bar.sync 1, %0;\n" ::"r"(32 * kGemvWarpsK));
    float *red = reinterpret_cast<float *>(smem + L.red);  // [warp][m][128]
    // accumulator element (mg, h, j, e): row i = g (+8 for e >= 2) -> batch
    // 8mg + i/2, column parity i&1; n-slot 2t (+1 for odd e) -> column group
    // 64h + 8*slot, column within group 2j + parity.
#pragma unroll
    for (int mg = 0; mg < MG; ++mg)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = g + ((e >> 1) << 3);
                    const int b = 8 * mg + (i >> 1);
                    const int slot = 2 * t + (e & 1);
                    const int col = 64 * h + 8 * slot + 2 * j + (i & 1);
                    if (b < m)
                        red[(warp * m + b) * 128 + col] = acc[mg][h][j][e];
                }
    asm volatile("bar.sync 1, %0;\n" ::"r"(32 * kGemvWarpsK));
    if (*flag < 0)
        return;
    const int tid = threadIdx.x;  // 0 .. 255 among consumers
    for (int e = tid; e < m * 128; e += 32 * kGemvWarpsK) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kGemvWarpsK; ++w)
            sum += red[w * m * 128 + e];
        red[e] = sum;  // row 0 of the buffer now holds the CTA's partial; w = 0 is read first
    }
    asm volatile("bar.sync 1, %0;\n" ::"r"(32 * kGemvWarpsK));

    if (p.splits > 1) {
        // publish partial, take a ticket; the last CTA finishes the block
        for (int e = tid; e < m * 128; e += 32 * kGemvWarpsK) {
            const int b = e >> 7, c = e & 127;
            p.partials[((int64_t)split * m + b) * n + nb * 128 + c] = red[e];
        }
        __threadfence();
        asm volatile("bar.sync 1, %0;\n" ::"r"(32 * kGemvWarpsK));
        if (tid == 0) {
            const uint32_t ticket = atomicAdd(&p.counters[nb], 1u);
            *flag = (ticket == (uint32_t)(p.splits - 1)) ? 1 : 0;
        }
        asm volatile("bar.sync 1, %0;\n" ::"r"(32 * kGemvWarpsK));
        if (*flag != 1)
            return;
        __threadfence();
        for (int e = tid; e < m * 128; e += 32 * kGemvWarpsK) {
            const int b = e >> 7, c = e & 127;
            float sum = 0.f;
            for (int sp = 0; sp < p.splits; ++sp)
                sum += __ldcg(&p.partials[((int64_t)sp * m + b) * n + nb * 128 + c]);
            red[e] = sum;
        }
        if (tid == 0)
            p.counters[nb] = 0u;
        asm volatile("bar.sync 1, %0;\n" ::"r"(32 * kGemvWarpsK));
    }

    // ------------------------------------ output rotation, scales, fp16 y ---
    for (int b = warp; b < m; b += kGemvWarpsK) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            v[e] = red[b * 128 + lane * 4 + e];
        warp_fwht128(v);
        const int c = nb * 128 + lane * 4;
        const uint2 sr = *reinterpret_cast<const uint2 *>(p.svh + c);
        const __half2 *sv = reinterpret_cast<const __half2 *>(&sr);
        const float s = 0.08838834764831845f;
        __half2 o0 = __floats2half2_rn(v[0] * s * __low2float(sv[0]), v[1] * s * __high2float(sv[0]));
        __half2 o1 = __floats2half2_rn(v[2] * s * __low2float(sv[1]), v[3] * s * __high2float(sv[1]));
        uint2 out;
        out.x = *reinterpret_cast<uint32_t *>(&o0);
        out.y = *reinterpret_cast<uint32_t *>(&o1);
        *reinterpret_cast<uint2 *>(p.y + (int64_t)b * n + c) = out;
    }
}

// ------------------------------------------------------------- dispatch ---

struct GemvPlan {
    int splits, rows_per_split, smem;
};

static int g_num_sms = 0;

static int num_sms()
{
    if (g_num_sms <= 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        g_num_sms = v;
    }
    return g_num_sms;
}

// Splits so that about two CTAs per SM are in flight; each split covers a
// whole number of 128-channel blocks (8 tile rows) and its rotated
// activations fit in 64 KB of shared memory.
static GemvPlan gemv_plan(int64_t m, int64_t k, int64_t n, int K, int sms)
{
    GemvPlan pl;
    const int64_t blocks_k = k / 128;
    const int64_t nblocks = n / 128;
    int64_t splits = (2 * sms + nblocks - 1) / nblocks;
    if (splits > blocks_k)
        splits = blocks_k;
    if (splits < 1)
        splits = 1;
    // shared-memory cap on the rotated activations: rows*16*m*4 <= 64 KB
    const int64_t max_blocks = (64 * 1024) / (128 * m * 4);
    int64_t per = (blocks_k + splits - 1) / splits;
    if (per > max_blocks)
        per = max_blocks;
    if (per < 1)
        per = 1;
    splits = (blocks_k + per - 1) / per;
    pl.splits = (int)splits;
    pl.rows_per_split = (int)(per * 8);
    pl.smem = gemv_smem_layout(K, (int)m, pl.rows_per_split).total;
    return pl;
}

size_t gemv_workspace_bytes(int64_t m, int64_t k, int64_t n, int K, int sms)
{
    const GemvPlan pl = gemv_plan(m, k, n, K, sms);
    size_t bytes = 256;                                // status word + padding
    bytes += (size_t)((n / 128) * 4 + 255) / 256 * 256;  // counters
    if (pl.splits > 1)
        bytes += (size_t)pl.splits * (size_t)m * (size_t)n * 4;
    return bytes;
}

template <int K, int MG>
static exl3_status launch_gemv_t(const GemvParams &p, int smem, cudaStream_t stream)
{
    auto kern = gemv_kernel<K, MG>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return EXL3_ERR_CUDA;
    dim3 grid((unsigned)(p.n / 128), (unsigned)p.splits);
    kern<<<grid, kGemvThreads, smem, stream>>>(p);
    return launch_status();
}

template <int MG>
static exl3_status launch_gemv_k(const GemvParams &p, int K, int smem, cudaStream_t stream)
{
    switch (K) {
    case 1: return launch_gemv_t<1, MG>(p, smem, stream);
    case 2: return launch_gemv_t<2, MG>(p, smem, stream);
    case 3: return launch_gemv_t<3, MG>(p, smem, stream);
    case 4: return launch_gemv_t<4, MG>(p, smem, stream);
    case 5: return launch_gemv_t<5, MG>(p, smem, stream);
    case 6: return launch_gemv_t<6, MG>(p, smem, stream);
    case 7: return launch_gemv_t<7, MG>(p, smem, stream);
    default: return launch_gemv_t<8, MG>(p, smem, stream);
    }
}

exl3_status run_gemv(const void *x, const uint16_t *trellis, const void *suh, const void *svh,
                     void *y, int64_t m, int64_t k, int64_t n, int K, void *workspace,
                     size_t workspace_bytes, cudaStream_t stream)
{
    const int sms = num_sms();
    const GemvPlan pl = gemv_plan(m, k, n, K, sms);
    if (!workspace || !aligned16(workspace) || workspace_bytes < gemv_workspace_bytes(m, k, n, K, sms))
        return EXL3_ERR_WORKSPACE;
    unsigned char *ws = (unsigned char *)workspace;
    GemvParams p;
    p.x = (const __half *)x;
    p.trellis = trellis;
    p.suh = (const __half *)suh;
    p.svh = (const __half *)svh;
    p.y = (__half *)y;
    p.m = (int)m;
    p.k = (int)k;
    p.n = (int)n;
    p.splits = pl.splits;
    p.rows_per_split = pl.rows_per_split;
    p.status = (uint32_t *)ws;
    p.counters = (uint32_t *)(ws + 256);
    p.partials = (float *)(ws + 256 + (size_t)((n / 128) * 4 + 255) / 256 * 256);
    p.wait_ns = wait_limit_ns();
    if (m <= 8)
        return launch_gemv_k<1>(p, K, pl.smem, stream);
    return launch_gemv_k<2>(p, K, pl.smem, stream);
}

}  // namespace exl3

extern "C" size_t exl3_gemv_workspace_size(int64_t m, int64_t k, int64_t n, int K)
{
    if (m < 1 || m > 16 || k < 128 || n < 128 || (k % 128) || (n % 128) || K < 1 || K > 8)
        return 0;
    return exl3::gemv_workspace_bytes(m, k, n, K, exl3::num_sms());
}

extern "C" exl3_status exl3_gemv(const void *x, const uint16_t *trellis, const void *suh,
                                 const void *svh, void *y, int64_t m, int64_t k, int64_t n, int K,
                                 void *workspace, size_t workspace_bytes, void *stream)
{
    using namespace exl3;
    const exl3_status st = check_linear_args(x, trellis, suh, svh, y, m, k, n, K);
    if (st != EXL3_OK)
        return st;
    if (m > 16)
        return EXL3_ERR_UNSUPPORTED;
    return run_gemv(x, trellis, suh, svh, y, m, k, n, K, workspace, workspace_bytes,
                    (cudaStream_t)stream);
}
