// gemv.cu -- exl3_gemv: y = svh .* H(H(x .* suh) . W_hat) for 1 <= m <= 16,
// with W_hat decoded on the fly from the trellis (EXL3 GEMM kernel article,
// section 小批量GEMV: in decoding the bottleneck moves from compute to memory
// bandwidth, so a dedicated GEMV path streams the quantised weights once).
//
// B200 design (the pages' consumer-GPU GEMV is prior art, not copied):
//   * grid = (n/128 column blocks) x (k splits), 8 warps per CTA, all on the
//     same 128 output columns (8 trellis tiles); warp w takes tile rows
//     w, w+8, ... of the CTA's k range.  The split count is chosen so the
//     CTAs fill whole waves of the GPU.
//   * Lane (g, t) owns tile g of the column block and, in each of 4 row
//     groups q, the whole tile row rho(q, t) (16 weights): rows are ordered
//     so that all lanes of a group share the row parity, which makes every
//     bit-window operation a compile-time byte permute (see row_states).
//     Loads go straight from HBM into registers in this fragment order
//     (read-only path, 8/16-byte vectors where aligned), one tile row ahead
//     of the math -- no shared-memory staging, no bank conflicts.
//   * The MAC runs on the tensor cores (mma.sync m16n8k16, fp32 accumulate):
//     a codebook word's two fp16 halves form a pair of k slots in B and the
//     activation is duplicated over that pair in A, so the tensor core forms
//     x*(hi + lo) exactly in fp32 (the fp16 rounding of hi + lo that defines
//     W_hat is skipped: at most half an fp16 ulp per weight, far inside the
//     output tolerance).  Weights 2j, 2j+1 of a lane's row feed MMA j (k
//     pairs t and t+4); A rows are (batch, column parity) with zeros
//     elsewhere, so parities never mix.  The activation fragments are kept in
//     shared memory as {x, 0, 0, x} records: one 8-byte load gives a lane its
//     (a0, a2) pair for either parity.  Batch rows 0..7 per group, two groups
//     for m > 8 (one decode feeds both).
//   * x' = H(x .* suh)/sqrt(128) for the CTA's k range is computed once into
//     those records (fp32 butterflies, rounded to fp16).
//   * Split-k: every CTA writes fp32 partials; the last CTA to arrive on the
//     column block's counter (atomic ticket, no spinning) sums them in split
//     order (deterministic), applies H/sqrt(128) and svh, writes fp16 y and
//     re-arms the counter.  Nothing in the kernel waits on another CTA.
//   * With EXL3_LAUNCH_PDL the first tile rows are requested before the
//     kernel waits for its predecessor (griddepcontrol), and the next kernel
//     is released as soon as this CTA's weight stream is consumed.
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = 32 * kGemvWarps;

struct GemvParams {
    const __half *x;
    const uint16_t *trellis;
    const __half *suh;
    const __half *svh;
    __half *y;
    int m, k, n;
    int splits;
    int rows_per_split;  // tile rows (16 input channels each) per split; last may be shorter
    float *partials;     // [splits][m][n]
    uint32_t *counters;  // [n / 128]
    Codebook cb;
};

// Activation records, in MMA A-fragment register order.  For batch group mg
// (batches 8mg..8mg+7), quad ba (batches 8mg+ba and 8mg+ba+4) and A-row
// parity p, a 16-byte record holds the lane's {a0, a1, a2, a3}:
//   p = 0: {x(8mg+ba), x(8mg+ba+4), 0, 0}     p = 1: {0, 0, x(8mg+ba), x(8mg+ba+4)}
// with x the rotated activation duplicated in both fp16 halves (absent batches
// are zero).  Only quads holding a batch < m are stored; per input channel
// there are rec_slots(m) records.
__host__ __device__ inline int rec_quads(int m, int mg)
{
    const int q = m - 8 * mg;
    return q <= 0 ? 0 : (q < 4 ? q : 4);
}

__host__ __device__ inline int rec_slots(int m)
{
    return 2 * (rec_quads(m, 0) + rec_quads(m, 1));
}

// Dynamic shared memory: a flag, one zero record, then the records
// [k_local][rec_slots] (16 B each), later reused as the cross-warp reduction
// buffer [warps][m][128] f32.
__host__ __device__ inline int gemv_smem_bytes(int m, int rows_per_split)
{
    const int rec = rows_per_split * 16 * rec_slots(m) * 16;
    const int red = kGemvWarps * m * 128 * 4;
    return 32 + (rec > red ? rec : red);
}

// Row of tile-row group q for lane t: groups 0,1 take the even rows, groups
// 2,3 the odd rows, so a group's lanes share the row parity.
__device__ __forceinline__ int row_of(int q, int t)
{
    return 2 * (4 * (q & 1) + t) + (q >> 1);
}

template <int K>
struct RowBuf {
    static constexpr int N =
        RowSpan<K, 0>::N32 > RowSpan<K, 1>::N32 ? RowSpan<K, 0>::N32 : RowSpan<K, 1>::N32;
    uint32_t w[4][N];
};

template <int K>
__device__ __forceinline__ void load_tile_row(const uint32_t *tile, int t, RowBuf<K> &b)
{
    load_row<K, 0>(tile, row_of(0, t), b.w[0]);
    load_row<K, 0>(tile, row_of(1, t), b.w[1]);
    load_row<K, 1>(tile, row_of(2, t), b.w[2]);
    load_row<K, 1>(tile, row_of(3, t), b.w[3]);
}

// Activation-record address of one lane for one batch group (zero record,
// stride 0, when the lane's quad holds no batch).
struct RecPtr {
    const unsigned char *base;
    int stride;
};

template <int K, int MG>
__device__ __forceinline__ void mac_tile_row(const RowBuf<K> &buf, int kl0, const RecPtr (&rp)[MG], int t,
                                             const Codebook &cb, float (&acc)[MG][8][4])
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int kl = kl0 + row_of(q, t);
        uint32_t A[MG][4];
#pragma unroll
        for (int mg = 0; mg < MG; ++mg) {
            const uint4 r = *reinterpret_cast<const uint4 *>(rp[mg].base + kl * rp[mg].stride);
            A[mg][0] = r.x;
            A[mg][1] = r.y;
            A[mg][2] = r.z;
            A[mg][3] = r.w;
        }
        uint32_t s[16];
        if (q < 2)
            row_states<K, RowSpan<K, 0>::P>(buf.w[q], s);
        else
            row_states<K, RowSpan<K, 1>::P>(buf.w[q], s);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t b0 = codebook_word(s[2 * j], cb);
            const uint32_t b1 = codebook_word(s[2 * j + 1], cb);
#pragma unroll
            for (int mg = 0; mg < MG; ++mg)
                mma_16816(acc[mg][j], A[mg], b0, b1);
        }
    }
}

template <int K, int MG>
__global__ void __launch_bounds__(kGemvThreads, MG == 1 ? 2 : 1) gemv_kernel(const GemvParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    volatile int *flag = reinterpret_cast<volatile int *>(smem);
    unsigned char *zero_rec = smem + 16;  // 16 zero bytes
    unsigned char *recs = smem + 32;      // x' records, later the reduction buffer

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nb = blockIdx.x, split = blockIdx.y;
    const int m = p.m, n = p.n;
    const int tn_count = n >> 4;
    const int row_begin = split * p.rows_per_split;
    int row_end = row_begin + p.rows_per_split;
    if (row_end > (p.k >> 4))
        row_end = p.k >> 4;
    const int rows = row_end - row_begin;

    // this warp's first two tile rows: requested before anything else
    const uint32_t *tiles =
        reinterpret_cast<const uint32_t *>(p.trellis) + ((int64_t)nb * 8 + g) * 8 * K;
    const int64_t row_stride = (int64_t)tn_count * 8 * K;  // u32 per tile row of the matrix
    RowBuf<K> buf0, buf1, buf2;
    int tr = warp;
    if (tr < rows)
        load_tile_row<K>(tiles + (int64_t)(row_begin + tr) * row_stride, t, buf0);
    if (tr + kGemvWarps < rows)
        load_tile_row<K>(tiles + (int64_t)(row_begin + tr + kGemvWarps) * row_stride, t, buf1);
    const Codebook cb = p.cb;

    // everything below reads x or touches the workspace/output: wait for the
    // preceding kernel (a no-op unless launched with programmatic overlap)
    grid_dep_wait();

    // activation records for this split's k range.  A job is (quad, 128-block):
    // the warp rotates the quad's one or two batches and writes whole records
    // (both parities), so no zero-fill pass is needed.
    const int slots = rec_slots(m);
    {
        const int k0 = row_begin * 16;
        const int nblk = rows / 8;
        const int q0 = rec_quads(m, 0), nq = q0 + rec_quads(m, 1);
        const float s128 = 0.08838834764831845f;
        for (int job = warp; job < nq * nblk; job += kGemvWarps) {
            const int qd = job / nblk, blk = job - qd * nblk;
            const int mg = qd >= q0 ? 1 : 0, ba = qd - mg * q0;
            const int b0 = 8 * mg + ba, b1 = b0 + 4;
            const int c = k0 + blk * 128 + lane * 4;
            const uint2 sr = *reinterpret_cast<const uint2 *>(p.suh + c);
            const uint2 r0 = *reinterpret_cast<const uint2 *>(p.x + (int64_t)b0 * p.k + c);
            uint2 r1 = make_uint2(0u, 0u);
            if (b1 < m)
                r1 = *reinterpret_cast<const uint2 *>(p.x + (int64_t)b1 * p.k + c);
            const __half2 *sv = reinterpret_cast<const __half2 *>(&sr);
            const __half2 *x0 = reinterpret_cast<const __half2 *>(&r0);
            const __half2 *x1 = reinterpret_cast<const __half2 *>(&r1);
            float v0[4] = {__low2float(x0[0]) * __low2float(sv[0]), __high2float(x0[0]) * __high2float(sv[0]),
                           __low2float(x0[1]) * __low2float(sv[1]), __high2float(x0[1]) * __high2float(sv[1])};
            float v1[4] = {__low2float(x1[0]) * __low2float(sv[0]), __high2float(x1[0]) * __high2float(sv[0]),
                           __low2float(x1[1]) * __low2float(sv[1]), __high2float(x1[1]) * __high2float(sv[1])};
            warp_fwht128(v0);
            if (b1 < m)
                warp_fwht128(v1);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t h0 = (uint32_t)__half_as_ushort(__float2half_rn(v0[e] * s128));
                const uint32_t h1 = b1 < m ? (uint32_t)__half_as_ushort(__float2half_rn(v1[e] * s128)) : 0u;
                const uint32_t d0 = h0 | (h0 << 16), d1 = h1 | (h1 << 16);
                uint4 *rec = reinterpret_cast<uint4 *>(recs + ((blk * 128 + lane * 4 + e) * slots + 2 * qd) * 16);
                rec[0] = make_uint4(d0, d1, 0u, 0u);  // even A rows
                rec[1] = make_uint4(0u, 0u, d0, d1);  // odd A rows
            }
        }
        if (threadIdx.x == 0)
            *reinterpret_cast<uint4 *>(zero_rec) = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();

    RecPtr rp[MG];
#pragma unroll
    for (int mg = 0; mg < MG; ++mg) {
        const int ba = g >> 1;
        const int qbase = mg * rec_quads(m, 0);
        if (ba < rec_quads(m, mg)) {
            rp[mg].base = recs + (2 * (qbase + ba) + (g & 1)) * 16;
            rp[mg].stride = slots * 16;
        } else {
            rp[mg].base = zero_rec;
            rp[mg].stride = 0;
        }
    }

    float acc[MG][8][4];
#pragma unroll
    for (int a = 0; a < MG; ++a)
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[a][j][e] = 0.f;

    // three buffers in rotation: two tile rows' loads are in flight during the math
    constexpr int W = kGemvWarps;
    for (; tr < rows;) {
        if (tr + 2 * W < rows)
            load_tile_row<K>(tiles + (int64_t)(row_begin + tr + 2 * W) * row_stride, t, buf2);
        mac_tile_row<K, MG>(buf0, tr * 16, rp, t, cb, acc);
        tr += W;
        if (tr >= rows)
            break;
        if (tr + 2 * W < rows)
            load_tile_row<K>(tiles + (int64_t)(row_begin + tr + 2 * W) * row_stride, t, buf0);
        mac_tile_row<K, MG>(buf1, tr * 16, rp, t, cb, acc);
        tr += W;
        if (tr >= rows)
            break;
        if (tr + 2 * W < rows)
            load_tile_row<K>(tiles + (int64_t)(row_begin + tr + 2 * W) * row_stride, t, buf1);
        mac_tile_row<K, MG>(buf2, tr * 16, rp, t, cb, acc);
        tr += W;
    }

    // the weight stream of this CTA is done: let the next kernel start launching
    grid_dep_launch();

    // ------------------------------------------------- reduce across warps ---
    __syncthreads();  // records no longer needed: reuse as [warp][m][128] f32
    float *red = reinterpret_cast<float *>(recs);
    // accumulator (mg, j, e): A row i = g (+8 for e >= 2) -> batch 8mg + i/2,
    // column parity i&1; n-slot 2t (+1 for odd e) -> tile of the block;
    // column = 16 * slot + 2j + parity.
#pragma unroll
    for (int mg = 0; mg < MG; ++mg)
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = g + ((e >> 1) << 3);
                const int b = 8 * mg + (i >> 1);
                const int col = 16 * (2 * t + (e & 1)) + 2 * j + (i & 1);
                if (b < m)
                    red[(warp * m + b) * 128 + col] = acc[mg][j][e];
            }
    __syncthreads();
    const int tid = threadIdx.x;
    for (int e = tid; e < m * 128; e += kGemvThreads) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kGemvWarps; ++w)
            sum += red[w * m * 128 + e];
        red[e] = sum;
    }
    __syncthreads();

    if (p.splits > 1) {
        for (int e = tid; e < m * 128; e += kGemvThreads) {
            const int b = e >> 7, c = e & 127;
            p.partials[((int64_t)split * m + b) * n + nb * 128 + c] = red[e];
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            const uint32_t ticket = atomicAdd(&p.counters[nb], 1u);
            *flag = (ticket == (uint32_t)(p.splits - 1)) ? 1 : 0;
        }
        __syncthreads();
        if (*flag != 1)
            return;
        __threadfence();
        // sum the partials in split order; eight independent loads in flight
        // per thread, and for m = 1 two threads per element (even / odd
        // splits) combined afterwards, so the L2 latency is paid a few times
        // rather than once per split
        const int E = m * 128;
        const int per_elem = E < kGemvThreads ? 2 : 1;
        float *part2 = red + E;  // second-half sums when per_elem == 2
        for (int u = tid; u < E * per_elem; u += kGemvThreads) {
            const int e = u % E, h = u / E;
            const int b = e >> 7, c = e & 127;
            const float *src = p.partials + (int64_t)b * n + nb * 128 + c;
            const int64_t sstride = (int64_t)m * n;
            float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            int sp = h;
            for (; sp + 7 * per_elem < p.splits; sp += 8 * per_elem) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    acc8[i] += __ldcg(src + (int64_t)(sp + i * per_elem) * sstride);
            }
            float tail = 0.f;
            for (; sp < p.splits; sp += per_elem)
                tail += __ldcg(src + (int64_t)sp * sstride);
            const float sum =
                (((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) + ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]))) + tail;
            if (h == 0)
                red[e] = sum;
            else
                part2[e] = sum;
        }
        __syncthreads();
        if (per_elem == 2)
            for (int e = tid; e < E; e += kGemvThreads)
                red[e] += part2[e];
        if (tid == 0)
            p.counters[nb] = 0u;
        __syncthreads();
    }

    // ------------------------------------ output rotation, scales, fp16 y ---
    for (int b = warp; b < m; b += kGemvWarps) {
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

int num_sms()
{
    if (g_num_sms <= 0) {
        int dev = 0;
        int v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
            cudaGetLastError();
            v = 148;
        }
        g_num_sms = v;
    }
    return g_num_sms;
}

// Split count: each split covers whole 128-channel blocks and its x' records
// fit 96 KB of shared memory (192 KB for m > 8, one CTA per SM); among the candidates take the smallest
// estimated time = waves x (blocks per split + 1), a wave being the resident
// CTAs (2 per SM for m <= 8, 1 above) and the +1 the per-CTA fixed cost; ties go to fewer splits.
static GemvPlan gemv_plan(int64_t m, int64_t k, int64_t n, int sms)
{
    GemvPlan pl;
    const int64_t blocks_k = k / 128;
    const int64_t nblocks = n / 128;
    const int64_t slots = (m <= 8 ? 2 : 1) * (int64_t)sms;  // resident CTAs per SM
    const int64_t rec_budget = (m <= 8 ? 96 : 192) * 1024;  // x' records per CTA
    int64_t max_per = rec_budget / (128 * rec_slots((int)m) * 16);
    if (max_per < 1)
        max_per = 1;
    int64_t best_per = blocks_k < max_per ? blocks_k : max_per, best_cost = -1;
    for (int64_t s = 1; s <= blocks_k && s <= 64; ++s) {
        const int64_t per = (blocks_k + s - 1) / s;
        if (per > max_per)
            continue;
        const int64_t real_s = (blocks_k + per - 1) / per;
        const int64_t units = nblocks * real_s;
        const int64_t waves = (units + slots - 1) / slots;
        const int64_t cost = waves * (per + 1) * 64 + real_s;
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best_per = per;
        }
    }
    pl.splits = (int)((blocks_k + best_per - 1) / best_per);
    pl.rows_per_split = (int)(best_per * 8);
    pl.smem = gemv_smem_bytes((int)m, pl.rows_per_split);
    return pl;
}

size_t gemv_workspace_bytes(int64_t m, int64_t k, int64_t n, int sms)
{
    const GemvPlan pl = gemv_plan(m, k, n, sms);
    size_t bytes = 256;                                  // status word + padding
    bytes += (size_t)((n / 128) * 4 + 255) / 256 * 256;  // counters
    if (pl.splits > 1)
        bytes += (size_t)pl.splits * (size_t)m * (size_t)n * 4;
    return bytes;
}

template <int K, int MG>
static exl3_status launch_gemv_t(const GemvParams &p, int smem, cudaStream_t stream)
{
    auto kern = gemv_kernel<K, MG>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return EXL3_ERR_CUDA;
    dim3 grid((unsigned)(p.n / 128), (unsigned)p.splits);
    if (launch_kernel(kern, grid, dim3(kGemvThreads), (size_t)smem, stream, p) != cudaSuccess)
        return EXL3_ERR_CUDA;
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
    const GemvPlan pl = gemv_plan(m, k, n, sms);
    if (!workspace || !aligned16(workspace) || workspace_bytes < gemv_workspace_bytes(m, k, n, sms))
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
    p.counters = (uint32_t *)(ws + 256);
    p.partials = (float *)(ws + 256 + (size_t)((n / 128) * 4 + 255) / 256 * 256);
    p.cb = codebook_constants();
    if (m <= 8)
        return launch_gemv_k<1>(p, K, pl.smem, stream);
    return launch_gemv_k<2>(p, K, pl.smem, stream);
}

}  // namespace exl3

extern "C" size_t exl3_gemv_workspace_size(int64_t m, int64_t k, int64_t n, int K)
{
    if (m < 1 || m > 16 || k < 128 || n < 128 || (k % 128) || (n % 128) || K < 1 || K > 8)
        return 0;
    return exl3::gemv_workspace_bytes(m, k, n, exl3::num_sms());
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

// ------------------------------------------------ no-allocation variant ---
//
// exl3_gemv_noalloc runs the GEMV above with its scratch (split-k partials
// and arrival counters) in a fixed array compiled into the library, for
// callers that must not allocate device memory themselves.  The array is a
// file-scope __device__ symbol: every GPU that loads the library holds its
// kNoAllocScratchBytes until the process exits.  In host code the symbol's
// name is only a host-side stand-in, so the device address is looked up once
// per device with cudaGetSymbolAddress (with that device current) and cached.

#include <mutex>

namespace exl3 {

constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
static void *g_noalloc_ptr[kMaxDevices];
static std::mutex g_noalloc_mutex;

// Device address of this device's scratch array (set up on first use).
static exl3_status noalloc_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return EXL3_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices)
        return EXL3_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return EXL3_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return EXL3_OK;
}

}  // namespace exl3

extern "C" size_t exl3_gemv_noalloc_max_scratch(void)
{
    return exl3::kNoAllocScratchBytes;
}

extern "C" exl3_status exl3_gemv_noalloc(const void *x, const uint16_t *trellis, const void *suh,
                                         const void *svh, void *y, int64_t m, int64_t k, int64_t n,
                                         int K, void *stream)
{
    using namespace exl3;
    const exl3_status st = check_linear_args(x, trellis, suh, svh, y, m, k, n, K);
    if (st != EXL3_OK)
        return st;
    if (m > 16)
        return EXL3_ERR_UNSUPPORTED;
    const size_t need = gemv_workspace_bytes(m, k, n, num_sms());
    if (need > kNoAllocScratchBytes)
        return EXL3_ERR_WORKSPACE;  // this shape needs more scratch than the built-in array
    void *scratch = nullptr;
    const exl3_status sst = noalloc_scratch(&scratch);
    if (sst != EXL3_OK)
        return sst;
    // the array keeps whatever the last call left: the arrival counters must
    // start at zero (the kernel re-arms them, but a call that never finished
    // could have left them set), so clear them on the caller's stream
    const size_t counter_bytes = 256 + (size_t)((n / 128) * 4 + 255) / 256 * 256;
    if (cudaMemsetAsync(scratch, 0, counter_bytes, (cudaStream_t)stream) != cudaSuccess)
        return EXL3_ERR_CUDA;
    return run_gemv(x, trellis, suh, svh, y, m, k, n, K, scratch, kNoAllocScratchBytes,
                    (cudaStream_t)stream);
}
