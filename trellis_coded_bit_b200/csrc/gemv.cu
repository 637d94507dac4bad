// gemv.cu -- exl3_gemv: y = svh .* H(H(x .* suh) . W_hat) for 1 <= m <= 16,
// with W_hat decoded on the fly from the trellis (EXL3 GEMM kernel article,
// section 小批量GEMV: in decoding the bottleneck moves from compute to memory
// bandwidth, so a dedicated GEMV path streams the quantised weights once).
//
// B200 design (the pages' consumer-GPU GEMV is prior art, not copied):
//   * Two launches.  A rotation kernel computes x' = H(x .* suh)/sqrt(128)
//     (fp32 butterflies, fp16 result) and writes it into the workspace as
//     tensor-core A-fragment records (see below).  The main kernel then has
//     no prologue: every warp starts streaming weights at once.
//   * The main kernel is persistent, "stream-K" balanced: the work units are
//     (128-column block, tile row of 16 input channels) pairs in column-block
//     order, and CTA c owns the contiguous range [cU/G, (c+1)U/G) -- every
//     CTA gets the same amount of work, whatever the shape.  A range is cut
//     into segments at column-block boundaries; inside a segment the 8 warps
//     take tile rows w, w+8, ...; at a segment end the warps' partial sums
//     meet in shared memory (one barrier) and either finish the column block
//     (output rotation, svh, fp16 y) or go to the workspace, where the last
//     segment to arrive on the block's counter (atomic ticket, no spinning)
//     sums all segments in segment order (deterministic) and finishes it.
//   * Lane (g, t) owns tile g of the column block and, in each of 4 row
//     groups q, the whole tile row rho(q, t) (16 weights): rows are ordered
//     so that all lanes of a group share the row parity, which makes every
//     bit-window operation a compile-time byte permute (see row_states).
//     Loads go straight from HBM into registers in this fragment order
//     (read-only path, 8/16-byte vectors where aligned), one unit ahead of
//     the math and across segment boundaries.
//   * The MAC runs on the tensor cores (mma.sync m16n8k16, fp32 accumulate):
//     a codebook word's two fp16 halves form a pair of k slots in B and the
//     activation is duplicated over that pair in A, so the tensor core forms
//     x*(hi + lo) exactly in fp32 (the fp16 rounding of hi + lo that defines
//     W_hat is skipped: at most half an fp16 ulp per weight, far inside the
//     output tolerance).  Weights 2j, 2j+1 of a lane's row feed MMA j (k
//     pairs t and t+4); A rows are (batch, column parity) with zeros
//     elsewhere, so parities never mix.  Batch rows 0..7 per group, two
//     groups for m > 8 (one decode feeds both).
//   * With EXL3_LAUNCH_PDL the main kernel requests its first weights before
//     it waits for the rotation kernel (griddepcontrol).
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = 32 * kGemvWarps;

// Activation records, in MMA A-fragment register order.  For batch group mg
// (batches 8mg..8mg+7), quad ba (batches 8mg+ba and 8mg+ba+4) and A-row
// parity p, a 16-byte record holds the lane's {a0, a1, a2, a3}:
//   p = 0: {x(8mg+ba), x(8mg+ba+4), 0, 0}     p = 1: {0, 0, x(8mg+ba), x(8mg+ba+4)}
// with x the rotated activation duplicated in both fp16 halves (a batch
// >= m is zero).  Each input channel has rec_slots_for(MG) = 8 MG slots, slot
// 8mg + 2ba + p, record (kk, slot) at recs + (kk * 8 MG + slot) * 16.  Only
// quads holding a batch < m are written: a record of an absent quad feeds only
// A rows of absent batches, whose accumulator rows are never stored, so
// whatever it holds is harmless.
__host__ __device__ inline int rec_quads(int m, int mg)
{
    const int q = m - 8 * mg;
    return q <= 0 ? 0 : (q < 4 ? q : 4);
}

__host__ __device__ constexpr int rec_slots_for(int MG)
{
    return 8 * MG;
}

__host__ __device__ inline int gemv_mg(int64_t m)
{
    return m > 8 ? 2 : 1;
}

// Up to kGemvMaxLayers layers (same K and m) share one launch; their work
// units and column blocks are numbered consecutively across the layers.
constexpr int kGemvMaxLayers = 16;

// ------------------------------------------------------ rotation kernel ---

struct GemvRotLayer {
    const __half *x;
    const __half *suh;
    unsigned char *recs;
    int k;
    int64_t job_begin;  // first job of this layer
};

constexpr int kGemvRotMaxLayers = 32;  // one rotation launch may serve several main launches

struct GemvRotParams {
    GemvRotLayer L[kGemvRotMaxLayers];
    int count, m;
    int64_t jobs;
};

// One warp per (layer, quad, 128-channel block): rotates the quad's one or
// two batches and writes both parity records of each channel.
__global__ void __launch_bounds__(256) gemv_rotate_kernel(const GemvRotParams rp)
{
    grid_dep_wait();    // x may come from the preceding kernel
    grid_dep_launch();  // the main kernel may start streaming weights meanwhile
    const int lane = threadIdx.x & 31;
    const int m = rp.m;
    const int slots = rec_slots_for(gemv_mg(m));
    const int q0 = rec_quads(m, 0);
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const float s128 = 0.08838834764831845f;
    int l = 0;
    for (int64_t job = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); job < rp.jobs; job += warps) {
        while (l + 1 < rp.count && job >= rp.L[l + 1].job_begin)
            ++l;
        const GemvRotLayer &L = rp.L[l];
        const int k = L.k, nblk = k / 128;
        const int64_t lj = job - L.job_begin;
        const int qd = (int)(lj / nblk), blk = (int)(lj - (int64_t)qd * nblk);
        const int mg = qd >= q0 ? 1 : 0, ba = qd - mg * q0;
        const int b0 = 8 * mg + ba, b1 = b0 + 4;
        const int c = blk * 128 + lane * 4;
        const uint2 sr = *reinterpret_cast<const uint2 *>(L.suh + c);
        const uint2 r0 = *reinterpret_cast<const uint2 *>(L.x + (int64_t)b0 * k + c);
        uint2 r1 = make_uint2(0u, 0u);
        if (b1 < m)
            r1 = *reinterpret_cast<const uint2 *>(L.x + (int64_t)b1 * k + c);
        const __half2 *sv = reinterpret_cast<const __half2 *>(&sr);
        const __half2 *x0 = reinterpret_cast<const __half2 *>(&r0);
        const __half2 *x1 = reinterpret_cast<const __half2 *>(&r1);
        float v0[4] = {__low2float(x0[0]) * __low2float(sv[0]), __high2float(x0[0]) * __high2float(sv[0]),
                       __low2float(x0[1]) * __low2float(sv[1]), __high2float(x0[1]) * __high2float(sv[1])};
        float v1[4] = {__low2float(x1[0]) * __low2float(sv[0]), __high2float(x1[0]) * __high2float(sv[0]),
                       __low2float(x1[1]) * __low2float(sv[1]), __high2float(x1[1]) * __high2float(sv[1])};
        warp_fwht128(v0);
        warp_fwht128(v1);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t h0 = (uint32_t)__half_as_ushort(__float2half_rn(v0[e] * s128));
            const uint32_t h1 = b1 < m ? (uint32_t)__half_as_ushort(__float2half_rn(v1[e] * s128)) : 0u;
            const uint32_t d0 = h0 | (h0 << 16), d1 = h1 | (h1 << 16);
            uint4 *rec = reinterpret_cast<uint4 *>(L.recs + ((int64_t)(c + e) * slots + 8 * mg + 2 * ba) * 16);
            rec[0] = make_uint4(d0, d1, 0u, 0u);  // even A rows
            rec[1] = make_uint4(0u, 0u, d0, d1);  // odd A rows
        }
    }
}

// ---------------------------------------------------------- main kernel ---

// One layer of a launch.  Global unit u of the layer is unit_begin + cb * TR
// + tr (column block cb, tile row tr); its column blocks are the launch's
// column blocks cb_begin .. cb_begin + n/128 - 1.
struct GemvLayer {
    const unsigned char *trellis;
    const __half *svh;
    __half *y;
    const unsigned char *recs;
    float *partials;     // [n/128][max_seg][m][128]
    uint32_t *counters;  // [n/128]
    int64_t unit_begin;
    int n, tr_count, cb_begin, max_seg;
};

struct GemvParams {
    GemvLayer L[kGemvMaxLayers];
    int count, m, ctas;
    int64_t units;  // all layers' units
    Codebook cb;
};

// Per-warp shared-memory ring: each stage holds one unit -- the 8 tiles of a
// tile row (each padded to 32K + 16 bytes, which spreads the lanes' row reads
// over the banks) and that tile row's 16 x 8MG activation records.  The
// layout is a compile-time function of K and MG, so every shared-memory
// access of the inner loop is a lane pointer plus an immediate offset.
template <int K, int MG>
struct GemvStage {
    static constexpr int kTileStride = 32 * K + 16;
    static constexpr int kTileBytes = 8 * kTileStride;
    static constexpr int kSlots = rec_slots_for(MG);
    static constexpr int kRecRowBytes = 16 * kSlots * 16;  // records of one tile row
    static constexpr int kBytes = (kTileBytes + kRecRowBytes + 127) & ~127;
};

__host__ __device__ inline int gemv_stage_bytes(int K, int MG)
{
    const int tiles = 8 * (32 * K + 16), recs = 16 * rec_slots_for(MG) * 16;
    return (tiles + recs + 127) & ~127;
}

constexpr int kGemvDepth = 3;  // units in flight per warp (one consumed, two loading)

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr(smem_dst)), "l"(gsrc)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Lane (g, t) owns tile g of the unit and, in row group q, the tile row
// rho(q, t) = 2t + c(q) with c(q) = 8(q & 1) + (q >> 1): groups 0, 1 take
// the even rows, groups 2, 3 the odd ones, so a group's lanes share the row
// parity (compile-time bit windows).  Row rho starts at word rho K; its
// prefix word (rho K - 1) wraps to the tile's last word for rho = 0.
template <int K>
__host__ __device__ constexpr int gemv_row_imm(int q)
{
    return 4 * (((8 * (q & 1) + (q >> 1)) * K - 1) >> 1);  // floor, -4 for c(q) = 0
}

// The lane's base pointers into its ring (stage 0): row words, the q = 0
// prefix word (the wrap lane differs), activation records.
struct GemvLanePtrs {
    const unsigned char *row, *pre0, *rec;
};

// Loads the words of tile row rho(q, t) of stage S: raw[0] the prefix word,
// then the row's words, as wide as the row's alignment allows.
template <int K, int MG, int S, int q, int N>
__device__ __forceinline__ void load_row_q(const GemvLanePtrs &lp, uint32_t (&raw)[N])
{
    using St = GemvStage<K, MG>;
    constexpr int PAR = q >> 1;
    constexpr int P = RowSpan<K, PAR>::P;
    constexpr int N32 = RowSpan<K, PAR>::N32;
    constexpr int off = S * St::kBytes + gemv_row_imm<K>(q);
    const unsigned char *row = lp.row + off;
    raw[0] = (q == 0) ? *reinterpret_cast<const uint32_t *>(lp.pre0 + S * St::kBytes)
                      : *reinterpret_cast<const uint32_t *>(row - 4);
    if constexpr (K == 4 && P == 1) {
        const uint2 v = *reinterpret_cast<const uint2 *>(row);
        raw[1] = v.x;
        raw[2] = v.y;
    } else if constexpr (K == 8 && P == 1) {
        const uint4 v = *reinterpret_cast<const uint4 *>(row);
        raw[1] = v.x;
        raw[2] = v.y;
        raw[3] = v.z;
        raw[4] = v.w;
    } else {
#pragma unroll
        for (int i = 1; i < N32; ++i)
            raw[i] = *reinterpret_cast<const uint32_t *>(row + 4 * (i - 1));
    }
}

template <int K, int MG, int S, int q>
__device__ __forceinline__ void mac_row(const GemvLanePtrs &lp, const Codebook &cb, float (&acc)[MG][8][4])
{
    using St = GemvStage<K, MG>;
    constexpr int PAR = q >> 1;
    constexpr int cq = 8 * (q & 1) + (q >> 1);
    uint32_t A[MG][4];
#pragma unroll
    for (int mg = 0; mg < MG; ++mg) {
        const uint4 r = *reinterpret_cast<const uint4 *>(lp.rec + S * St::kBytes + cq * St::kSlots * 16 + mg * 128);
        A[mg][0] = r.x;
        A[mg][1] = r.y;
        A[mg][2] = r.z;
        A[mg][3] = r.w;
    }
    uint32_t raw[RowSpan<K, PAR>::N32];
    load_row_q<K, MG, S, q>(lp, raw);
    uint32_t st[16];
    row_states<K, RowSpan<K, PAR>::P>(raw, st);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t b0 = codebook_word(st[2 * j], cb);
        const uint32_t b1 = codebook_word(st[2 * j + 1], cb);
#pragma unroll
        for (int mg = 0; mg < MG; ++mg)
            mma_16816(acc[mg][j], A[mg], b0, b1);
    }
}

template <int K, int MG, int S>
__device__ __forceinline__ void mac_stage(const GemvLanePtrs &lp, const Codebook &cb, float (&acc)[MG][8][4])
{
    mac_row<K, MG, S, 0>(lp, cb, acc);
    mac_row<K, MG, S, 1>(lp, cb, acc);
    mac_row<K, MG, S, 2>(lp, cb, acc);
    mac_row<K, MG, S, 3>(lp, cb, acc);
}

// CTA owning unit u: the largest c with floor(c U / G) <= u.
__device__ __forceinline__ int owner_cta(int64_t u, int64_t U, int G)
{
    return (int)(((u + 1) * G - 1) / U);
}

// Output rotation, svh and fp16 store of one column block's m x 128 y'.
__device__ __forceinline__ void finish_block(const GemvLayer &L, int m, const float *red, int cb, int warp,
                                             int lane)
{
    for (int b = warp; b < m; b += kGemvWarps) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            v[e] = red[b * 128 + lane * 4 + e];
        warp_fwht128(v);
        const int c = cb * 128 + lane * 4;
        const uint2 sr = *reinterpret_cast<const uint2 *>(L.svh + c);
        const __half2 *sv = reinterpret_cast<const __half2 *>(&sr);
        const float s = 0.08838834764831845f;
        __half2 o0 = __floats2half2_rn(v[0] * s * __low2float(sv[0]), v[1] * s * __high2float(sv[0]));
        __half2 o1 = __floats2half2_rn(v[2] * s * __low2float(sv[1]), v[3] * s * __high2float(sv[1]));
        uint2 out;
        out.x = *reinterpret_cast<uint32_t *>(&o0);
        out.y = *reinterpret_cast<uint32_t *>(&o1);
        *reinterpret_cast<uint2 *>(L.y + (int64_t)b * L.n + c) = out;
    }
}

// Position of global unit u: layer l (scanning on from l; always 0 for a
// single-layer launch), column block cb within it, tile row tr.
template <bool MULTI>
__device__ __forceinline__ void gemv_locate(const GemvParams &p, int64_t u, int &l, int &cb, int &tr)
{
    while (MULTI && l + 1 < p.count && u >= p.L[l + 1].unit_begin)
        ++l;
    const int64_t lu = u - p.L[l].unit_begin;
    const int TR = p.L[l].tr_count;
    cb = (int)(lu / TR);
    tr = (int)(lu - (int64_t)cb * TR);
}

template <int K, int MG, bool MULTI>
__global__ void __launch_bounds__(kGemvThreads, MG == 1 ? 2 : 1) gemv_kernel(const GemvParams p)
{
    using St = GemvStage<K, MG>;
    constexpr int SB = St::kBytes;
    constexpr int kTrChunks = (16 * K + 31) / 32;  // 16-byte trellis chunks per lane per unit
    constexpr int kRecChunks = St::kRecRowBytes / 16 / 32;
    extern __shared__ __align__(128) unsigned char smem[];
    volatile int *flag = reinterpret_cast<volatile int *>(smem);
    const int m = p.m;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *ring = smem + 128 + warp * kGemvDepth * SB;
    float *red = reinterpret_cast<float *>(smem + 128 + kGemvWarps * kGemvDepth * SB);

    const int g = lane >> 2, t = lane & 3;
    const int64_t U = p.units;
    const int G = p.ctas;
    const int64_t u0 = (int64_t)blockIdx.x * U / G, u1 = (int64_t)(blockIdx.x + 1) * U / G;

    // lane-constant pointers and copy offsets
    GemvLanePtrs lp;
    lp.row = ring + g * St::kTileStride + 4 * (t * K + 1);
    lp.pre0 = t == 0 ? ring + g * St::kTileStride + 4 * (8 * K - 1)  // row 0: the tile's last word
                     : lp.row + gemv_row_imm<K>(0) - 4;
    lp.rec = ring + St::kTileBytes + (2 * t * St::kSlots + g) * 16;
    unsigned char *tdst[kTrChunks];
#pragma unroll
    for (int r = 0; r < kTrChunks; ++r) {
        const int i = lane + 32 * r;  // chunk i: tile i / 2K, 16-byte piece i % 2K
        tdst[r] = ring + (i / (2 * K)) * St::kTileStride + (i % (2 * K)) * 16;
    }
    const bool last_chunk = (16 * K) % 32 == 0 || lane + 32 * (kTrChunks - 1) < 16 * K;

    // this warp's units: u0 + warp, u0 + warp + 8, ... (< u1), as (layer,
    // column block, tile row) advanced incrementally; the issue iterator runs
    // kGemvDepth units ahead of consumption
    int64_t iu = u0 + warp;
    int il = 0, icb = 0, itr = 0;
    gemv_locate<MULTI>(p, iu < u1 ? iu : u0, il, icb, itr);
    int64_t tile_row_bytes = 0;
    int itr_lim = 0, incb = 0;  // the issue layer's tile rows and column blocks
    const unsigned char *isrc = nullptr, *irsrc = nullptr;
    auto point = [&]() {
        const GemvLayer &L = p.L[il];
        itr_lim = L.tr_count;
        incb = L.n >> 7;
        tile_row_bytes = (int64_t)(L.n >> 4) * 32 * K;  // one tile row of the layer's matrix
        isrc = L.trellis + itr * tile_row_bytes + (int64_t)icb * 8 * 32 * K + lane * 16;
        irsrc = L.recs + (int64_t)itr * St::kRecRowBytes + lane * 16;
    };
    point();
    int64_t cu = iu;
    int cl = il, ccb = icb, ctr = itr;  // consumed unit: layer, column block, tile row
    int cg = p.L[il].cb_begin + icb;    // consumed unit's global column block
    int ctr_lim = itr_lim, cncb = incb;  // the consumed unit's layer: tile rows, column blocks

    auto issue = [&](int stage) {
        if (iu < u1) {
            const int so = stage * SB;
#pragma unroll
            for (int r = 0; r < kTrChunks; ++r)
                if (r < kTrChunks - 1 || last_chunk)
                    cp_async16(tdst[r] + so, isrc + 512 * r);
#pragma unroll
            for (int r = 0; r < kRecChunks; ++r)
                cp_async16(ring + so + St::kTileBytes + (lane + 32 * r) * 16, irsrc + 512 * r);
            iu += kGemvWarps;
            itr += kGemvWarps;
            isrc += kGemvWarps * tile_row_bytes;
            irsrc += kGemvWarps * St::kRecRowBytes;
            if (itr >= itr_lim) {  // next column block, perhaps of the next layer (units advance by 8 <= TR)
                itr -= itr_lim;
                if (++icb == incb) {
                    icb = 0;
                    if (MULTI)
                        ++il;
                }
                if (iu < u1)
                    point();
            }
        }
        cp_async_commit();
    };

    // records come from the rotation kernel: wait for it (no-op without PDL)
    grid_dep_wait();
#pragma unroll
    for (int d = 0; d < kGemvDepth; ++d)
        issue(d);
    __syncwarp();

    const Codebook cb = p.cb;
    float acc[MG][8][4];
#pragma unroll
    for (int a = 0; a < MG; ++a)
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[a][j][e] = 0.f;

    // the CTA's range as global column blocks [g0, g1]
    int l0 = 0, c0 = 0, r0 = 0, l1 = 0, c1 = 0, r1 = 0;
    gemv_locate<MULTI>(p, u0, l0, c0, r0);
    l1 = l0;
    gemv_locate<MULTI>(p, u1 - 1, l1, c1, r1);
    const int g0 = p.L[l0].cb_begin + c0, g1 = p.L[l1].cb_begin + c1;
    int sl = l0;  // layer of the current segment's column block
    int st = 0;
    for (int gk = g0; gk <= g1; ++gk) {
        while (MULTI && sl + 1 < p.count && gk >= p.L[sl + 1].cb_begin)
            ++sl;
        const GemvLayer &SL = p.L[sl];
        const int TR = SL.tr_count;
        const int cbk = gk - SL.cb_begin;  // column block within the layer
        while (cu < u1 && cg == gk) {
            cp_async_wait<kGemvDepth - 1>();
            __syncwarp();
            if (st == 0)
                mac_stage<K, MG, 0>(lp, cb, acc);
            else if (st == 1)
                mac_stage<K, MG, 1>(lp, cb, acc);
            else
                mac_stage<K, MG, 2>(lp, cb, acc);
            __syncwarp();  // every lane is done with the stage before it is refilled
            issue(st);
            st = st + 1 == kGemvDepth ? 0 : st + 1;
            cu += kGemvWarps;
            // the consumed unit's column block: units advance by 8 <= TR tile rows
            ctr += kGemvWarps;
            if (ctr >= ctr_lim) {
                ctr -= ctr_lim;
                if (++ccb == cncb) {
                    ccb = 0;
                    if (MULTI)
                        ++cl;
                    if (MULTI && cu < u1) {
                        ctr_lim = p.L[cl].tr_count;
                        cncb = p.L[cl].n >> 7;
                    }
                }
                cg = cu < u1 ? p.L[cl].cb_begin + ccb : cg + 1;
            }
        }
        const int64_t blk_begin = SL.unit_begin + (int64_t)cbk * TR, blk_end = blk_begin + TR;
        const int64_t seg_begin = blk_begin > u0 ? blk_begin : u0;
        const int64_t seg_end = blk_end < u1 ? blk_end : u1;

    // ------------------------------------------- segment end: reduce ---
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
                    acc[mg][j][e] = 0.f;
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
        const bool whole = seg_begin == blk_begin && seg_end == blk_end;
        if (whole) {
            finish_block(SL, m, red, cbk, warp, lane);
        } else {
            const int c_first = owner_cta(blk_begin, U, G);
            const int c_last = owner_cta(blk_end - 1, U, G);
            const int nseg = c_last - c_first + 1;
            const int j = (int)blockIdx.x - c_first;
            float *part = SL.partials + ((int64_t)cbk * SL.max_seg) * m * 128;
            for (int e = tid; e < m * 128; e += kGemvThreads)
                part[(int64_t)j * m * 128 + e] = red[e];
            __threadfence();
            __syncthreads();
            if (tid == 0) {
                const uint32_t ticket = atomicAdd(&SL.counters[cbk], 1u);
                *flag = (ticket == (uint32_t)(nseg - 1)) ? 1 : 0;
            }
            __syncthreads();
            if (*flag == 1) {
                __threadfence();
                // segment order, eight independent loads in flight per thread
                for (int e = tid; e < m * 128; e += kGemvThreads) {
                    float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    int s2 = 0;
                    for (; s2 + 8 <= nseg; s2 += 8)
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            a8[i] += __ldcg(part + (int64_t)(s2 + i) * m * 128 + e);
                    float tail = 0.f;
                    for (; s2 < nseg; ++s2)
                        tail += __ldcg(part + (int64_t)s2 * m * 128 + e);
                    red[e] = (((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]))) + tail;
                }
                if (tid == 0)
                    SL.counters[cbk] = 0u;
                __syncthreads();
                finish_block(SL, m, red, cbk, warp, lane);
            }
        }
        __syncthreads();  // red is reused by the next segment
    }
    cp_async_wait<0>();  // nothing may still be landing in shared memory at exit
}

// ------------------------------------------------------------- dispatch ---

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

static int64_t owner_cta_host(int64_t u, int64_t U, int64_t G)
{
    return ((u + 1) * G - 1) / U;
}

// Plan of one launch over `count` layers (same K, same m): grid, shared
// memory, and the workspace layout -- [0, 256) status word; the layers'
// arrival counters (one per column block, consecutive); then per layer its
// activation records (k * 8 MG * 16) and split partials [n/128][max_seg][m][128].
struct GemvGroupPlan {
    int ctas, smem;
    int64_t units;
    int64_t unit_begin[kGemvMaxLayers];
    int cb_begin[kGemvMaxLayers], max_seg[kGemvMaxLayers];
    size_t counters[kGemvMaxLayers], recs[kGemvMaxLayers], partials[kGemvMaxLayers], total;
};

// Grid: every CTA resident at once -- resident CTAs per SM from the register
// budget (2 for m <= 8, 1 above) and the shared memory (228 KB per SM, 1 KB
// reserved per CTA) -- but at least two units per warp; max_seg = the most
// CTAs any column block of the layer is split over.
static GemvGroupPlan gemv_group_plan(const int64_t *k, const int64_t *n, int count, int64_t m, int K, int sms)
{
    GemvGroupPlan pl;
    pl.units = 0;
    int cb = 0;
    for (int l = 0; l < count; ++l) {
        pl.unit_begin[l] = pl.units;
        pl.cb_begin[l] = cb;
        pl.units += (k[l] / 16) * (n[l] / 128);
        cb += (int)(n[l] / 128);
    }
    pl.smem = 128 + kGemvWarps * kGemvDepth * gemv_stage_bytes(K, gemv_mg(m)) + kGemvWarps * (int)m * 128 * 4;
    int64_t occ = m <= 8 ? 2 : 1;
    const int64_t occ_smem = (228 * 1024) / (pl.smem + 1024);
    if (occ_smem < occ)
        occ = occ_smem > 0 ? occ_smem : 1;
    int64_t G = occ * (int64_t)sms;
    const int64_t gmax = pl.units / (2 * kGemvWarps);  // at least 2 units per warp
    if (G > gmax)
        G = gmax > 0 ? gmax : 1;
    if (count == 1) {
        // A whole number of CTAs per column block aligns the CTA ranges with
        // the column blocks, so no CTA straddles two (one segment end instead
        // of two, each about as costly as 8 units).  Take it when the busiest
        // SM's modelled work (units + 8 per segment end) is lower.
        const int64_t ncb = n[0] / 128;
        const int64_t s_blk = G / ncb;
        if (s_blk >= 1 && s_blk * ncb != G) {
            auto cost = [&](int64_t g, int64_t segs) {
                const int64_t per_sm = (g + sms - 1) / sms;
                return (pl.units + g - 1) / g * per_sm + 8 * segs * per_sm;
            };
            if (cost(s_blk * ncb, 1) < cost(G, 2))
                G = s_blk * ncb;
        }
    }
    pl.ctas = (int)G;
    size_t off = 256;
    for (int l = 0; l < count; ++l) {
        pl.counters[l] = off;
        off += (size_t)(n[l] / 128) * 4;
    }
    off = (off + 255) / 256 * 256;
    for (int l = 0; l < count; ++l) {
        const int64_t TR = k[l] / 16, ncb = n[l] / 128;
        int64_t max_seg = 1;
        for (int64_t c = 0; c < ncb; ++c) {
            const int64_t b0 = pl.unit_begin[l] + c * TR;
            const int64_t s = owner_cta_host(b0 + TR - 1, pl.units, G) - owner_cta_host(b0, pl.units, G) + 1;
            max_seg = s > max_seg ? s : max_seg;
        }
        pl.max_seg[l] = (int)max_seg;
        pl.recs[l] = off;
        off += ((size_t)k[l] * rec_slots_for(gemv_mg(m)) * 16 + 255) / 256 * 256;
    }
    for (int l = 0; l < count; ++l) {
        pl.partials[l] = off;
        off += ((size_t)(n[l] / 128) * (size_t)pl.max_seg[l] * (size_t)m * 128 * 4 + 255) / 256 * 256;
    }
    pl.total = off;
    return pl;
}

size_t gemv_workspace_bytes(int64_t m, int64_t k, int64_t n, int sms)
{
    size_t most = 0;
    for (int K = 1; K <= 8; ++K) {
        const size_t b = gemv_group_plan(&k, &n, 1, m, K, sms).total;
        most = b > most ? b : most;
    }
    return most;
}

template <int K, int MG>
static exl3_status launch_gemv_t(const GemvParams &p, int smem, cudaStream_t stream)
{
    auto kern = p.count > 1 ? gemv_kernel<K, MG, true> : gemv_kernel<K, MG, false>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return EXL3_ERR_CUDA;
    if (launch_kernel(kern, dim3((unsigned)p.ctas), dim3(kGemvThreads), (size_t)smem, stream, p) != cudaSuccess)
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

// Launches the rotation kernel over `count` (<= kGemvRotMaxLayers) layers:
// layer l's records go to recs[l].
static exl3_status launch_rotation(const exl3_linear *const *layers, unsigned char *const *recs, int count,
                                   int64_t m, cudaStream_t stream)
{
    const int sms = num_sms();
    GemvRotParams rp;
    rp.count = count;
    rp.m = (int)m;
    int64_t jobs = 0;
    const int quads = rec_quads((int)m, 0) + rec_quads((int)m, 1);
    for (int l = 0; l < count; ++l) {
        rp.L[l].x = (const __half *)layers[l]->x;
        rp.L[l].suh = (const __half *)layers[l]->suh;
        rp.L[l].recs = recs[l];
        rp.L[l].k = (int)layers[l]->k;
        rp.L[l].job_begin = jobs;
        jobs += (int64_t)quads * (layers[l]->k / 128);
    }
    rp.jobs = jobs;
    int64_t rgrid = (jobs + 7) / 8;
    if (rgrid > 4 * (int64_t)sms)
        rgrid = 4 * (int64_t)sms;
    if (rgrid < 1)
        rgrid = 1;
    if (launch_kernel(gemv_rotate_kernel, dim3((unsigned)rgrid), dim3(256), 0, stream, rp) != cudaSuccess)
        return EXL3_ERR_CUDA;
    return launch_status();
}

// The main launch over up to kGemvMaxLayers layers of the same K, with the
// workspace region `ws` laid out by gemv_group_plan; with `rotate` it first
// launches the rotation for them (else their records are already in place).
static exl3_status run_gemv_group(const exl3_linear *const *layers, int count, int64_t m, int K,
                                  unsigned char *ws, size_t ws_bytes, cudaStream_t stream, bool rotate = true)
{
    const int sms = num_sms();
    int64_t k[kGemvMaxLayers], n[kGemvMaxLayers];
    for (int l = 0; l < count; ++l) {
        k[l] = layers[l]->k;
        n[l] = layers[l]->n;
    }
    const GemvGroupPlan pl = gemv_group_plan(k, n, count, m, K, sms);
    if (!ws || !aligned16(ws) || ws_bytes < pl.total)
        return EXL3_ERR_WORKSPACE;

    if (rotate) {
        unsigned char *recs[kGemvMaxLayers];
        for (int l = 0; l < count; ++l)
            recs[l] = ws + pl.recs[l];
        const exl3_status rs = launch_rotation(layers, recs, count, m, stream);
        if (rs != EXL3_OK)
            return rs;
    }

    GemvParams p;
    p.count = count;
    p.m = (int)m;
    p.ctas = pl.ctas;
    p.units = pl.units;
    p.cb = codebook_constants();
    for (int l = 0; l < count; ++l) {
        GemvLayer &L = p.L[l];
        L.trellis = reinterpret_cast<const unsigned char *>(layers[l]->trellis);
        L.svh = (const __half *)layers[l]->svh;
        L.y = (__half *)layers[l]->y;
        L.recs = ws + pl.recs[l];
        L.partials = reinterpret_cast<float *>(ws + pl.partials[l]);
        L.counters = reinterpret_cast<uint32_t *>(ws + pl.counters[l]);
        L.unit_begin = pl.unit_begin[l];
        L.n = (int)n[l];
        L.tr_count = (int)(k[l] / 16);
        L.cb_begin = pl.cb_begin[l];
        L.max_seg = pl.max_seg[l];
    }
    if (m <= 8)
        return launch_gemv_k<1>(p, K, pl.smem, stream);
    return launch_gemv_k<2>(p, K, pl.smem, stream);
}

exl3_status run_gemv(const void *x, const uint16_t *trellis, const void *suh, const void *svh,
                     void *y, int64_t m, int64_t k, int64_t n, int K, void *workspace,
                     size_t workspace_bytes, cudaStream_t stream)
{
    exl3_linear d;
    d.x = x;
    d.trellis = trellis;
    d.suh = suh;
    d.svh = svh;
    d.y = y;
    d.k = k;
    d.n = n;
    d.K = K;
    const exl3_linear *one = &d;
    return run_gemv_group(&one, 1, m, K, (unsigned char *)workspace, workspace_bytes, stream);
}

// The layers of a multi call, grouped by K (in call order) into launches of
// at most kGemvMaxLayers; calls f(group, count, K, workspace offset, bytes).
template <typename F>
static exl3_status for_each_gemv_group(const exl3_linear *layers, int count, int64_t m, F &&f)
{
    const int sms = num_sms();
    size_t off = 0;
    for (int K = 1; K <= 8; ++K) {
        const exl3_linear *grp[kGemvMaxLayers];
        int cnt = 0;
        for (int i = 0; i <= count; ++i) {
            const bool flush = (i == count && cnt > 0) || cnt == kGemvMaxLayers;
            if (flush) {
                int64_t k[kGemvMaxLayers], n[kGemvMaxLayers];
                for (int l = 0; l < cnt; ++l) {
                    k[l] = grp[l]->k;
                    n[l] = grp[l]->n;
                }
                const size_t bytes = gemv_group_plan(k, n, cnt, m, K, sms).total;
                const exl3_status st = f(grp, cnt, K, off, bytes);
                if (st != EXL3_OK)
                    return st;
                off += (bytes + 255) / 256 * 256;
                cnt = 0;
            }
            if (i < count && layers[i].K == K)
                grp[cnt++] = &layers[i];
        }
    }
    return EXL3_OK;
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

static exl3_status check_multi(const exl3_linear *layers, int count, int64_t m)
{
    using namespace exl3;
    if (!layers || count < 1)
        return EXL3_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        const exl3_linear &d = layers[i];
        const exl3_status st = check_linear_args(d.x, d.trellis, d.suh, d.svh, d.y, m, d.k, d.n, d.K);
        if (st != EXL3_OK)
            return st;
    }
    return m > 16 ? EXL3_ERR_UNSUPPORTED : EXL3_OK;
}

extern "C" size_t exl3_gemv_multi_workspace_size(const exl3_linear *layers, int count, int64_t m)
{
    using namespace exl3;
    if (check_multi(layers, count, m) != EXL3_OK)
        return 0;
    size_t total = 0;
    for_each_gemv_group(layers, count, m, [&](const exl3_linear *const *, int, int, size_t off, size_t bytes) {
        total = off + (bytes + 255) / 256 * 256;
        return EXL3_OK;
    });
    return total;
}

extern "C" exl3_status exl3_gemv_multi(const exl3_linear *layers, int count, int64_t m, void *workspace,
                                       size_t workspace_bytes, void *stream)
{
    using namespace exl3;
    const exl3_status st = check_multi(layers, count, m);
    if (st != EXL3_OK)
        return st;
    if (!workspace || !aligned16(workspace) || workspace_bytes < exl3_gemv_multi_workspace_size(layers, count, m))
        return EXL3_ERR_WORKSPACE;
    unsigned char *ws = (unsigned char *)workspace;
    cudaStream_t s = (cudaStream_t)stream;
    // every layer's rotation first, in launches of up to kGemvRotMaxLayers
    // layers, then one main launch per group reading its records
    const int sms = num_sms();
    const exl3_linear *rl[kGemvRotMaxLayers];
    unsigned char *rr[kGemvRotMaxLayers];
    int nr = 0;
    exl3_status st2 = for_each_gemv_group(
        layers, count, m, [&](const exl3_linear *const *grp, int cnt, int K, size_t off, size_t) {
            int64_t k[kGemvMaxLayers], n[kGemvMaxLayers];
            for (int l = 0; l < cnt; ++l) {
                k[l] = grp[l]->k;
                n[l] = grp[l]->n;
            }
            const GemvGroupPlan pl = gemv_group_plan(k, n, cnt, m, K, sms);
            for (int l = 0; l < cnt; ++l) {
                rl[nr] = grp[l];
                rr[nr] = ws + off + pl.recs[l];
                if (++nr == kGemvRotMaxLayers) {
                    const exl3_status rs = launch_rotation(rl, rr, nr, m, s);
                    if (rs != EXL3_OK)
                        return rs;
                    nr = 0;
                }
            }
            return EXL3_OK;
        });
    if (st2 == EXL3_OK && nr > 0)
        st2 = launch_rotation(rl, rr, nr, m, s);
    if (st2 != EXL3_OK)
        return st2;
    return for_each_gemv_group(layers, count, m,
                               [&](const exl3_linear *const *grp, int cnt, int K, size_t off, size_t bytes) {
                                   return run_gemv_group(grp, cnt, m, K, ws + off, bytes, s, false);
                               });
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
