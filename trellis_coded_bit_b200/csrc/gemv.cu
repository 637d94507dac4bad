// gemv.cu -- exl3_gemv: y = svh .* H(H(x .* suh) . W_hat) for 1 <= m <= 16,
// with W_hat decoded on the fly from the trellis (EXL3 GEMM kernel article,
// section 小批量GEMV: in decoding the bottleneck moves from compute to memory
// bandwidth, so a dedicated GEMV path streams the quantised weights once).
//
// B200 design (the pages' consumer-GPU GEMV is prior art, not copied):
//   * The input rotation x' = H(x .* suh)/sqrt(128) (fp32 butterflies, fp16
//     result) goes into the workspace as tensor-core B-fragment activation
//     blocks (see below), which the main loop copies into shared memory with
//     the weights.  When each CTA's unit range is short (single layers at
//     small m, where the fixed cost of a call dominates) the call is ONE
//     launch: after requesting its first weights every CTA rotates just the
//     128-channel blocks its own range reads, and a CTA barrier is all the
//     synchronisation.  Otherwise (long ranges: many layers, or m large
//     enough that a CTA would rotate many blocks) a rotation kernel runs
//     just before the main kernel, which is resident and streaming weights
//     meanwhile (programmatic dependent launch).  Sharing that rotation over
//     the main kernel's own warps behind a grid barrier measured slower on
//     the 20-layer decode step (170.4 against 169.2 us per step back to back).
//   * The kernel is persistent and "stream-K" balanced.  One launch
//     serves every layer of an exl3_gemv_multi call (up to 32, any mix of K):
//     its CTAs are split into one group per K, in proportion to the group's
//     cost, so that each CTA runs the decode compiled for one K.  Within a
//     group the work units -- (layer, 128-column block, tile row of 16 input
//     channels) -- are numbered consecutively and CTA c of G owns the
//     contiguous range [cU/G, (c+1)U/G); its 8 warps take units u0 + w,
//     u0 + w + 8, ..., so a CTA's concurrent loads stay within a few
//     consecutive tile rows.  A range is cut into segments at column-block
//     boundaries.  At a segment end the warps' partials meet in shared memory
//     (one barrier) and either finish the block (output rotation, svh, fp16 y)
//     or go to the workspace, where the last segment to arrive on the block's
//     counter (atomic ticket, no spinning) sums all segments in segment order
//     (deterministic) and finishes it.
//   * The MAC runs on the tensor cores (mma.sync m16n8k16, fp32 accumulate)
//     with the WEIGHTS in the A operand: a codebook word's two fp16 halves
//     form a pair of k slots and the activation is duplicated over that pair
//     in B, so the tensor core forms x*(hi + lo) exactly in fp32 (the fp16
//     rounding of hi + lo that defines W_hat is skipped: at most half an fp16
//     ulp per weight, far inside the output tolerance).  One MMA thus takes
//     16 output columns x 8 input channels = 128 weights, and its 8 B columns
//     are 8 batches: at m = 1 the tensor pipe does half the work it would
//     with the weights in B.
//   * Lane (g, t) owns tile g of the 128-column block and, in k-step ks, the
//     two adjacent tile rows 8ks + 2t and 8ks + 2t + 1: one contiguous run of
//     2K + 1 words (with the prefix word) whose 32 bit windows are
//     compile-time byte permutes and multiplies (pair_codes), which move what
//     they can from the ALU pipe (byte permutes and the codebook's mask/xor)
//     to the FMA pipe (the codebook's multiply, shifts as multiplies, and an
//     exact correction that lets a window skip its zero-fill when the 16 bits
//     above it are another window's state).  Weight (row 8ks + 2t + p,
//     column c) goes to A row g + 8(c & 1), k-pair t + 4p of MMA c / 2, so
//     MMA j accumulates columns 2j and 2j + 1 of every tile of the block.
//   * Each warp streams its units through its own 3-deep cp.async ring in
//     shared memory (8 tiles padded against bank conflicts, plus the unit's
//     activation block), loaded by 16-byte copies spread over the lanes.
//   * With EXL3_LAUNCH_PDL the kernel is resident and requests its first
//     weights while the preceding kernel drains, and waits for it
//     (griddepcontrol) only before it reads x.
#include <cuda_fp16.h>

#include "exl3_device.cuh"
#include "exl3_host.h"

namespace exl3 {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = 32 * kGemvWarps;

// Activation blocks, in MMA B-fragment register order.  For tile row tr
// (input channels 16tr .. 16tr+15) and batch group mg (batches 8mg .. 8mg+7)
// a 512-byte block; its 8-byte entry (ks, g, t) at ks*256 + g*32 + t*8 holds
// channels 16tr + 8ks + 2t and 16tr + 8ks + 2t + 1 of batch 8mg + g, each an
// fp16 duplicated into both halves of a 32-bit word: exactly the (b0, b1)
// that lane (g, t) feeds the MMA in k-step ks.  Block (tr, mg) sits at
// (tr * MG + mg) * 512.  Only batches < m are written and copied; the ring's
// entries of absent batches are zero (they feed only B columns whose
// accumulators are never stored).
constexpr int kGemvActBlock = 512;

// The first bytes of every GEMV workspace hold the words a call needs to find
// at zero when it starts (status word, arrival counters; every call leaves
// them at zero), and no call writes data there, so one workspace can serve
// calls of any shapes in turn.
constexpr size_t kGemvSyncArea = 64 * 1024;

__host__ __device__ inline int gemv_mg(int64_t m)
{
    return m > 8 ? 2 : 1;
}

// ---------------------------------------------------------- main kernel ---

// One launch covers up to kGemvMaxLayers layers with the same m and any mix
// of K.  The layers are grouped by K; each group gets its own share of the
// grid's CTAs (in proportion to its estimated cost), so that every CTA runs
// the decode compiled for one K.  Within a group the work units -- (layer,
// 128-column block, tile row) -- are numbered consecutively: layer by layer,
// column block by column block, tile row by tile row.
constexpr int kGemvMaxLayers = 32;

struct GemvLayer {
    const unsigned char *trellis;  // uint16 [k/16][n/16][16K]
    const __half *x, *suh, *svh;
    __half *y;
    unsigned char *acts;        // activation blocks [k/16][MG][512 B]
    float *partials;            // [n/128][max_seg][m][128]
    uint32_t *counters;         // [n/128]
    int64_t unit_begin;         // the layer's first unit within its group
    int n, tr_count, max_seg;
    int cb_begin;               // the layer's first column block within its group
};

// A group: the layers [l_begin, l_end) of one K, run by the CTAs
// [cta_begin, cta_begin + ctas) over its `units` units.
struct GemvGroup {
    int64_t units;
    int K, l_begin, l_end, cta_begin, ctas;
};

// Multipliers the window extraction uses in place of shifts, passed in as
// launch parameters so that they stay opaque registers: a multiply by a
// register runs on the FMA pipe (IMAD), which the decode leaves half idle,
// while shifts and byte permutes compete with the codebook's LOP3 for the
// ALU pipe.  pow2[i] = 2^i.  (The upper-half word windows stay byte permutes:
// as a mul.hi by 2^16 they measured slower.)
struct GemvMults {
    uint32_t pow2[8];
};

struct GemvParams {
    GemvLayer L[kGemvMaxLayers];
    GemvGroup grp[8];
    int ngroups, m;
    // Input rotation: rot_local != 0 -- every CTA rotates the 128-channel
    // blocks its own unit range reads; 0 -- the rotation kernel launched just
    // before has written every activation block.
    int rot_local;
    Codebook cb;
    GemvMults mu;
};

// Per-warp shared-memory ring of kGemvDepth stages; a stage holds one unit:
// the tile row's activation blocks (MG x 512 bytes, at the stage start, so
// their place does not depend on K) and then the unit's 8 tiles, each padded
// to 32K + pad bytes so that the lanes' run reads spread over the banks (the
// pad per K minimises the modelled shared-memory wavefronts of those reads).
// Within a stage every offset is a compile-time function of K and MG, so the
// inner loop addresses shared memory as a lane pointer plus immediates.
__host__ __device__ constexpr int gemv_tile_pad(int K)
{
    return K == 4 ? 64 : ((K == 2 || K == 6) ? 32 : 16);
}

__host__ __device__ constexpr int gemv_tile_stride(int K)
{
    return 32 * K + gemv_tile_pad(K);
}

__host__ __device__ constexpr int gemv_stage_bytes(int K, int MG)
{
    return (MG * kGemvActBlock + 8 * gemv_tile_stride(K) + 127) & ~127;
}

constexpr int kGemvDepth = 3;  // units in flight per warp (one consumed, the rest loading)

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

// The 32 codebook words of a row pair from its run of words.  R[0] holds the
// prefix word in its upper half, R[i] (i = 1..K) holds the pair's words
// 2i - 2 (lower half) and 2i - 1 (upper half).  Counting stream positions
// from the prefix word W'[0] (W'[i] = positions 16i .. 16i + 15; W'[2i-1] is
// R[i]'s lower half, W'[2i] its upper half), weight jj (row jj / 16, column
// jj % 16) has the window ending at position e = 16 + (jj + 1) K.
//   * When e is a multiple of 16 the window is the word W'[e/16 - 1]: an
//     upper half is one byte permute with zero fill; a lower half, when K
//     divides 16, needs no extraction at all: with R = W'[w+1] 2^16 + W'[w]
//     and W'[w+1] itself the state of weight jj' = jj + 16/K, R*C1 + C2
//     differs from the wanted s*C1 + C2 only by (W'[w+1] C1 mod 2^16) 2^16,
//     and W'[w+1] C1 mod 2^16 is the low half of jj''s own product less C2:
//     so v = R*C1 + (C2 + C2 2^16) - v' 2^16, two multiply-adds on the FMA
//     pipe, exact mod 2^32.
//   * A window 8 bits off a word boundary that lies inside one loaded
//     register (a even) is one byte permute of that register.  For K = 8 one
//     that straddles two registers is the low half of the 32-bit window
//     ending at the same place (one byte permute of the two registers),
//     whose upper half is the state of weight jj - 2, and is corrected the
//     same way.
//   * Otherwise the window lies in V = W'[a-1]:W'[a] (a = e / 16, as one
//     big-endian 32-bit value) shifted right by c = 16 - e % 16, and is one
//     byte permute with zero fill of V, or of V times 2^(8 - c % 8) (a left
//     shift, as a multiply on the FMA pipe).
// All selectors are compile-time constants, and the V values and their
// shifted copies are shared between windows.  The result is the codebook
// word (v & mask) ^ xor of each window's state.
template <int K>
__device__ __forceinline__ void pair_codes(const uint32_t (&R)[K + 1], uint32_t (&w)[32], const Codebook &cb,
                                           uint32_t c2p, const GemvMults &mu)
{
    constexpr bool kJunk = (16 % K) == 0;
    constexpr int kStep = kJunk ? 16 / K : 0;
    uint32_t v[32];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
        const int e = 16 + (jj + 1) * K;
        const int a = e >> 4, rb = e & 15;
        const int c = 16 - rb;
        uint32_t s;
        if (rb == 0) {
            const int wd = a - 1;
            if (wd & 1) {
                if (kJunk)
                    continue;  // corrected below from the window 16 bits later
                s = __byte_perm(R[(wd + 1) >> 1], 0u, 0x4410u);
            } else {
                s = __byte_perm(R[wd >> 1], 0u, 0x4432u);
            }
        } else if (c == 8 && !(a & 1)) {
            s = __byte_perm(R[a >> 1], 0u, 0x4403u);
        } else if (c == 8 && K == 8 && jj >= kStep) {
            continue;  // corrected below from the window 16 bits earlier
        } else {
            const uint32_t vv = (a & 1) ? __byte_perm(R[(a - 1) >> 1], R[(a + 1) >> 1], 0x3254u)
                                        : __byte_perm(R[a >> 1], 0u, 0x1032u);
            const int r = c & 7, cbt = c >> 3;
            if (r == 0) {
                s = __byte_perm(vv, 0u, 0x4400u | ((uint32_t)(cbt + 1) << 4) | (uint32_t)cbt);
            } else {
                // bits [c, c + 16) of vv are bits [8(cbt + 1), 8(cbt + 1) + 16) of
                // vv * 2^(8 - r); the bits shifted out lie above the window
                const uint32_t vs = vv * mu.pow2[8 - r];
                s = __byte_perm(vs, 0u, 0x4400u | ((uint32_t)(cbt + 2) << 4) | (uint32_t)(cbt + 1));
            }
        }
        v[jj] = s * cb.mul + cb.add;
    }
    if constexpr (kJunk) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
            const int e = 16 + (jj + 1) * K;
            const int a = e >> 4, rb = e & 15;
            if (rb == 0 && ((a - 1) & 1)) {
                v[jj] = v[jj + kStep] * 0xFFFF0000u + (R[a >> 1] * cb.mul + c2p);
            } else if (K == 8 && rb == 8 && (a & 1) && jj >= kStep) {
                const uint32_t xw = __byte_perm(R[(a - 1) >> 1], R[(a + 1) >> 1], 0x0325u);
                v[jj] = v[jj - kStep] * 0xFFFF0000u + (xw * cb.mul + c2p);
            }
        }
    }
#pragma unroll
    for (int jj = 0; jj < 32; ++jj)
        w[jj] = (v[jj] & cb.mask) ^ cb.xr;
}

// The lane's pointers into a stage of its ring (stage 0 as set up; the loop
// adds the stage offset): its tile's k-step-0 run (word tK), its k-step-0
// prefix word (the tile's last word for t = 0: the tail-biting wrap), and its
// activation entry.
struct GemvLanePtrs {
    const unsigned char *run, *pre0, *act;
};

// Loads the words of the lane's row pair of k-step KS: R[0] the prefix word,
// R[1..K] the pair's 2K words, as wide as the run's alignment allows (4tK
// bytes into a 16-byte aligned tile: 16 bytes for K % 4 == 0, 8 for even K,
// else 4).
template <int K, int KS>
__device__ __forceinline__ void load_pair(const GemvLanePtrs &lp, uint32_t (&R)[K + 1])
{
    const unsigned char *run = lp.run + KS * 16 * K;
    R[0] = KS == 0 ? *reinterpret_cast<const uint32_t *>(lp.pre0) : *reinterpret_cast<const uint32_t *>(run - 4);
    if constexpr (K % 4 == 0) {
#pragma unroll
        for (int i = 0; i < K / 4; ++i) {
            const uint4 v = *reinterpret_cast<const uint4 *>(run + 16 * i);
            R[4 * i + 1] = v.x;
            R[4 * i + 2] = v.y;
            R[4 * i + 3] = v.z;
            R[4 * i + 4] = v.w;
        }
    } else if constexpr (K % 2 == 0) {
#pragma unroll
        for (int i = 0; i < K / 2; ++i) {
            const uint2 v = *reinterpret_cast<const uint2 *>(run + 8 * i);
            R[2 * i + 1] = v.x;
            R[2 * i + 2] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < K; ++i)
            R[i + 1] = *reinterpret_cast<const uint32_t *>(run + 4 * i);
    }
}

// One unit held in the ring stage the lane pointers point into: for each
// k-step decode the lane's row pair (32 weights) and run the 8 MMAs (per
// batch group) that consume it.  Both k-steps are unrolled (their loads and
// decodes overlap); the stage is a run-time base (one compiled copy of the
// body per K: three copies with compile-time stage offsets measured 6%
// slower on the decode step, from instruction-cache misses).
template <int K, int MG>
__device__ __forceinline__ void mac_unit(const GemvLanePtrs &lp, const Codebook &cb, const GemvMults &mu,
                                         float (&acc)[MG][8][4])
{
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t B[MG][2];
#pragma unroll
        for (int mg = 0; mg < MG; ++mg) {
            const uint2 b = *reinterpret_cast<const uint2 *>(lp.act + ks * 256 + mg * kGemvActBlock);
            B[mg][0] = b.x;
            B[mg][1] = b.y;
        }
        uint32_t R[K + 1];
        if (ks == 0)
            load_pair<K, 0>(lp, R);
        else
            load_pair<K, 1>(lp, R);
        uint32_t wv[32];
        pair_codes<K>(R, wv, cb, cb.add + (cb.add << 16), mu);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t a[4] = {wv[2 * j], wv[2 * j + 1], wv[16 + 2 * j], wv[17 + 2 * j]};
#pragma unroll
            for (int mg = 0; mg < MG; ++mg)
                mma_16816(acc[mg][j], a, B[mg][0], B[mg][1]);
        }
    }
}

// CTA owning unit u: the largest c with floor(c U / G) <= u.
__host__ __device__ inline int64_t gemv_owner_cta(int64_t u, int64_t U, int64_t G)
{
    return ((u + 1) * G - 1) / U;
}

// Position of unit u of a group: layer l (scanning on from l, within
// [lb, le)), column block cb within it, tile row tr.
__device__ __forceinline__ void gemv_locate(const GemvParams &p, int le, int64_t u, int &l, int &cb, int &tr)
{
    while (l + 1 < le && u >= p.L[l + 1].unit_begin)
        ++l;
    const int64_t lu = u - p.L[l].unit_begin;
    const int TR = p.L[l].tr_count;
    cb = (int)(lu / TR);
    tr = (int)(lu - (int64_t)cb * TR);
}

// Output rotation, svh and fp16 store of one column block's m x 128 y'
// (summed in shared memory): a warp per batch row.
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

// ------------------------------------------------------ input rotation ---

// x' = H(x .* suh)/sqrt(128) for one 128-channel block `blk` of batch row b
// of a layer with k input channels, by one warp: lane l rotates channels
// 4l .. 4l+3 (fp32 butterflies, fp16 result) and writes them as one 16-byte
// piece of the activation blocks `acts` (each value duplicated into both
// halves of a word).
__device__ __forceinline__ void rotate_block(const __half *x, const __half *suh, unsigned char *acts, int k,
                                             int m, int b, int blk, int lane)
{
    const int MG = gemv_mg(m);
    const int c = blk * 128 + lane * 4;
    const uint2 sr = *reinterpret_cast<const uint2 *>(suh + c);
    const uint2 r0 = *reinterpret_cast<const uint2 *>(x + (int64_t)b * k + c);
    const __half2 *sv = reinterpret_cast<const __half2 *>(&sr);
    const __half2 *x0 = reinterpret_cast<const __half2 *>(&r0);
    float v[4] = {__low2float(x0[0]) * __low2float(sv[0]), __high2float(x0[0]) * __high2float(sv[0]),
                  __low2float(x0[1]) * __low2float(sv[1]), __high2float(x0[1]) * __high2float(sv[1])};
    warp_fwht128(v);
    const float s128 = 0.08838834764831845f;
    uint32_t d[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t h = (uint32_t)__half_as_ushort(__float2half_rn(v[e] * s128));
        d[e] = h | (h << 16);
    }
    // channels c .. c+3: tile row c / 16, rows r .. r+3 with r = c % 16
    // (r = 8ks + 2t0, t0 even): entries (ks, g, t0) and (ks, g, t0 + 1)
    const int tr = c >> 4, r = c & 15;
    const int mg = b >> 3, g = b & 7;
    unsigned char *dst =
        acts + ((int64_t)tr * MG + mg) * kGemvActBlock + (r >> 3) * 256 + g * 32 + ((r & 7) >> 1) * 8;
    *reinterpret_cast<uint4 *>(dst) = make_uint4(d[0], d[1], d[2], d[3]);
}

// Local rotation: the CTA rotates the blocks that hold the tile rows of its
// own unit range [u0, u1), which the host guarantees to span at most two
// column blocks: rows [r0, r1] of one, or rows [r0, TR) of the first and
// [0, r1] of the second (possibly of the next layer).  CTAs whose ranges
// share a block write the same bytes.  A CTA barrier afterwards makes the
// blocks visible to the CTA's own copies.
__device__ __forceinline__ void rotate_local(const GemvParams &p, int lb, int le, int64_t u0, int64_t u1,
                                             int warp, int lane)
{
    int l0 = lb, c0 = 0, r0 = 0, l1 = lb, c1 = 0, r1 = 0;
    gemv_locate(p, le, u0, l0, c0, r0);
    gemv_locate(p, le, u1 - 1, l1, c1, r1);
    const int m = p.m;
    const bool one = l0 == l1 && c0 == c1;
    // segment A: layer l0, blocks [a0, a1]; segment B: layer l1, blocks [0, b1]
    const int a0 = r0 >> 3, a1 = one ? (r1 >> 3) : ((p.L[l0].tr_count - 1) >> 3);
    const int nA = (a1 - a0 + 1) * m, nB = one ? 0 : ((r1 >> 3) + 1) * m;
    for (int j = warp; j < nA + nB; j += kGemvWarps) {
        const GemvLayer &L = p.L[j < nA ? l0 : l1];
        const int jj = j < nA ? j : j - nA;
        rotate_block(L.x, L.suh, L.acts, 16 * L.tr_count, m, jj % m, (j < nA ? a0 : 0) + jj / m, lane);
    }
}

// The work of one CTA of a K group.  CTA c of the group's G owns the
// contiguous unit range [cU/G, (c+1)U/G); its 8 warps take units u0 + w,
// u0 + w + 8, ..., so that a CTA's concurrent loads stay within a few
// consecutive tile rows.  The range is cut into segments at column-block
// boundaries; at a segment end the warps' partials meet in shared memory (a
// CTA barrier) and either finish the block or go to the workspace, where the
// last segment to arrive (atomic ticket, no spinning) sums all segments in
// segment order and finishes it.
template <int K, int MG>
__device__ __forceinline__ void gemv_cta(const GemvParams &p, const GemvGroup &gp)
{
    constexpr int SB = gemv_stage_bytes(K, MG);
    constexpr int S = gemv_tile_stride(K);
    constexpr int kTrChunks = (16 * K + 31) / 32;  // 16-byte trellis chunks per lane per unit
    extern __shared__ __align__(128) unsigned char smem[];
    volatile int *flag = reinterpret_cast<volatile int *>(smem);
    const int m = p.m;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    float *red = reinterpret_cast<float *>(smem + 128);
    unsigned char *ring = smem + 128 + kGemvWarps * m * 128 * 4 + warp * kGemvDepth * SB;
    const int lb = gp.l_begin, le = gp.l_end;
    const int64_t U = gp.units;
    const int64_t G = gp.ctas;
    const int64_t c = (int64_t)blockIdx.x - gp.cta_begin;
    const int64_t u0 = c * U / G, u1 = (c + 1) * U / G;

    GemvLanePtrs lp;
    lp.run = ring + MG * kGemvActBlock + g * S + 4 * t * K;
    lp.pre0 = t == 0 ? ring + MG * kGemvActBlock + g * S + 4 * (8 * K - 1) : lp.run - 4;
    lp.act = ring + g * 32 + t * 8;
    // the lane's trellis chunks (chunk i = lane + 32r of the unit's 16K: tile
    // i / 2K, 16-byte piece i % 2K) and activation chunks (entry row (ks, g')
    // with g' = (lane >> 1) & 7, i.e. batch 8 mg + g'; only batches < m)
    unsigned char *tdst[kTrChunks];
#pragma unroll
    for (int r = 0; r < kTrChunks; ++r) {
        const int i = lane + 32 * r;
        tdst[r] = ring + MG * kGemvActBlock + (i / (2 * K)) * S + (i % (2 * K)) * 16;
    }
    const bool last_chunk = (16 * K) % 32 == 0 || lane + 32 * (kTrChunks - 1) < 16 * K;
    bool act_live[MG];
#pragma unroll
    for (int mg = 0; mg < MG; ++mg)
        act_live[mg] = 8 * mg + ((lane >> 1) & 7) < m;

    // this warp's units: u0 + warp + kGemvWarps i, i < nunits
    const int nunits = u0 + warp < u1 ? (int)((u1 - u0 - warp + kGemvWarps - 1) / kGemvWarps) : 0;

    // issue iterator (runs kGemvDepth units ahead of consumption): the next
    // unit to copy is at (layer il, column block icb, tile row itr); `rem`
    // units are left to copy.  A step of kGemvWarps tile rows crosses at most
    // one column block while kGemvWarps <= every layer's tile rows (k >= 128)
    int rem = nunits;
    int il = lb, icb = 0, itr = 0;
    gemv_locate(p, le, rem ? u0 + warp : u0, il, icb, itr);
    int itr_lim = 0, incb = 0;
    int64_t tile_rows_step = 0;  // kGemvWarps tile rows of the layer's matrix, in bytes
    const unsigned char *isrc = nullptr, *iasrc = nullptr;
    auto enter_block = [&]() {
        const GemvLayer &L = p.L[il];
        itr_lim = L.tr_count;
        incb = L.n >> 7;
        const int64_t tile_row_bytes = (int64_t)(L.n >> 4) * 32 * K;
        tile_rows_step = kGemvWarps * tile_row_bytes;
        isrc = L.trellis + itr * tile_row_bytes + (int64_t)icb * 256 * K + lane * 16;
        iasrc = L.acts + (int64_t)itr * MG * kGemvActBlock + lane * 16;
    };
    if (rem)
        enter_block();
    auto copy_acts = [&](int stage, const unsigned char *src) {
#pragma unroll
        for (int mg = 0; mg < MG; ++mg)
            if (act_live[mg])
                cp_async16(ring + stage * SB + mg * kGemvActBlock + lane * 16, src + mg * kGemvActBlock);
    };
    // copies the trellis of the issue iterator's unit into `stage` (rem > 0),
    // returns the unit's activation source and advances by 8 units
    auto issue_trellis = [&](int stage) -> const unsigned char * {
        const unsigned char *asrc = iasrc;
        const int so = stage * SB;
#pragma unroll
        for (int r = 0; r < kTrChunks; ++r)
            if (r < kTrChunks - 1 || last_chunk)
                cp_async16(tdst[r] + so, isrc + 512 * r);
        --rem;
        isrc += tile_rows_step;
        iasrc += kGemvWarps * MG * kGemvActBlock;
        itr += kGemvWarps;
        if (itr >= itr_lim) {  // next column block, perhaps of the next layer (8 <= every TR)
            itr -= itr_lim;
            if (++icb == incb) {
                icb = 0;
                ++il;
            }
            if (rem)
                enter_block();
        }
        return asrc;
    };
    auto issue = [&](int stage) {
        if (rem > 0)
            copy_acts(stage, issue_trellis(stage));
        cp_async_commit();
    };

    // Prologue: the first kGemvDepth units' weights are requested before the
    // wait for the preceding kernel (which may write x; a no-op without PDL),
    // then the input rotation writes the activation blocks, and the units'
    // activations are copied after it.  The ring's entries of absent batches
    // are zeroed once; copies never touch them.
    const unsigned char *asrc0[kGemvDepth];
#pragma unroll
    for (int d = 0; d < kGemvDepth; ++d) {
        asrc0[d] = rem > 0 ? issue_trellis(d) : nullptr;
        cp_async_commit();
    }
#pragma unroll
    for (int d = 0; d < kGemvDepth; ++d)
#pragma unroll
        for (int o = lane * 16; o < MG * kGemvActBlock; o += 512)
            *reinterpret_cast<uint4 *>(ring + d * SB + o) = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    grid_dep_wait();
    grid_dep_launch();  // a dependent launch still waits for this grid to complete
    if (p.rot_local) {
        rotate_local(p, lb, le, u0, u1, warp, lane);
        __syncthreads();
    }
#pragma unroll
    for (int d = 0; d < kGemvDepth; ++d)
        if (asrc0[d])
            copy_acts(d, asrc0[d]);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();

    const Codebook cb = p.cb;
    const GemvMults mu = p.mu;
    float acc[MG][8][4];
#pragma unroll
    for (int a = 0; a < MG; ++a)
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[a][j][e] = 0.f;

    // the CTA's range as the group's column blocks [g0, g1]
    int l0 = lb, c0 = 0, r0 = 0, c1 = 0, r1 = 0;
    gemv_locate(p, le, u0, l0, c0, r0);
    int l1 = l0;
    gemv_locate(p, le, u1 - 1, l1, c1, r1);
    const int g0 = p.L[l0].cb_begin + c0, g1 = p.L[l1].cb_begin + c1;
    int sl = l0;  // layer of the current segment's column block
    int st = 0;
    int ci = 0;  // units consumed
    for (int gk = g0; gk <= g1; ++gk) {
        while (sl + 1 < le && gk >= p.L[sl + 1].cb_begin)
            ++sl;
        const GemvLayer &SL = p.L[sl];
        const int TR = SL.tr_count;
        const int cbk = gk - SL.cb_begin;  // column block within the layer
        const int64_t blk_begin = SL.unit_begin + (int64_t)cbk * TR, blk_end = blk_begin + TR;
        const int64_t seg_begin = blk_begin > u0 ? blk_begin : u0;
        const int64_t seg_end = blk_end < u1 ? blk_end : u1;
        // this warp's units below seg_end: ceil((seg_end - u0 - warp) / kGemvWarps)
        const int rel_end = (int)(seg_end - u0) - warp;
        const int upto = rel_end > 0 ? (rel_end + kGemvWarps - 1) / kGemvWarps : 0;
        for (; ci < upto; ++ci) {
            cp_async_wait<kGemvDepth - 1>();
            __syncwarp();
            {
                const int so = st * SB;
                GemvLanePtrs ls;
                ls.run = lp.run + so;
                ls.pre0 = lp.pre0 + so;
                ls.act = lp.act + so;
                mac_unit<K, MG>(ls, cb, mu, acc);
            }
            __syncwarp();  // every lane is done with the stage before it is refilled
            issue(st);
            st = st + 1 == kGemvDepth ? 0 : st + 1;
        }

        // ------------------------------------------- segment end: reduce ---
        // accumulator (mg, j, e): A row g + 8 (e >> 1) -> block column 16g + 2j
        // + (e >> 1); B column 2t + (e & 1) -> batch 8mg + 2t + (e & 1)
#pragma unroll
        for (int mg = 0; mg < MG; ++mg)
#pragma unroll
            for (int pb = 0; pb < 2; ++pb) {
                const int b = 8 * mg + 2 * t + pb;
                if (b < m) {
                    float4 *dst = reinterpret_cast<float4 *>(red + (warp * m + b) * 128 + 16 * g);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_float4(acc[mg][2 * q][pb], acc[mg][2 * q][2 + pb], acc[mg][2 * q + 1][pb],
                                             acc[mg][2 * q + 1][2 + pb]);
                }
            }
#pragma unroll
        for (int mg = 0; mg < MG; ++mg)
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[mg][j][e] = 0.f;
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
            const int c_first = (int)gemv_owner_cta(blk_begin, U, G);
            const int c_last = (int)gemv_owner_cta(blk_end - 1, U, G);
            const int nseg = c_last - c_first + 1;
            const int j = (int)c - c_first;
            float *part = SL.partials + ((int64_t)cbk * SL.max_seg) * m * 128;
            for (int e = tid; e < m * 128; e += kGemvThreads)
                part[(int64_t)j * m * 128 + e] = red[e];
            __syncthreads();
            if (tid == 0) {
                __threadfence();  // the barrier orders the other threads' stores before this fence
                const uint32_t ticket = atomicAdd(&SL.counters[cbk], 1u);
                *flag = (ticket == (uint32_t)(nseg - 1)) ? 1 : 0;
                __threadfence();
            }
            __syncthreads();
            if (*flag == 1) {
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

// The persistent main kernel: each CTA finds its K group and runs the body
// compiled for that K.
template <int MG>
__global__ void __launch_bounds__(kGemvThreads, MG == 1 ? 2 : 1) gemv_kernel(const GemvParams p)
{
    int q = 0;
    while (q + 1 < p.ngroups && (int)blockIdx.x >= p.grp[q + 1].cta_begin)
        ++q;
    const GemvGroup &gp = p.grp[q];
    switch (gp.K) {
    case 1: gemv_cta<1, MG>(p, gp); break;
    case 2: gemv_cta<2, MG>(p, gp); break;
    case 3: gemv_cta<3, MG>(p, gp); break;
    case 4: gemv_cta<4, MG>(p, gp); break;
    case 5: gemv_cta<5, MG>(p, gp); break;
    case 6: gemv_cta<6, MG>(p, gp); break;
    case 7: gemv_cta<7, MG>(p, gp); break;
    default: gemv_cta<8, MG>(p, gp); break;
    }
}

// ------------------------------------------------------------- dispatch ---

// Plan of one launch over `count` layers (same m): the K groups and their
// CTAs, shared memory, and the workspace layout -- [0, 256) status word; the
// layers' arrival counters (one per column block, consecutive); from
// kGemvSyncArea on, per layer its activation blocks (k / 16 * MG * 512 bytes)
// and split partials [n/128][max_seg][m][128].  Workspace offsets are indexed by the layer's
// place in the call; the group order is `order`.
struct GemvPlan {
    int ctas, smem, ngroups;
    GemvGroup grp[8];
    int order[kGemvMaxLayers];  // call index of the plan's l-th layer (grouped by K)
    int64_t unit_begin[kGemvMaxLayers];
    int cb_begin[kGemvMaxLayers], max_seg[kGemvMaxLayers];  // by plan index
    size_t counters[kGemvMaxLayers], acts[kGemvMaxLayers], partials[kGemvMaxLayers];  // by call index
    size_t sync_bytes, total;
    int rot_local;  // input rotation per CTA (1) or shared with a grid barrier (0)
};

// Relative time of one unit at m = 1 by K: each K group of the Llama-3.1-8B
// decode set timed alone on B200, less about 8.5 us of fixed launch cost (K =
// 1, 5, 7 interpolated; K = 4 and 8 load their runs in 16-byte pieces and have
// the cheapest windows, odd K load 4-byte pieces).  It sets each group's share
// of the grid.
static int64_t gemv_unit_cost(int K)
{
    static const int64_t cost[9] = {0, 296, 301, 323, 306, 335, 346, 336, 326};
    return cost[K < 1 ? 1 : (K > 8 ? 8 : K)];
}

// Grid: every CTA resident at once -- resident CTAs per SM from the register
// budget (2 for m <= 8, 1 above) and the shared memory (228 KB per SM, 1 KB
// reserved per CTA) -- split between the K groups in proportion to their
// cost, each with at least two units per warp; max_seg = the most CTAs any
// column block of the layer is split over.
static GemvPlan gemv_plan(const int64_t *k, const int64_t *n, const int *K, int count, int64_t m, int sms)
{
    GemvPlan pl;
    const int MG = gemv_mg(m);
    pl.ngroups = 0;
    int np = 0, max_sb = 0;
    for (int kk = 1; kk <= 8; ++kk) {
        GemvGroup gr;
        gr.K = kk;
        gr.l_begin = np;
        gr.units = 0;
        int cbn = 0;
        for (int l = 0; l < count; ++l) {
            if (K[l] != kk)
                continue;
            pl.order[np] = l;
            pl.unit_begin[np] = gr.units;
            pl.cb_begin[np] = cbn;
            gr.units += (k[l] / 16) * (n[l] / 128);
            cbn += (int)(n[l] / 128);
            ++np;
        }
        gr.l_end = np;
        if (gr.l_end > gr.l_begin) {
            pl.grp[pl.ngroups++] = gr;
            const int sb = gemv_stage_bytes(kk, MG);
            max_sb = sb > max_sb ? sb : max_sb;
        }
    }
    pl.smem = 128 + kGemvWarps * (int)m * 128 * 4 + kGemvWarps * kGemvDepth * max_sb;
    int64_t occ = m <= 8 ? 2 : 1;
    const int64_t occ_smem = (228 * 1024) / (pl.smem + 1024);
    if (occ_smem < occ)
        occ = occ_smem > 0 ? occ_smem : 1;
    const int64_t G = occ * (int64_t)sms;

    // CTAs per group: proportional to cost (largest remainder), at least 1,
    // at most units / 16 (two units per warp)
    int64_t cost_sum = 0;
    for (int q = 0; q < pl.ngroups; ++q)
        cost_sum += pl.grp[q].units * gemv_unit_cost(pl.grp[q].K);
    int64_t given = 0;
    int64_t rem[8];
    for (int q = 0; q < pl.ngroups; ++q) {
        const int64_t num = G * pl.grp[q].units * gemv_unit_cost(pl.grp[q].K);
        int64_t gq = num / cost_sum;
        rem[q] = num - gq * cost_sum;
        const int64_t cap = pl.grp[q].units / (2 * kGemvWarps) > 0 ? pl.grp[q].units / (2 * kGemvWarps) : 1;
        gq = gq < 1 ? 1 : (gq > cap ? cap : gq);
        pl.grp[q].ctas = (int)gq;
        given += gq;
    }
    while (given < G) {  // hand out what rounding left, largest remainder first
        int best = -1;
        for (int q = 0; q < pl.ngroups; ++q) {
            const int64_t cap = pl.grp[q].units / (2 * kGemvWarps);
            if (pl.grp[q].ctas < cap && (best < 0 || rem[q] > rem[best]))
                best = q;
        }
        if (best < 0)
            break;
        ++pl.grp[best].ctas;
        rem[best] = -1;
        ++given;
        bool any = false;
        for (int q = 0; q < pl.ngroups; ++q)
            any = any || rem[q] >= 0;
        if (!any)
            for (int q = 0; q < pl.ngroups; ++q)
                rem[q] = 0;
    }
    if (count == 1) {
        // A whole number of CTAs per column block aligns the CTA ranges with
        // the column blocks, so no CTA straddles two (one segment end instead
        // of two, each about as costly as 8 units).  Take it when the busiest
        // SM's modelled work (units + 8 per segment end) is lower.
        GemvGroup &gr = pl.grp[0];
        const int64_t Gq = gr.ctas;
        const int64_t ncb = n[0] / 128;
        const int64_t s_blk = Gq / ncb;
        if (s_blk >= 1 && s_blk * ncb != Gq) {
            auto cost = [&](int64_t gg, int64_t segs) {
                const int64_t per_sm = (gg + sms - 1) / sms;
                return (gr.units + gg - 1) / gg * per_sm + 8 * segs * per_sm;
            };
            if (cost(s_blk * ncb, 1) < cost(Gq, 2))
                gr.ctas = (int)(s_blk * ncb);
        }
    }
    int cta = 0;
    for (int q = 0; q < pl.ngroups; ++q) {
        pl.grp[q].cta_begin = cta;
        cta += pl.grp[q].ctas;
    }
    pl.ctas = cta;

    // Input rotation.  Per CTA, inside the one launch, when every CTA's range
    // spans at most two column blocks (its length is at most the smallest
    // tile-row count of its group) and touches few enough 128-channel blocks
    // that each warp rotates at most two (range / 8 + 2 blocks, m rows each);
    // otherwise by the rotation kernel, launched just before.
    pl.rot_local = 1;
    for (int q = 0; q < pl.ngroups; ++q) {
        const GemvGroup &gr = pl.grp[q];
        const int64_t range = (gr.units + gr.ctas - 1) / gr.ctas;
        int64_t tr_min = INT64_MAX;
        for (int i = gr.l_begin; i < gr.l_end; ++i)
            tr_min = k[pl.order[i]] / 16 < tr_min ? k[pl.order[i]] / 16 : tr_min;
        if (range > tr_min || (range / 8 + 2) * m > 2 * kGemvWarps)
            pl.rot_local = 0;
    }

    size_t off = 256;
    for (int l = 0; l < count; ++l) {
        pl.counters[l] = off;
        off += (size_t)(n[l] / 128) * 4;
    }
    off = (off + 255) / 256 * 256;
    pl.sync_bytes = off;
    off = off > kGemvSyncArea ? off : kGemvSyncArea;
    for (int q = 0; q < pl.ngroups; ++q) {
        const GemvGroup &gr = pl.grp[q];
        for (int i = gr.l_begin; i < gr.l_end; ++i) {
            const int l = pl.order[i];
            const int64_t TR = k[l] / 16, ncb = n[l] / 128;
            int64_t max_seg = 1;
            for (int64_t c = 0; c < ncb; ++c) {
                const int64_t b0 = pl.unit_begin[i] + c * TR;
                const int64_t sg =
                    gemv_owner_cta(b0 + TR - 1, gr.units, gr.ctas) - gemv_owner_cta(b0, gr.units, gr.ctas) + 1;
                max_seg = sg > max_seg ? sg : max_seg;
            }
            pl.max_seg[i] = (int)max_seg;
        }
    }
    for (int l = 0; l < count; ++l) {
        pl.acts[l] = off;
        off += ((size_t)(k[l] / 16) * MG * kGemvActBlock + 255) / 256 * 256;
    }
    for (int i = 0; i < count; ++i) {
        const int l = pl.order[i];
        pl.partials[l] = off;
        off += ((size_t)(n[l] / 128) * (size_t)pl.max_seg[i] * (size_t)m * 128 * 4 + 255) / 256 * 256;
    }
    pl.total = off;
    return pl;
}

// Bytes at the start of a one-layer workspace that must be zero when a call
// starts (status word and arrival counters).
size_t gemv_sync_bytes(int64_t m, int64_t k, int64_t n, int K, int sms)
{
    return gemv_plan(&k, &n, &K, 1, m, sms).sync_bytes;
}

size_t gemv_workspace_bytes(int64_t m, int64_t k, int64_t n, int sms)
{
    size_t most = 0;
    for (int K = 1; K <= 8; ++K) {
        const size_t b = gemv_plan(&k, &n, &K, 1, m, sms).total;
        most = b > most ? b : most;
    }
    return most;
}

// The rotation kernel, for launches whose CTA ranges are long: one warp per
// (layer, batch row, 128-channel block) job, layer by layer.
struct GemvRotLayer {
    const __half *x, *suh;
    unsigned char *acts;
    int k;
    int64_t job_begin;  // first job of this layer
};

struct GemvRotParams {
    GemvRotLayer L[kGemvMaxLayers];
    int count, m;
    int64_t jobs;
};

__global__ void __launch_bounds__(256) gemv_rotate_kernel(const GemvRotParams rp)
{
    grid_dep_wait();    // x may come from the preceding kernel
    grid_dep_launch();  // the main kernel may start streaming weights meanwhile
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    int l = 0;
    for (int64_t job = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); job < rp.jobs; job += warps) {
        while (l + 1 < rp.count && job >= rp.L[l + 1].job_begin)
            ++l;
        const GemvRotLayer &L = rp.L[l];
        const int nblk = L.k / 128;
        const int64_t lj = job - L.job_begin;
        const int b = (int)(lj / nblk);
        rotate_block(L.x, L.suh, L.acts, L.k, rp.m, b, (int)(lj - (int64_t)b * nblk), lane);
    }
}

static exl3_status launch_rotation(const exl3_linear *const *layers, unsigned char *const *acts, int count,
                                   int64_t m, cudaStream_t stream)
{
    const int sms = num_sms();
    GemvRotParams rp;
    rp.count = count;
    rp.m = (int)m;
    int64_t jobs = 0;
    for (int l = 0; l < count; ++l) {
        rp.L[l].x = (const __half *)layers[l]->x;
        rp.L[l].suh = (const __half *)layers[l]->suh;
        rp.L[l].acts = acts[l];
        rp.L[l].k = (int)layers[l]->k;
        rp.L[l].job_begin = jobs;
        jobs += m * (layers[l]->k / 128);
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

// One launch over up to kGemvMaxLayers layers (two when the rotation runs as
// its own kernel), with the workspace region `ws` laid out by gemv_plan.
static exl3_status run_gemv_launch(const exl3_linear *const *layers, int count, int64_t m, unsigned char *ws,
                                   size_t ws_bytes, cudaStream_t stream)
{
    const int sms = num_sms();
    int64_t k[kGemvMaxLayers], n[kGemvMaxLayers];
    int K[kGemvMaxLayers];
    for (int l = 0; l < count; ++l) {
        k[l] = layers[l]->k;
        n[l] = layers[l]->n;
        K[l] = layers[l]->K;
    }
    const GemvPlan pl = gemv_plan(k, n, K, count, m, sms);
    if (!ws || !aligned16(ws) || ws_bytes < pl.total)
        return EXL3_ERR_WORKSPACE;
    if (!pl.rot_local) {
        unsigned char *acts[kGemvMaxLayers];
        for (int l = 0; l < count; ++l)
            acts[l] = ws + pl.acts[l];
        const exl3_status rs = launch_rotation(layers, acts, count, m, stream);
        if (rs != EXL3_OK)
            return rs;
    }

    GemvParams p;
    p.m = (int)m;
    p.rot_local = pl.rot_local;
    p.ngroups = pl.ngroups;
    for (int q = 0; q < pl.ngroups; ++q)
        p.grp[q] = pl.grp[q];
    p.cb = codebook_constants();
    for (int i = 0; i < 8; ++i)
        p.mu.pow2[i] = 1u << i;
    for (int i = 0; i < count; ++i) {
        const int l = pl.order[i];
        GemvLayer &L = p.L[i];
        L.trellis = reinterpret_cast<const unsigned char *>(layers[l]->trellis);
        L.x = (const __half *)layers[l]->x;
        L.suh = (const __half *)layers[l]->suh;
        L.svh = (const __half *)layers[l]->svh;
        L.y = (__half *)layers[l]->y;
        L.acts = ws + pl.acts[l];
        L.partials = reinterpret_cast<float *>(ws + pl.partials[l]);
        L.counters = reinterpret_cast<uint32_t *>(ws + pl.counters[l]);
        L.unit_begin = pl.unit_begin[i];
        L.n = (int)n[l];
        L.tr_count = (int)(k[l] / 16);
        L.max_seg = pl.max_seg[i];
        L.cb_begin = pl.cb_begin[i];
    }
    auto kern = m <= 8 ? gemv_kernel<1> : gemv_kernel<2>;
    if (pl.smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem) != cudaSuccess)
        return EXL3_ERR_CUDA;
    if (launch_kernel(kern, dim3((unsigned)pl.ctas), dim3(kGemvThreads), (size_t)pl.smem, stream, p) !=
        cudaSuccess)
        return EXL3_ERR_CUDA;
    return launch_status();
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
    return run_gemv_launch(&one, 1, m, (unsigned char *)workspace, workspace_bytes, stream);
}

// The layers of a multi call in launches of at most kGemvMaxLayers, in call
// order; calls f(layers, count, workspace offset, bytes) per launch.
template <typename F>
static exl3_status for_each_gemv_launch(const exl3_linear *layers, int count, int64_t m, F &&f)
{
    const int sms = num_sms();
    size_t off = 0;
    for (int first = 0; first < count; first += kGemvMaxLayers) {
        const int cnt = count - first < kGemvMaxLayers ? count - first : kGemvMaxLayers;
        const exl3_linear *grp[kGemvMaxLayers];
        int64_t k[kGemvMaxLayers], n[kGemvMaxLayers];
        int K[kGemvMaxLayers];
        for (int l = 0; l < cnt; ++l) {
            grp[l] = &layers[first + l];
            k[l] = grp[l]->k;
            n[l] = grp[l]->n;
            K[l] = grp[l]->K;
        }
        const size_t bytes = gemv_plan(k, n, K, cnt, m, sms).total;
        const exl3_status st = f(grp, cnt, off, bytes);
        if (st != EXL3_OK)
            return st;
        off += (bytes + 255) / 256 * 256;
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
    for_each_gemv_launch(layers, count, m, [&](const exl3_linear *const *, int, size_t off, size_t bytes) {
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
    return for_each_gemv_launch(layers, count, m,
                                [&](const exl3_linear *const *grp, int cnt, size_t off, size_t bytes) {
                                    return run_gemv_launch(grp, cnt, m, ws + off, bytes, (cudaStream_t)stream);
                                });
}

// ------------------------------------------------ no-allocation variant ---
//
// exl3_gemv_noalloc runs the GEMV above with its scratch (split-k partials
// and arrival counters) in a fixed array
// compiled into the library, for callers that must not allocate device
// memory themselves.  The array is a file-scope __device__ symbol: every GPU
// that loads the library holds its kNoAllocScratchBytes until the process
// exits.  In host code the symbol's name is only a host-side stand-in, so the
// device address is looked up with cudaGetSymbolAddress (with the device
// current) and cached per device and context.

#include <mutex>

namespace exl3 {

constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
struct NoAllocCache {
    void *ptr;
    void *ctx;  // the context (CUcontext) the address belongs to
};
static NoAllocCache g_noalloc[kMaxDevices];
static std::mutex g_noalloc_mutex;

// The driver's cuCtxGetCurrent, fetched through the runtime (the library
// links only the runtime).  Returns null when it is unavailable.
static void *current_context()
{
    typedef int (*GetCurrent)(void **);
    static GetCurrent fn = []() -> GetCurrent {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<GetCurrent>(f);
    }();
    void *ctx = nullptr;
    if (!fn || fn(&ctx) != 0)
        return nullptr;
    return ctx;
}

// Device address of this device's scratch array.  It is looked up again
// whenever the current context differs from the one it was looked up in (a
// cudaDeviceReset makes a new primary context, and the old address with it
// invalid).  Inside a stream capture the lookup is refused with
// EXL3_ERR_UNSUPPORTED: make a first call on the device outside capture.
static exl3_status noalloc_scratch(cudaStream_t stream, void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return EXL3_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices)
        return EXL3_ERR_UNSUPPORTED;
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc[dev].ptr || g_noalloc[dev].ctx != ctx) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess)
            return EXL3_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone)
            return EXL3_ERR_UNSUPPORTED;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return EXL3_ERR_CUDA;
        ctx = current_context();
        g_noalloc[dev].ptr = p;
        g_noalloc[dev].ctx = ctx;
    }
    *out = g_noalloc[dev].ptr;
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
    const exl3_status sst = noalloc_scratch((cudaStream_t)stream, &scratch);
    if (sst != EXL3_OK)
        return sst;
    // the array keeps whatever the last call left: the status word and the
    // arrival counters must start at zero (the kernel re-arms the counters,
    // but a call that never finished could have left them set), so clear
    // them on the caller's stream
    if (cudaMemsetAsync(scratch, 0, gemv_sync_bytes(m, k, n, K, num_sms()), (cudaStream_t)stream) != cudaSuccess)
        return EXL3_ERR_CUDA;
    return run_gemv(x, trellis, suh, svh, y, m, k, n, K, scratch, kNoAllocScratchBytes,
                    (cudaStream_t)stream);
}
