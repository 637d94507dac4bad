// ldlq.cu -- exl3_udu and exl3_ldlq: the Hessian-aware rounding that feeds the
// trellis encoder (EXL3 GEMM kernel article, section Viterbi编码内核剖析:
// ldlq() performs a block-wise LDLQ decomposition of the layer before
// quantize_tiles() runs the trellis kernel on its 16x16 tiles).
//
// Readings (the pages name the step, not its algebra): the proxy loss of a
// quantised layer is tr(E^T H E), E = W_hat - W, W the k x n weight (rows =
// input channels), H the k x k input Hessian.  H = U D U^T with U unit
// block-upper-triangular and D block-diagonal, 16 x 16 blocks (one per tile
// row).  Tile rows are quantised in order: row block b's target is
//     T_b = W_b - sum_{c<b} U_{c,b}^T (W_hat_c - W_c),
// rounded to fp32 and encoded; then tr(E^T H E) = sum_b tr(F_b^T D_b F_b)
// with F_b = W_hat_b - T_b.  The factorisation and the feedback run in fp64;
// the encoder decides in fp32 on the fp32 targets.
//
// B200 mapping: both are sequences of small steps, one per 16-row block.
//   * exl3_udu, bottom-up over blocks b: one CTA inverts D_b (Gauss-Jordan,
//     256 threads, fp64), a grid forms the panel U_{:,b} = A_{:,b} D_b^-1, and
//     a tiled grid applies the rank-16 update A_{aa'} -= U_ab A_{a'b}^T to the
//     blocks on or above the diagonal of the leading 16b x 16b part (64 x 64
//     fp64 output tiles, 16-deep operands staged in shared memory); the panel
//     then replaces column block b.  The strict lower blocks are zeroed.
//   * exl3_ldlq, forward over blocks b: a tiled grid forms the 16 x n target
//     (fp64 sums, 64 columns per CTA, U and E staged in shared memory, fp32
//     result); exl3_encode writes tile row b of the trellis; exl3_decode_tiles
//     decodes it; one more grid stores E_b = W_hat_b - W_b (fp64) for the
//     following blocks (and W_hat_b if asked).
#include <cuda_fp16.h>

#include "exl3_host.h"

namespace exl3 {

constexpr int kUduB = 16;

// D_b^-1 by Gauss-Jordan without pivoting (D_b is symmetric positive
// definite).  One CTA of 256 threads, element (r, c) per thread.
__global__ void __launch_bounds__(256) udu_dinv_kernel(const double *a, int64_t k, int b, double *dinv)
{
    __shared__ double m[kUduB][2 * kUduB];
    const int t = threadIdx.x, r = t >> 4, c = t & 15;
    const int64_t o = (int64_t)b * kUduB;
    m[r][c] = a[(o + r) * k + o + c];
    m[r][kUduB + c] = r == c ? 1.0 : 0.0;
    __syncthreads();
    for (int p = 0; p < kUduB; ++p) {
        const double piv = m[p][p];
        const double f = m[r][p];
        const double left = m[p][c], right = m[p][kUduB + c];
        __syncthreads();
        if (r == p) {
            m[r][c] = left / piv;
            m[r][kUduB + c] = right / piv;
        } else {
            m[r][c] -= f * (left / piv);
            m[r][kUduB + c] -= f * (right / piv);
        }
        __syncthreads();
    }
    dinv[r * kUduB + c] = m[r][kUduB + c];
}

// Panel: p[row][j] = sum_i a[row][16b + i] dinv[i][j] for row < 16b.
__global__ void __launch_bounds__(256) udu_panel_kernel(const double *a, int64_t k, int b, const double *dinv,
                                                        double *p)
{
    __shared__ double di[kUduB][kUduB];
    const int t = threadIdx.x;
    di[t >> 4][t & 15] = dinv[t];
    __syncthreads();
    const int64_t rows = (int64_t)b * kUduB;
    const int64_t idx = (int64_t)blockIdx.x * 256 + t;
    if (idx >= rows * kUduB)
        return;
    const int64_t row = idx >> 4;
    const int j = (int)(idx & 15);
    const double *ar = a + row * k + (int64_t)b * kUduB;
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < kUduB; ++i)
        s += ar[i] * di[i][j];
    p[idx] = s;
}

// Rank-16 update of the leading 16b x 16b part, on and above the block
// diagonal: a[r][c] -= sum_i p[r][i] a[c][16b + i].  64 x 64 output tiles
// (CTA tiles strictly below the diagonal are skipped), 4 x 4 per thread.
__global__ void __launch_bounds__(256) udu_update_kernel(double *a, int64_t k, int b, const double *p)
{
    const int64_t n0 = (int64_t)b * kUduB;  // size of the leading part
    const int64_t tr = blockIdx.y, tc = blockIdx.x;
    if (tr > tc)
        return;
    __shared__ double ps[64][kUduB + 1];
    __shared__ double qs[64][kUduB + 1];
    const int t = threadIdx.x;
    for (int e = t; e < 64 * kUduB; e += 256) {
        const int rr = e >> 4, ii = e & 15;
        const int64_t gr = tr * 64 + rr, gc = tc * 64 + rr;
        ps[rr][ii] = gr < n0 ? p[gr * kUduB + ii] : 0.0;
        qs[rr][ii] = gc < n0 ? a[gc * k + n0 + ii] : 0.0;
    }
    __syncthreads();
    const int ty = t >> 4, tx = t & 15;
    double acc[4][4] = {};
#pragma unroll
    for (int i = 0; i < kUduB; ++i) {
        double pv[4], qv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            pv[u] = ps[ty * 4 + u][i];
            qv[u] = qs[tx * 4 + u][i];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v)
                acc[u][v] += pv[u] * qv[v];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t gr = tr * 64 + ty * 4 + u;
        if (gr >= n0)
            continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int64_t gc = tc * 64 + tx * 4 + v;
            if (gc < n0 && (gr >> 4) <= (gc >> 4))
                a[gr * k + gc] -= acc[u][v];
        }
    }
}

// Column block b (rows < 16b) takes the panel U_{:,b}.
__global__ void __launch_bounds__(256) udu_store_kernel(double *a, int64_t k, int b, const double *p)
{
    const int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (idx >= (int64_t)b * kUduB * kUduB)
        return;
    a[(idx >> 4) * k + (int64_t)b * kUduB + (idx & 15)] = p[idx];
}

// Strict lower blocks to zero.
__global__ void __launch_bounds__(256) udu_lower_kernel(double *a, int64_t k)
{
    const int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (idx >= k * k)
        return;
    const int64_t r = idx / k, c = idx - r * k;
    if ((r >> 4) > (c >> 4))
        a[idx] = 0.0;
}

static size_t udu_scratch_bytes(int64_t k)
{
    return 256 + (size_t)kUduB * kUduB * 8 + (size_t)k * kUduB * 8;
}

// Factorises ud (k x k fp64, holding H) in place; scratch: Dinv then the panel.
static exl3_status run_udu(double *ud, int64_t k, unsigned char *scratch, cudaStream_t s)
{
    double *dinv = reinterpret_cast<double *>(scratch + 256);
    double *panel = dinv + kUduB * kUduB;
    const int nb = (int)(k / kUduB);
    const unsigned tiles = (unsigned)((k + 63) / 64);
    for (int b = nb - 1; b >= 0; --b) {
        udu_dinv_kernel<<<1, 256, 0, s>>>(ud, k, b, dinv);
        if (b > 0) {
            const int64_t outs = (int64_t)b * kUduB * kUduB;
            udu_panel_kernel<<<(unsigned)((outs + 255) / 256), 256, 0, s>>>(ud, k, b, dinv, panel);
            const unsigned tb = (unsigned)(((int64_t)b * kUduB + 63) / 64);
            udu_update_kernel<<<dim3(tb, tb), 256, 0, s>>>(ud, k, b, panel);
            udu_store_kernel<<<(unsigned)((outs + 255) / 256), 256, 0, s>>>(ud, k, b, panel);
        }
    }
    (void)tiles;
    udu_lower_kernel<<<(unsigned)((k * k + 255) / 256), 256, 0, s>>>(ud, k);
    return cudaGetLastError() == cudaSuccess ? EXL3_OK : EXL3_ERR_CUDA;
}

// Target of row block b: t[r][j] = w[16b + r][j] - sum_{i < 16b} u[i][16b + r]
// e[i][j], fp64 sums, fp32 result.  CTA = 64 columns x 16 rows, 256 threads,
// 4 rows of one column per thread; i in chunks of 64 staged in shared memory.
__global__ void __launch_bounds__(256) ldlq_target_kernel(const float *w, const double *u, const double *e,
                                                          int64_t k, int64_t n, int b, float *t)
{
    __shared__ double us[64][kUduB + 1];
    __shared__ double es[64][64 + 1];
    const int tid = threadIdx.x;
    const int col = tid & 63, rq = tid >> 6;  // rows 4rq .. 4rq+3
    const int64_t j0 = (int64_t)blockIdx.x * 64;
    const int64_t r0 = (int64_t)b * kUduB;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int64_t i0 = 0; i0 < r0; i0 += 64) {
        for (int x = tid; x < 64 * kUduB; x += 256) {
            const int ii = x >> 4, rr = x & 15;
            us[ii][rr] = i0 + ii < r0 ? u[(i0 + ii) * k + r0 + rr] : 0.0;
        }
        for (int x = tid; x < 64 * 64; x += 256) {
            const int ii = x >> 6, cc = x & 63;
            es[ii][cc] = (i0 + ii < r0 && j0 + cc < n) ? e[(i0 + ii) * n + j0 + cc] : 0.0;
        }
        __syncthreads();
#pragma unroll 8
        for (int ii = 0; ii < 64; ++ii) {
            const double ev = es[ii][col];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                acc[q] += us[ii][4 * rq + q] * ev;
        }
        __syncthreads();
    }
    const int64_t j = j0 + col;
    if (j < n)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t r = 4 * rq + q;
            t[r * n + j] = (float)((double)w[(r0 + r) * n + j] - acc[q]);
        }
}

// E_b = W_hat_b - W_b (fp64) from the decoded fp16 block; W_hat_b to w_hat if given.
__global__ void __launch_bounds__(256) ldlq_error_kernel(const __half *dec, const float *w, double *e, float *w_hat,
                                                         int64_t n, int b)
{
    const int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (idx >= (int64_t)kUduB * n)
        return;
    const int64_t g = (int64_t)b * kUduB * n + idx;
    const float v = __half2float(dec[idx]);
    e[g] = (double)v - (double)w[g];
    if (w_hat)
        w_hat[g] = v;
}

// Workspace of exl3_ldlq: [0, 256) header; the factor (k x k fp64); the
// factorisation scratch; the errors E (k x n fp64); the block target (16 x n
// fp32); the decoded block (16 x n fp16); the encoder's workspace for 16 x n.
struct LdlqLayout {
    size_t ud, scratch, err, target, dec, enc, enc_bytes, total;
};

static LdlqLayout ldlq_layout(int64_t k, int64_t n, int K)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    LdlqLayout l;
    l.ud = 256;
    l.scratch = up(l.ud + (size_t)k * k * 8);
    l.err = up(l.scratch + udu_scratch_bytes(k));
    l.target = up(l.err + (size_t)k * n * 8);
    l.dec = up(l.target + (size_t)kUduB * n * 4);
    l.enc = up(l.dec + (size_t)kUduB * n * 2);
    l.enc_bytes = exl3_encode_workspace_size(kUduB, n, K);
    l.total = up(l.enc + l.enc_bytes);
    return l;
}

static bool ldlq_shape_ok(int64_t k, int64_t n)
{
    return k >= 16 && n >= 16 && k % 16 == 0 && n % 16 == 0 && k <= ((int64_t)1 << 16) &&
           n <= ((int64_t)1 << 20);
}

}  // namespace exl3

extern "C" size_t exl3_udu_workspace_size(int64_t k)
{
    if (k < 16 || k % 16 || k > ((int64_t)1 << 16))
        return 0;
    return exl3::udu_scratch_bytes(k);
}

extern "C" exl3_status exl3_udu(const double *h, double *ud, int64_t k, void *workspace, size_t workspace_bytes,
                                void *stream)
{
    using namespace exl3;
    if (!h || !ud || !aligned16(h) || !aligned16(ud) || k < 16 || k % 16 || k > ((int64_t)1 << 16))
        return EXL3_ERR_INVALID_ARG;
    if (h != ud && ranges_overlap(h, (size_t)(k * k * 8), ud, (size_t)(k * k * 8)))
        return EXL3_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || workspace_bytes < udu_scratch_bytes(k))
        return EXL3_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    if (h != ud && cudaMemcpyAsync(ud, h, (size_t)(k * k * 8), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return EXL3_ERR_CUDA;
    return run_udu(ud, k, (unsigned char *)workspace, s);
}

extern "C" size_t exl3_ldlq_workspace_size(int64_t k, int64_t n, int K)
{
    if (!exl3::ldlq_shape_ok(k, n) || K < 1 || K > 8)
        return 0;
    return exl3::ldlq_layout(k, n, K).total;
}

extern "C" exl3_status exl3_ldlq(const float *w, const double *h, uint16_t *trellis, float *w_hat, int64_t k,
                                 int64_t n, int K, void *workspace, size_t workspace_bytes, void *stream)
{
    using namespace exl3;
    if (!w || !h || !trellis || !aligned16(w) || !aligned16(h) || !aligned16(trellis) ||
        (w_hat && !aligned16(w_hat)))
        return EXL3_ERR_INVALID_ARG;
    if (!ldlq_shape_ok(k, n) || K < 1 || K > 8)
        return EXL3_ERR_INVALID_ARG;
    if (ranges_overlap(w, (size_t)(k * n * 4), trellis, (size_t)(k * n * K / 8)) ||
        (w_hat && (ranges_overlap(w_hat, (size_t)(k * n * 4), trellis, (size_t)(k * n * K / 8)) ||
                   ranges_overlap(w_hat, (size_t)(k * n * 4), w, (size_t)(k * n * 4)))))
        return EXL3_ERR_INVALID_ARG;
    const LdlqLayout lay = ldlq_layout(k, n, K);
    if (!workspace || !aligned16(workspace) || workspace_bytes < lay.total)
        return EXL3_ERR_WORKSPACE;
    unsigned char *ws = (unsigned char *)workspace;
    cudaStream_t s = (cudaStream_t)stream;
    double *ud = reinterpret_cast<double *>(ws + lay.ud);
    double *err = reinterpret_cast<double *>(ws + lay.err);
    float *target = reinterpret_cast<float *>(ws + lay.target);
    __half *dec = reinterpret_cast<__half *>(ws + lay.dec);
    if (cudaMemcpyAsync(ud, h, (size_t)(k * k * 8), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return EXL3_ERR_CUDA;
    exl3_status st = run_udu(ud, k, ws + lay.scratch, s);
    if (st != EXL3_OK)
        return st;
    const int64_t tn = n / 16;
    for (int b = 0; b < (int)(k / kUduB); ++b) {
        ldlq_target_kernel<<<(unsigned)((n + 63) / 64), 256, 0, s>>>(w, ud, err, k, n, b, target);
        if (cudaGetLastError() != cudaSuccess)
            return EXL3_ERR_CUDA;
        uint16_t *row = trellis + (int64_t)b * tn * 16 * K;
        st = exl3_encode(target, row, nullptr, kUduB, n, K, ws + lay.enc, lay.enc_bytes, stream);
        if (st != EXL3_OK)
            return st;
        st = exl3_decode_tiles(row, dec, kUduB, n, K, stream);
        if (st != EXL3_OK)
            return st;
        ldlq_error_kernel<<<(unsigned)((kUduB * n + 255) / 256), 256, 0, s>>>(dec, w, err, w_hat, n, b);
        if (cudaGetLastError() != cudaSuccess)
            return EXL3_ERR_CUDA;
    }
    return EXL3_OK;
}
