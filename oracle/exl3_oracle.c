/*
 * exl3_oracle.c -- plain, slow, fp64 CPU oracle for the EXL3 trellis-decoded
 * matmul.  TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and
 * the bench's CPU-baseline leg call it; the product path never does.  It shares
 * no code, header, table or constant generator with the CUDA library.
 *
 * What it computes (each function names the passage it follows; "EXL3 GEMM
 * kernel article" is the page "ExLlamaV3推理快的秘密: EXL3 GEMM内核与融合Viterbi
 * 编码CUDA实现剖析", "ExLlamaV3 overview" is "为什么ExLlamaV3值得关注"):
 *
 *   - fp16 bit pattern -> double, double -> fp16 round-to-nearest-even,
 *     written from the IEEE 754 binary16 definition (no compiler half type).
 *   - the procedural codebook: state -> one integer multiply-add, one
 *     mask/xor, two fp16 halves summed and rounded to fp16
 *     (EXL3 GEMM kernel article, sections "先看结论" and "GEMM内核": "one
 *     integer multiply plus one lop3 turns an index into a half, no table").
 *   - the tail-biting bitshift trellis state of every weight of a 16x16 tile
 *     (EXL3 GEMM kernel article, section "Viterbi编码内核剖析": 16x16 tiles,
 *     tail-biting so the codeword's head and tail agree; ExLlamaV3 overview:
 *     "simplified QTIP variant, tail-biting trellis, K = 1..8 bits").
 *   - the 128-point Sylvester Hadamard rotation, blockwise, 1/sqrt(128)
 *     normalised (EXL3 GEMM kernel article, section "GEMM内核": the kernel
 *     rotates the input A with a 128-point Hadamard before the matmul).
 *   - the linear layer y = x . W_hat with both rotations, in fp64.
 *   - the tail-biting trellis encoder: for each 16x16 tile, the Viterbi
 *     search for the bit string whose decoded weights are closest (squared
 *     error) to the tile's target values (EXL3 GEMM kernel article, section
 *     "Viterbi编码内核剖析"; readings at oracle_encode_seq).
 *
 * Readings of points the pages leave open (the pages give no bit order, tile
 * layout or normalisation):
 *   - trellis layout [k/16][n/16][16*K] uint16; tile (tk, tn) covers
 *     W[16tk + r][16tn + c], weight index i = 16 r + c (row-major, r along the
 *     input channels k, c along the output channels n);
 *   - the tile's 16*K words form one big-endian bit string: bit position p is
 *     bit 15 - (p mod 16) of word p / 16;
 *   - weight i's state is the 16 positions [iK + K - 16, iK + K) taken modulo
 *     256*K, the earliest position as the most significant bit (so weight 0
 *     reads the stream's last 16 - K bits: the tail-biting wrap);
 *   - the two codebook halves are bit patterns reinterpreted as fp16 (not
 *     integer conversions); their sum is rounded to fp16 nearest-even;
 *   - H[i][j] = (-1)^popcount(i & j); x' = H (x .* suh) / sqrt(128) per
 *     128-channel block; y = svh .* (H y' / sqrt(128)) per block;
 *   - everything after decoding is kept in fp64 (no fp16 rounding of x' or y').
 *
 * Build: gcc -O2 -fPIC -shared [-fopenmp] exl3_oracle.c -o liboracle.so -lm
 * (the builder next to this file does it).  OpenMP, when present, only splits
 * oracle_linear over independent 128-column output blocks; every block is
 * computed by the same single-threaded loops.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- fp16 -- */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double mag;
    if (e == 0)
        mag = ldexp((double)f, -24); /* subnormal: f * 2^-24 */
    else if (e == 31)
        mag = f ? NAN : INFINITY;
    else
        mag = ldexp(1.0 + (double)f / 1024.0, e - 15);
    return sign ? -mag : mag;
}

/* Round-to-nearest-even of a double to binary16 (overflow -> inf). */
uint16_t oracle_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x))
        return 0x7e00;
    if (a == 0.0)
        return sign;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: units of 2^-24, ties to even (default FP mode) */
        double q = nearbyint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)q); /* q == 1024 is the smallest normal */
    }
    int E;
    frexp(a, &E);             /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;            /* a in [2^e, 2^(e+1)) */
    double m = nearbyint((ldexp(a, -e) - 1.0) * 1024.0);
    if (m >= 1024.0) {
        m = 0.0;
        e += 1;
    }
    if (e + 15 >= 31)
        return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)m);
}

/* ------------------------------------------------------------ codebook -- */

/* state (16 bits) -> fp16 weight bits.  One multiply-add modulo 2^32, one
 * mask and xor, then the upper and lower 16-bit halves are read as fp16 and
 * added; the sum is rounded to fp16.  Constants: multiplier 89226354, addend
 * 64248484, mask 0x8fff8fff, xor 0x3b603b60. */
uint16_t oracle_codebook(uint16_t state)
{
    uint32_t v = (uint32_t)state * 89226354u + 64248484u;
    v = (v & 0x8fff8fffu) ^ 0x3b603b60u;
    double hi = oracle_half_to_double((uint16_t)(v >> 16));
    double lo = oracle_half_to_double((uint16_t)(v & 0xffffu));
    return oracle_double_to_half(hi + lo); /* the fp64 sum of two halves is exact */
}

/* ------------------------------------------------------------- trellis -- */

/* Bit at big-endian position p of a tile's word string. */
static int stream_bit(const uint16_t *words, long p)
{
    return (words[p / 16] >> (15 - (p % 16))) & 1;
}

/* State of weight i (0..255) of one tile: the 16 positions ending at the end
 * of weight i's K bits, cyclic over the tile's 256*K bits. */
uint16_t oracle_state(const uint16_t *tile_words, int K, int i)
{
    long nbits = 256L * K;
    long first = (long)i * K + K - 16;
    unsigned s = 0;
    for (int j = 0; j < 16; ++j) {
        long p = ((first + j) % nbits + nbits) % nbits;
        s = (s << 1) | (unsigned)stream_bit(tile_words, p);
    }
    return (uint16_t)s;
}

/* All 256 states of every tile: out[(tk*(n/16) + tn)*256 + i]. */
void oracle_states(const uint16_t *trellis, int64_t k, int64_t n, int K, uint16_t *out)
{
    int64_t tiles = (k / 16) * (n / 16);
    for (int64_t t = 0; t < tiles; ++t)
        for (int i = 0; i < 256; ++i)
            out[t * 256 + i] = oracle_state(trellis + t * 16 * K, K, i);
}

/* Decoded weights, k x n row-major fp16 bits. */
void oracle_decode_tiles(const uint16_t *trellis, int64_t k, int64_t n, int K, uint16_t *w)
{
    int64_t tn_count = n / 16;
    for (int64_t tk = 0; tk < k / 16; ++tk)
        for (int64_t tn = 0; tn < tn_count; ++tn) {
            const uint16_t *tile = trellis + (tk * tn_count + tn) * 16 * K;
            for (int i = 0; i < 256; ++i) {
                int r = i / 16, c = i % 16;
                w[(tk * 16 + r) * n + tn * 16 + c] = oracle_codebook(oracle_state(tile, K, i));
            }
        }
}

/* ------------------------------------------------------------- encoder -- */

/* Tail-biting Viterbi encoding of one sequence (EXL3 GEMM kernel article,
 * section "Viterbi编码内核剖析": a 16x16 block of weights is encoded by a
 * Viterbi forward pass over the trellis that keeps the accumulated cost of
 * every path and takes the cheapest; the tail-biting boundary is closed by
 * enumerating start states, so that the codeword's head and tail agree).
 *
 * Generic in the trellis size so that tests can compare it with exhaustive
 * search on a small trellis: T weights, L-bit states (16 for EXL3), K bits
 * per weight (2K <= L), and the value of every state in `cb` (2^L floats;
 * for EXL3 the codebook).  The state of weight i is s_i = ((s_{i-1} << K) |
 * c_i) mod 2^L with c_i the weight's K new bits, and the code is tail-biting:
 * s_{-1} = s_{T-1}.
 *
 * Readings of what the pages leave open:
 *   - the cost of weight i in state s is (target_i - cb[s])^2, formed in fp32
 *     as fmaf(d, d, path cost) with d = target_i - cb[s] rounded to fp32 (the
 *     precision in which the GPU kernel takes the same decisions);
 *   - M_i[m] is the cheapest cost of a path through weight i whose state has
 *     low L-K bits m, i.e. the states that can precede a state whose high
 *     L-K bits are m: M_i[m] = min over h of fmaf(d, d, M_{i-1}[s >> K]) with
 *     s = (h << (L-K)) | m, the smallest h winning ties; h is recorded;
 *   - pass 1 enumerates every start state (M_{-1} = 0 everywhere).  The
 *     cheapest end, o = argmin_m M_{T-1}[m] (smallest m on ties), fixes the
 *     overlap: the low L-K bits of the last state, which a tail-biting code
 *     repeats as the high L-K bits of the first;
 *   - pass 2 closes the loop: M_{-1}[x] = 0 for x == o and +inf otherwise, so
 *     the first state's high bits are o; the path ends in the cheapest state
 *     with low bits o and is traced back through the recorded choices.
 * Outputs: chunks[i] = c_i (the low K bits of s_i), the pass-2 path cost
 * (fp32) and the overlap o.  Returns 0, or -1 if memory runs out. */
int oracle_encode_seq(const float *target, int T, int L, int K, const float *cb, unsigned char *chunks,
                      float *cost, int *overlap)
{
    const long nm = 1L << (L - K), nh = 1L << K;
    float *prev = (float *)malloc(sizeof(float) * nm);
    float *next = (float *)malloc(sizeof(float) * nm);
    unsigned char *choice = (unsigned char *)malloc((size_t)T * (size_t)nm);
    if (!prev || !next || !choice) {
        free(prev);
        free(next);
        free(choice);
        return -1;
    }
    int o = 0;
    for (int pass = 1; pass <= 2; ++pass) {
        for (long m = 0; m < nm; ++m)
            prev[m] = (pass == 1 || m == o) ? 0.0f : INFINITY;
        for (int i = 0; i < T; ++i) {
            for (long m = 0; m < nm; ++m) {
                float best = 0.0f;
                int best_h = 0;
                for (long h = 0; h < nh; ++h) {
                    const long s = (h << (L - K)) | m;
                    const float d = target[i] - cb[s];
                    const float v = fmaf(d, d, prev[s >> K]);
                    if (h == 0 || v < best) {
                        best = v;
                        best_h = (int)h;
                    }
                }
                next[m] = best;
                choice[(size_t)i * (size_t)nm + (size_t)m] = (unsigned char)best_h;
            }
            float *t = prev;
            prev = next;
            next = t;
        }
        if (pass == 1) {
            o = 0;
            for (long m = 1; m < nm; ++m)
                if (prev[m] < prev[o])
                    o = (int)m;
        }
    }
    /* trace back from the cheapest last state with low bits o */
    long s = ((long)choice[(size_t)(T - 1) * (size_t)nm + (size_t)o] << (L - K)) | o;
    chunks[T - 1] = (unsigned char)(s & (nh - 1));
    for (int i = T - 1; i > 0; --i) {
        const long m = s >> K;
        s = ((long)choice[(size_t)(i - 1) * (size_t)nm + (size_t)m] << (L - K)) | m;
        chunks[i - 1] = (unsigned char)(s & (nh - 1));
    }
    *cost = prev[o];
    *overlap = o;
    free(prev);
    free(next);
    free(choice);
    return 0;
}

/* Encodes a k x n fp32 matrix (row-major) into the trellis layout above: each
 * tile's 256 targets in weight order i = 16 r + c go through
 * oracle_encode_seq with L = 16, T = 256 and the codebook's values; chunk c_i
 * fills stream positions [iK, iK + K), most significant bit first.  cost[t]
 * is tile t's squared-error sum (tiles in [k/16][n/16] order).  OpenMP, when
 * present, only splits the independent tiles. */
int oracle_encode(const float *w, int64_t k, int64_t n, int K, uint16_t *trellis, float *cost, int threads)
{
    float *cb = (float *)malloc(sizeof(float) * 65536);
    if (!cb)
        return -1;
    for (long st = 0; st < 65536; ++st)
        cb[st] = (float)oracle_half_to_double(oracle_codebook((uint16_t)st));
    const int64_t tn_count = n / 16, tiles = (k / 16) * tn_count;
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : 1) reduction(| : failed)
#endif
    for (int64_t t = 0; t < tiles; ++t) {
        float target[256];
        unsigned char chunks[256];
        const int64_t tk = t / tn_count, tn = t % tn_count;
        for (int i = 0; i < 256; ++i)
            target[i] = w[(tk * 16 + i / 16) * n + tn * 16 + i % 16];
        int o = 0;
        if (oracle_encode_seq(target, 256, 16, K, cb, chunks, &cost[t], &o) != 0) {
            failed |= 1;
            continue;
        }
        uint16_t *words = trellis + t * 16 * K;
        memset(words, 0, sizeof(uint16_t) * 16 * (size_t)K);
        for (int i = 0; i < 256; ++i)
            for (int j = 0; j < K; ++j) {
                const long p = (long)i * K + j;
                if ((chunks[i] >> (K - 1 - j)) & 1)
                    words[p / 16] |= (uint16_t)(1u << (15 - p % 16));
            }
    }
    (void)threads;
    free(cb);
    return failed ? -1 : 0;
}

/* ------------------------------------------------------------ hadamard -- */

static int hadamard_sign(int i, int j)
{
    return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

/* y[r, 128b + i] = post[128b+i] * (1/sqrt(128)) * sum_j H[i][j] x[r,128b+j] pre[128b+j].
 * x, y: rows x cols doubles (cols % 128 == 0); pre/post may be NULL (= ones). */
void oracle_hadamard(const double *x, double *y, int64_t rows, int64_t cols,
                     const double *pre, const double *post)
{
    const double scale = 1.0 / sqrt(128.0);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 128; ++b)
            for (int i = 0; i < 128; ++i) {
                double acc = 0.0;
                for (int j = 0; j < 128; ++j) {
                    int64_t c = b * 128 + j;
                    double v = x[r * cols + c] * (pre ? pre[c] : 1.0);
                    acc += hadamard_sign(i, j) * v;
                }
                int64_t c = b * 128 + i;
                y[r * cols + c] = acc * scale * (post ? post[c] : 1.0);
            }
}

/* ------------------------------------------------------------- linear -- */

/* y[:, 128*nb0 : 128*nb1] of the EXL3 linear layer, in fp64.
 *   x: m x k fp16 bits, trellis: [k/16][n/16][16K] words, suh: k fp16 bits,
 *   svh: n fp16 bits.  y: m x (128*(nb1-nb0)) doubles, row-major.
 * Steps: x' = H(x .* suh)/sqrt(128) blockwise; y' = x' W_hat for the
 * requested columns (W_hat decoded tile by tile); y = svh .* H(y')/sqrt(128).
 * threads <= 1 runs single-threaded; otherwise the 128-column output blocks
 * are split across that many OpenMP threads (when built with OpenMP). */
void oracle_linear(const uint16_t *x, const uint16_t *trellis, const uint16_t *suh,
                   const uint16_t *svh, int64_t m, int64_t k, int64_t n, int K,
                   int64_t nb0, int64_t nb1, double *y, int threads)
{
    int64_t ncols = (nb1 - nb0) * 128;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(m * k));
    double *xr = (double *)malloc(sizeof(double) * (size_t)(m * k));
    double *sd = (double *)malloc(sizeof(double) * (size_t)k);
    for (int64_t i = 0; i < m * k; ++i)
        xd[i] = oracle_half_to_double(x[i]);
    for (int64_t i = 0; i < k; ++i)
        sd[i] = oracle_half_to_double(suh[i]);
    oracle_hadamard(xd, xr, m, k, sd, NULL);
    int64_t tn_count = n / 16;
    (void)threads;
#ifdef _OPENMP
    int nt = threads > 1 ? threads : 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
#endif
    for (int64_t b = nb0; b < nb1; ++b) {
        double *wblk = (double *)malloc(sizeof(double) * (size_t)(k * 128));
        double *yp = (double *)malloc(sizeof(double) * (size_t)(m * 128));
        double *yo = (double *)malloc(sizeof(double) * (size_t)(m * 128));
        double vh[128];
        /* decode the k x 128 column block of W_hat */
        for (int64_t tk = 0; tk < k / 16; ++tk)
            for (int64_t q = 0; q < 8; ++q) {
                int64_t tn = b * 8 + q;
                const uint16_t *tile = trellis + (tk * tn_count + tn) * 16 * K;
                for (int i = 0; i < 256; ++i) {
                    int r = i / 16, c = i % 16;
                    wblk[(tk * 16 + r) * 128 + q * 16 + c] =
                        oracle_half_to_double(oracle_codebook(oracle_state(tile, K, i)));
                }
            }
        /* y' = x' W_hat (block) */
        for (int64_t r = 0; r < m; ++r)
            for (int c = 0; c < 128; ++c) {
                double acc = 0.0;
                for (int64_t kk = 0; kk < k; ++kk)
                    acc += xr[r * k + kk] * wblk[kk * 128 + c];
                yp[r * 128 + c] = acc;
            }
        for (int c = 0; c < 128; ++c)
            vh[c] = oracle_half_to_double(svh[b * 128 + c]);
        oracle_hadamard(yp, yo, m, 128, NULL, vh);
        for (int64_t r = 0; r < m; ++r)
            memcpy(y + r * ncols + (b - nb0) * 128, yo + r * 128, sizeof(double) * 128);
        free(wblk);
        free(yp);
        free(yo);
    }
    free(xd);
    free(xr);
    free(sd);
}

/* Number of OpenMP threads the library would use for `requested` (1 without OpenMP). */
int oracle_threads_available(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
