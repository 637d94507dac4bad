/*
 * exl3.h -- C ABI of the B200 (sm_100a) EXL3 trellis-decoded matmul library.
 *
 * The operation: y = x . W_hat for fp16 activations x (m x k) and weights W_hat
 * (k x n) that are never stored densely.  W_hat is kept as 16 x 16 tiles, each a
 * K-bit-per-weight tail-biting bitshift trellis (K = 1..8) packed in uint16
 * words, and is decoded on the fly through a procedural codebook.  The product
 * is wrapped in two 128-point Hadamard rotations:
 *
 *     x' = H128(x .* suh) / sqrt(128)        (per 128-channel block of k)
 *     y' = x' . W_hat                         (fp32 accumulation)
 *     y  = svh .* H128(y') / sqrt(128)        (per 128-channel block of n)
 *
 * Sources (page titles):
 *   [GEMM] "ExLlamaV3推理快的秘密: EXL3 GEMM内核与融合Viterbi编码CUDA实现剖析",
 *          sections 先看结论 (conclusions), GEMM内核 (GEMM kernel: 128-point
 *          Hadamard on the input fused with the dequantising matmul; the
 *          codebook is one integer multiply + one lop3, no table),
 *          小批量GEMV (small-batch GEMV for the decode phase, bandwidth bound),
 *          Viterbi编码内核剖析 (16 x 16 tiles, tail-biting trellis, packed into
 *          a 16-bit index sequence).
 *   [OVW]  "为什么ExLlamaV3值得关注": EXL3 is a simplified QTIP variant with a
 *          procedural codebook and a tail-biting trellis, 1..8 bits per weight.
 *
 * Data layout (the pages do not fix one; this library's convention):
 *   x        m x k fp16, row-major.
 *   trellis  uint16 [k/16][n/16][16*K]; tile (tk, tn) covers
 *            W_hat[16tk + r][16tn + c], weight index i = 16 r + c.  The tile's
 *            16K words are one big-endian bit string (bit 15 of word 0 first);
 *            weight i's 16-bit state is the window of positions
 *            [iK + K - 16, iK + K) taken modulo 256K (weight 0 wraps to the
 *            stream's end), earliest position most significant.
 *   codebook v = state * 89226354 + 64248484 (mod 2^32);
 *            v = (v & 0x8fff8fff) ^ 0x3b603b60;
 *            w = fp16(v >> 16) + fp16(v & 0xffff), bit patterns read as fp16,
 *            sum rounded to nearest even.
 *   suh      k fp16 (+-1 signs), svh n fp16 (signed per-channel scales).
 *   y        m x n fp16, row-major.
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE memory owned by the caller, 16-byte
 *     aligned; the library never allocates, frees or synchronises inside these
 *     calls.  Work is enqueued asynchronously on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream).
 *   - k and n must be multiples of 128; 1 <= K <= 8; y must not overlap x.
 *   - Argument errors return EXL3_ERR_INVALID_ARG / EXL3_ERR_UNSUPPORTED /
 *     EXL3_ERR_WORKSPACE before anything is launched.  A failed launch returns
 *     EXL3_ERR_CUDA (the CUDA error is left for cudaGetLastError to report).
 *   - Device-side waits are bounded.  A wait that runs out records a timeout
 *     in the workspace's status word (read it with exl3_workspace_status) and
 *     the kernel returns early; the output is then undefined.
 *   - Calls are thread-safe; concurrent calls on different streams need
 *     distinct workspaces.
 */
#ifndef EXL3_B200_H
#define EXL3_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EXL3_OK = 0,
    EXL3_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad K          */
    EXL3_ERR_UNSUPPORTED = 2, /* valid request this build does not handle (m > 16 for gemv) */
    EXL3_ERR_WORKSPACE = 3,   /* workspace missing or smaller than *_workspace_size */
    EXL3_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed               */
    EXL3_ERR_TIMEOUT = 5      /* a bounded device wait ran out (see exl3_workspace_status) */
} exl3_status;

/* Static, human-readable name of a status code (never NULL). */
const char *exl3_status_string(int status);

/* Library version string, e.g. "exl3-b200 0.1 sm_100a". */
const char *exl3_version(void);

/*
 * exl3_hadamard -- blockwise 128-point Hadamard rotation ([GEMM] section
 * GEMM内核: the input is rotated by a 128-point Hadamard before the matmul).
 *   y[r, 128b + i] = post[128b+i] * (1/sqrt(128)) * sum_j H[i][j] * x[r,128b+j] * pre[128b+j]
 * with the Sylvester matrix H[i][j] = (-1)^popcount(i & j).
 *   x, y      rows x cols fp16, row-major; cols % 128 == 0; y may equal x
 *             (in place) but must not otherwise overlap it.
 *   pre, post cols fp16 each, or NULL for all ones.
 * Arithmetic in fp32, one fp16 rounding of the result.  rows == 0 is a no-op.
 */
exl3_status exl3_hadamard(const void *x, void *y, int64_t rows, int64_t cols,
                          const void *pre, const void *post, void *stream);

/*
 * exl3_decode_tiles -- decode a whole trellis to dense fp16 weights, for
 * checking ([GEMM] sections 先看结论 and GEMM内核: state -> fp16 through the
 * procedural codebook; Viterbi编码内核剖析: tail-biting 16 x 16 tiles).
 *   trellis   uint16 [k/16][n/16][16K] (layout above).
 *   w         k x n fp16, row-major (output, caller-owned).
 * Bit-exact: every weight equals the codebook value of its trellis state.
 */
exl3_status exl3_decode_tiles(const uint16_t *trellis, void *w, int64_t k, int64_t n, int K,
                              void *stream);

/*
 * exl3_gemv -- the linear layer for small batches, 1 <= m <= 16 ([GEMM]
 * section 小批量GEMV: in the decode phase the bottleneck is memory bandwidth).
 * Arguments as in the layout above.  `workspace` (device memory, at least
 * exl3_gemv_workspace_size bytes) holds fp32 split-k partial sums, arrival
 * counters and a status word; it must be zero-filled ONCE after allocation
 * (the kernels return the counters to zero themselves) and must not be shared
 * by calls that can run concurrently.
 */
size_t exl3_gemv_workspace_size(int64_t m, int64_t k, int64_t n, int K);
exl3_status exl3_gemv(const void *x, const uint16_t *trellis, const void *suh, const void *svh,
                      void *y, int64_t m, int64_t k, int64_t n, int K, void *workspace,
                      size_t workspace_bytes, void *stream);

/*
 * exl3_gemv_multi -- several independent layers with the same batch size m
 * (1 <= m <= 16) in one call: y_i = svh_i .* H(H(x_i .* suh_i) . W_hat_i).
 * ([GEMM] section 小批量GEMV: the decode-phase GEMV is bandwidth bound, and
 * a decoder step runs many such layers back to back.)
 *   layers    HOST array of `count` descriptors (copied during the call; the
 *             pointers in it are device memory, laid out as for exl3_gemv).
 *   count     1 .. any; every 32 layers (in call order, any mix of K) run
 *             as one persistent launch (preceded by one input-rotation
 *             launch unless every CTA's share is short enough to rotate its
 *             own inputs), so the fixed cost is paid once, not per layer or
 *             per K.  The
 *             persistent launch splits its CTAs into one group per K (in
 *             proportion to the group's estimated cost), and a group's CTAs
 *             share out its work units evenly.
 *   workspace at least exl3_gemv_multi_workspace_size bytes, zero-filled
 *             once after allocation, not shared by concurrent calls.
 * Layers must not write one another's inputs (x, trellis, suh, svh).  Results
 * match exl3_gemv to within the stated tolerance (the split of the sums over
 * CTAs differs, so the fp32 rounding may too); both are deterministic.
 * EXL3_ERR_INVALID_ARG if any descriptor is invalid (nothing is launched).
 */
typedef struct {
    const void *x;           /* m x k fp16 */
    const uint16_t *trellis; /* [k/16][n/16][16K] */
    const void *suh;         /* k fp16 */
    const void *svh;         /* n fp16 */
    void *y;                 /* m x n fp16 (output) */
    int64_t k, n;
    int K;
} exl3_linear;
size_t exl3_gemv_multi_workspace_size(const exl3_linear *layers, int count, int64_t m);
exl3_status exl3_gemv_multi(const exl3_linear *layers, int count, int64_t m, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * exl3_gemv_noalloc -- exl3_gemv for callers that cannot allocate device
 * memory.  (The pages have no counterpart: this is a library convenience.)
 *
 * Some callers cannot call cudaMalloc or an allocator of their own: code that
 * runs under a host framework which owns all device memory, a plugin with a
 * fixed memory budget, or a latency-critical path where an allocation (and the
 * device synchronisation it may imply) is not allowed.  This entry point needs
 * no workspace argument: its scratch (split-k partial sums and arrival
 * counters) is a fixed array of exl3_gemv_noalloc_max_scratch() bytes (4 MiB)
 * compiled into the library, which every GPU that loads the library holds
 * until the process exits.  The caller still passes x, the weights and y.
 *   - Shapes whose scratch exceeds that maximum are rejected with
 *     EXL3_ERR_WORKSPACE before anything is launched (exl3_gemv_workspace_size
 *     tells how much a shape needs).
 *   - The array's device address is looked up (cudaGetSymbolAddress) on the
 *     first call on a device and again whenever the current context changes
 *     (after cudaDeviceReset, for example).  The lookup cannot run inside a
 *     stream capture: a call that needs it while `stream` is capturing
 *     returns EXL3_ERR_UNSUPPORTED, so make the first call on a device
 *     outside any capture.
 *   - Every call on a device shares the one array and it keeps the last call's
 *     contents: each call first clears the status word and the arrival
 *     counters on its stream (one cudaMemsetAsync, which allocates nothing), and
 *     calls that can overlap on the GPU (different streams, or concurrent
 *     host threads) race on the array and must not be issued.
 *   - No cudaMalloc, cudaFree or other allocating routine is called.
 * Arguments and results otherwise as exl3_gemv.
 */
size_t exl3_gemv_noalloc_max_scratch(void);
exl3_status exl3_gemv_noalloc(const void *x, const uint16_t *trellis, const void *suh,
                              const void *svh, void *y, int64_t m, int64_t k, int64_t n, int K,
                              void *stream);

/*
 * exl3_gemm -- the linear layer on the tensor cores (tcgen05 / TMEM), any
 * m >= 1, tuned for m >= 64 ([GEMM] section GEMM内核: Hadamard rotation of the
 * input, then the dequantising matmul; the kernel map picks tiles by shape).
 * n is any multiple of 128: for n = 256j + 128 the last output tile carries
 * 128 columns (its other half is computed from stale bytes and not stored).
 * The kernel is persistent (one CTA per SM) and splits the work evenly over the CTAs by
 * (256 x 256 output tile, 64-channel k block) units, so a tile can be shared
 * by several CTAs; their fp32 partial sums meet in the workspace and are
 * added in a fixed order, so results are deterministic.  For m <= 64 the
 * decoded weights are the MMA's A operand (128 output channels per MMA) and
 * the rotated activations its B operand (N = m rounded up to 32), so a small
 * batch does not pay for 128-row MMAs; the result is the same function.
 * `workspace` (at least exl3_gemm_workspace_size bytes -- a size that depends
 * on the current device's SM count, so query it on the device that runs the
 * call -- zero-filled once after allocation) holds a status word, per-tile
 * arrival counters (each call returns them to zero), the rotated activations
 * x' (m rounded up to 256, x k fp16) and the split partial sums (two 256 KB
 * slots per CTA).  Same argument conventions as exl3_gemv.  After a call
 * that reported EXL3_ERR_TIMEOUT the counters may be left part-way: zero-fill
 * the workspace again before its next use.
 */
size_t exl3_gemm_workspace_size(int64_t m, int64_t k, int64_t n, int K);
exl3_status exl3_gemm(const void *x, const uint16_t *trellis, const void *suh, const void *svh,
                      void *y, int64_t m, int64_t k, int64_t n, int K, void *workspace,
                      size_t workspace_bytes, void *stream);

/*
 * exl3_gemm_multi -- several layers with the same batch size m, the same k and
 * the same K (each with its own x, suh, svh, y and n) through the tensor-core
 * GEMM in one call: y_i = svh_i .* H(H(x_i .* suh_i) . W_hat_i).  ([GEMM]
 * section GEMM内核: the kernel map picks the tiling for the shape; the layers
 * of a decoder block that read the same activations -- q/k/v, gate/up -- are
 * one problem with more output columns.)
 *   layers    HOST array of `count` descriptors, as for exl3_gemv_multi.
 *   count     1 .. any; every 8 layers (in call order) run as one rotation
 *             launch and one persistent GEMM launch whose output tiles are
 *             all the layers' tiles, so the stream-K split balances them
 *             together (a narrow layer such as a k or v projection alone
 *             would leave most of the GPU waiting on its few tiles).
 *   workspace at least exl3_gemm_multi_workspace_size bytes (one tiled x' per
 *             layer of a launch), zero-filled once after allocation, not
 *             shared by concurrent calls.
 * Layers must not write one another's inputs (x, trellis, suh, svh) and
 * their y must not overlap.  Results equal exl3_gemm's for each layer to
 * within the stated tolerance.  EXL3_ERR_INVALID_ARG if a descriptor is
 * invalid, EXL3_ERR_UNSUPPORTED if the layers' k or K differ (nothing is
 * launched in either case).
 */
size_t exl3_gemm_multi_workspace_size(const exl3_linear *layers, int count, int64_t m);
exl3_status exl3_gemm_multi(const exl3_linear *layers, int count, int64_t m, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * exl3_matmul -- the layer for any m >= 1 with the kernel chosen inside the
 * library ([GEMM] section GEMM内核: a kernel map picks the kernel from the
 * problem shape; section 小批量GEMV: the decode-phase small batches are
 * bandwidth bound and take the GEMV): m <= 16 runs exl3_gemv, larger m runs
 * exl3_gemm.  Arguments, layout and errors as those two calls.
 * `workspace` must hold exl3_matmul_workspace_size(m, k, n, K) bytes, the
 * size of the path that m selects (zero-filled once after allocation, as
 * for exl3_gemv / exl3_gemm).  Results are those of the selected call.
 */
size_t exl3_matmul_workspace_size(int64_t m, int64_t k, int64_t n, int K);
exl3_status exl3_matmul(const void *x, const uint16_t *trellis, const void *suh, const void *svh,
                        void *y, int64_t m, int64_t k, int64_t n, int K, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * exl3_matmul_multi -- several layers with the same batch size m in one call,
 * with the kernel chosen by m as for exl3_matmul: m <= 16 runs
 * exl3_gemv_multi (any mix of k and K), larger m runs exl3_gemm_multi (all
 * layers with the same k and K).  Workspace: exl3_matmul_multi_workspace_size
 * bytes, zero-filled once after allocation.  Errors as the selected call.
 */
size_t exl3_matmul_multi_workspace_size(const exl3_linear *layers, int count, int64_t m);
exl3_status exl3_matmul_multi(const exl3_linear *layers, int count, int64_t m, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * exl3_encode -- tail-biting trellis encoding of a weight matrix: for every
 * 16 x 16 tile, the bit string whose decoded weights are closest in squared
 * error to the tile's targets ([GEMM] section Viterbi编码内核剖析: a Viterbi
 * forward pass over the trellis keeps the accumulated cost of every path and
 * takes the cheapest; the tail-biting boundary is closed by enumerating start
 * states, so the codeword's head and tail agree).  The inverse direction of
 * exl3_decode_tiles: exl3_decode_tiles(exl3_encode(w)) is the encoded matrix.
 *   w         k x n fp32, row-major: the target values (already in the
 *             codebook's scale; the caller applies any scaling or rotation).
 *   trellis   uint16 [k/16][n/16][16K] (output, layout above).
 *   cost      (k/16) x (n/16) fp32 (output, nullable): each tile's sum of
 *             squared errors, as the search computed it.
 *   k, n      multiples of 16 (at most 2^22); K in [1, 8].
 * The search (two passes per tile): pass 1 lets every state start and takes
 * the low 16-K bits of the cheapest end as the overlap; pass 2 allows only
 * starts whose high 16-K bits are that overlap and ends in the cheapest state
 * whose low bits are it, then traces the path back.  Costs are fp32 (each
 * weight's (w - cb(s))^2 added by one fused multiply-add), ties go to the
 * smallest index; results are deterministic.
 * `workspace` (at least exl3_encode_workspace_size bytes, device memory, no
 * initialisation needed) holds the per-step choices of the CTAs in flight
 * (256 x 2^(16-K) bytes per CTA, for up to ~1 GiB) and, for K = 1, their
 * cost vectors.  Argument errors return EXL3_ERR_INVALID_ARG (null or
 * misaligned w / trellis, bad sizes, any two of w, trellis and cost
 * overlapping) or EXL3_ERR_WORKSPACE before anything is launched.
 */
size_t exl3_encode_workspace_size(int64_t k, int64_t n, int K);
exl3_status exl3_encode(const float *w, uint16_t *trellis, float *cost, int64_t k, int64_t n, int K,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * exl3_udu -- block factorisation H = U D U^T of a symmetric positive
 * definite k x k matrix (fp64), 16 x 16 blocks: U unit block-upper-triangular,
 * D block-diagonal ([GEMM] section Viterbi编码内核剖析: ldlq() performs a
 * block-wise LDL decomposition before the trellis encoding).
 *   h         k x k fp64, row-major (read; may equal ud).
 *   ud        k x k fp64 (output): the diagonal blocks hold D_b, the strictly
 *             upper blocks U_ab (a < b), the strictly lower blocks are zero.
 *   k         multiple of 16, at most 65536.
 *   workspace at least exl3_udu_workspace_size(k) bytes of device memory.
 * Bottom-up: D_b = H_bb - sum_{c>b} U_bc D_c U_bc^T, U_ab = (H_ab - sum_{c>b}
 * U_ac D_c U_bc^T) D_b^-1 (D_b inverted by Gauss-Jordan without pivoting), all
 * in fp64.  EXL3_ERR_INVALID_ARG for null or misaligned pointers, bad k, or h
 * and ud overlapping without being equal.
 */
size_t exl3_udu_workspace_size(int64_t k);
exl3_status exl3_udu(const double *h, double *ud, int64_t k, void *workspace, size_t workspace_bytes,
                     void *stream);

/*
 * exl3_ldlq -- Hessian-aware trellis quantisation of a layer (LDLQ with the
 * trellis encoder; [GEMM] section Viterbi编码内核剖析: ldlq() decomposes the
 * Hessian block-wise, then the trellis kernel encodes the 16 x 16 tiles).
 *   w         k x n fp32, row-major: the layer in the x . W orientation (rows
 *             = input channels).
 *   h         k x k fp64: the input Hessian (symmetric positive definite).
 *   trellis   uint16 [k/16][n/16][16K] (output).
 *   w_hat     k x n fp32 (output, nullable): the decoded weights.
 *   k         multiple of 16 (at most 65536); n multiple of 16; K in [1, 8].
 * With H = U D U^T (exl3_udu), tile rows are encoded in order: row block b's
 * target T_b = W_b - sum_{c<b} U_{c,b}^T (W_hat_c - W_c) is formed in fp64,
 * rounded to fp32 and encoded (exl3_encode), so that the proxy loss
 * tr((W_hat - W)^T H (W_hat - W)) is sum_b tr(F_b^T D_b F_b), F_b = W_hat_b -
 * T_b.  With H = I (or any block-diagonal H) this is exl3_encode of W.
 * `workspace`: at least exl3_ldlq_workspace_size bytes (the factor, the
 * errors and the encoder's workspace; no initialisation needed).  Argument
 * errors as exl3_encode (w_hat must not overlap w or trellis).
 */
size_t exl3_ldlq_workspace_size(int64_t k, int64_t n, int K);
exl3_status exl3_ldlq(const float *w, const double *h, uint16_t *trellis, float *w_hat, int64_t k, int64_t n,
                      int K, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Launch options, process-wide (default 0).
 *
 * EXL3_LAUNCH_PDL -- launch exl3_gemv / exl3_gemm kernels with programmatic
 *   dependent launch (CUDA programmatic stream serialization): a kernel may
 *   start while the preceding kernel in the stream is still finishing, and
 *   it begins streaming its WEIGHT operands (trellis, suh, svh) at once; all
 *   other reads (x, the workspace) and every write wait until the preceding
 *   kernel has completed and its writes are visible.  Enable it only when the
 *   weights are not written by the kernel launched immediately before on the
 *   same stream (true for inference with loaded weights).  Has no effect on
 *   results.
 */
#define EXL3_LAUNCH_PDL 1u
void exl3_set_launch_flags(unsigned flags);
unsigned exl3_launch_flags(void);

/*
 * exl3_workspace_status -- read (synchronously, on `stream`) the status word a
 * gemv/gemm call leaves in its workspace: EXL3_OK, or EXL3_ERR_TIMEOUT if a
 * bounded device wait ran out.  `clear` != 0 resets it to EXL3_OK and zeroes
 * the rest of the workspace's first 64 KiB (the arrival counters, which a
 * call that timed out may leave nonzero), so the workspace can serve further
 * calls.
 */
exl3_status exl3_workspace_status(void *workspace, size_t workspace_bytes, int clear, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* EXL3_B200_H */
