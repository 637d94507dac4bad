// matmul.cu -- exl3_matmul: the layer y = svh .* H(H(x .* suh) . W_hat) for
// any batch size, with the kernel chosen inside the library by m (EXL3 GEMM
// kernel article, section GEMM内核: a kernel map picks the kernel and its
// configuration from the problem shape; section 小批量GEMV: small batches in
// the decode phase are bandwidth bound and take a dedicated GEMV path).
//
// The map: m <= kMatmulGemvMaxM runs the memory-bound GEMV (exl3_gemv: one
// decode of each weight serves up to 16 batches in the A operand of
// mma.sync); every larger m runs the tensor-core GEMM (exl3_gemm), which for
// m <= 64 already swaps the operand roles so that a small batch does not pay
// for 128-row MMAs.  The crossover is where the GEMV's second batch group
// ends: a third would cost more registers than a CTA per SM can hold.
#include "exl3_host.h"

namespace exl3 {

constexpr int64_t kMatmulGemvMaxM = 16;

}  // namespace exl3

extern "C" size_t exl3_matmul_workspace_size(int64_t m, int64_t k, int64_t n, int K)
{
    return m <= exl3::kMatmulGemvMaxM ? exl3_gemv_workspace_size(m, k, n, K) : exl3_gemm_workspace_size(m, k, n, K);
}

extern "C" exl3_status exl3_matmul(const void *x, const uint16_t *trellis, const void *suh, const void *svh,
                                   void *y, int64_t m, int64_t k, int64_t n, int K, void *workspace,
                                   size_t workspace_bytes, void *stream)
{
    if (m >= 1 && m <= exl3::kMatmulGemvMaxM)
        return exl3_gemv(x, trellis, suh, svh, y, m, k, n, K, workspace, workspace_bytes, stream);
    return exl3_gemm(x, trellis, suh, svh, y, m, k, n, K, workspace, workspace_bytes, stream);
}

extern "C" size_t exl3_matmul_multi_workspace_size(const exl3_linear *layers, int count, int64_t m)
{
    return m <= exl3::kMatmulGemvMaxM ? exl3_gemv_multi_workspace_size(layers, count, m)
                                      : exl3_gemm_multi_workspace_size(layers, count, m);
}

extern "C" exl3_status exl3_matmul_multi(const exl3_linear *layers, int count, int64_t m, void *workspace,
                                         size_t workspace_bytes, void *stream)
{
    if (m >= 1 && m <= exl3::kMatmulGemvMaxM)
        return exl3_gemv_multi(layers, count, m, workspace, workspace_bytes, stream);
    return exl3_gemm_multi(layers, count, m, workspace, workspace_bytes, stream);
}
