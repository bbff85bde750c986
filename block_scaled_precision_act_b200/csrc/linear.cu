// linear.cu -- the nvfp4 linear forward as one call: activation quantizer into a
// caller workspace, then the block-scaled GEMM launched as a programmatic dependent of
// the quantizer ("BFL (fp8r / nvfp4)", Kernels table: activations are quantized at run
// time before the FP4 GEMM).  Host code only; the kernels are those of quant.cu and
// gemm.cu.
#include <cstdint>

#include "bsp_internal.h"

namespace bsp {
namespace {

constexpr int64_t kWorkspaceAlign = 256;

int64_t codes_bytes(int64_t M, int64_t K) { return M * (K / 2); }

int64_t scales_offset(int64_t M, int64_t K)
{
    return (codes_bytes(M, K) + kWorkspaceAlign - 1) / kWorkspaceAlign * kWorkspaceAlign;
}

int64_t align_up(int64_t v) { return (v + kWorkspaceAlign - 1) / kWorkspaceAlign * kWorkspaceAlign; }

// after the scales, at a 256-byte boundary: the dynamic path's per-CTA maxima
int64_t partials_offset(int64_t M, int64_t K)
{
    return align_up(scales_offset(M, K) + nvfp4_sf_bytes(M, K, BSP_SF_MMA));
}

}  // namespace
}  // namespace bsp

extern "C" {

int64_t nvfp4_linear_workspace_bytes(int64_t M, int64_t K)
{
    if (M < 0 || K <= 0 || K % 64 != 0) return BSP_ERR_INVALID_ARG;
    if (M > (int64_t{1} << 40) / K) return BSP_ERR_UNSUPPORTED_SHAPE;
    const int64_t sf = nvfp4_sf_bytes(M, K, BSP_SF_MMA);
    if (sf < 0) return sf;
    return bsp::partials_offset(M, K) + bsp::kDynamicPartials * 4;
}

int nvfp4_linear(const void* x_bf16, const float* input_scale, const uint8_t* w_codes,
                 const uint8_t* w_sf, const float* w_scale, const void* bias_bf16,
                 void* out_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                 int64_t workspace_bytes, bsp_stream_t stream)
{
    if (M < 0 || N < 0 || K <= 0) return BSP_ERR_INVALID_ARG;
    if (K % 64 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return BSP_OK;
    const int64_t need = nvfp4_linear_workspace_bytes(M, K);
    if (need < 0) return static_cast<int>(need);
    if (!workspace || workspace_bytes < need) return BSP_ERR_INVALID_ARG;
    if (!bsp::aligned16(workspace)) return BSP_ERR_MISALIGNED;
    auto* a_codes = static_cast<uint8_t*>(workspace);
    uint8_t* a_sf = a_codes + bsp::scales_offset(M, K);
    int st = nvfp4_quantize_act(x_bf16, M, K, input_scale, a_codes, a_sf, BSP_SF_MMA, stream);
    if (st != BSP_OK) return st;
    // launched as a programmatic dependent of the quantizer (as every GEMM launch is),
    // fetching its first weight stages while the quantizer finishes
    return bsp::gemm_after_quantizer(true, a_codes, a_sf, input_scale, w_codes, w_sf, w_scale,
                                     bias_bf16, out_bf16, M, N, K, stream);
}

int nvfp4_linear_dynamic(const void* x_bf16, float* input_scale_out, const uint8_t* w_codes,
                         const uint8_t* w_sf, const float* w_scale, const void* bias_bf16,
                         void* out_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                         int64_t workspace_bytes, bsp_stream_t stream)
{
    if (M < 0 || N < 0 || K <= 0) return BSP_ERR_INVALID_ARG;
    if (K % 64 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return BSP_OK;
    if (!input_scale_out) return BSP_ERR_INVALID_ARG;
    const int64_t need = nvfp4_linear_workspace_bytes(M, K);
    if (need < 0) return static_cast<int>(need);
    if (!workspace || workspace_bytes < need) return BSP_ERR_INVALID_ARG;
    if (!bsp::aligned16(workspace)) return BSP_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(input_scale_out) & 3u) return BSP_ERR_MISALIGNED;
    // g = amax(x) / (448 * 6) of this very activation: per-CTA maxima into the workspace,
    // reduced by the quantizer's CTAs, which also publish g for the GEMM
    auto* a_codes = static_cast<uint8_t*>(workspace);
    uint8_t* a_sf = a_codes + bsp::scales_offset(M, K);
    auto* partials = reinterpret_cast<uint32_t*>(a_codes + bsp::partials_offset(M, K));
    int st = bsp::dynamic_quantize_front(x_bf16, M, K, partials, input_scale_out, a_codes, a_sf,
                                        stream);
    if (st != BSP_OK) return st;
    return bsp::gemm_after_quantizer(true, a_codes, a_sf, input_scale_out, w_codes, w_sf, w_scale,
                                     bias_bf16, out_bf16, M, N, K, stream);
}

int64_t fp8r_linear_workspace_bytes(int64_t M, int64_t K)
{
    if (M < 0 || K <= 0 || K % 8 != 0) return BSP_ERR_INVALID_ARG;
    if (M > (int64_t{1} << 40) / K) return BSP_ERR_UNSUPPORTED_SHAPE;
    return bsp::align_up(M * K) + bsp::align_up(4 * M);
}

int fp8r_linear(const void* x_bf16, const uint8_t* w_e4m3, const float* w_row_scale,
                const void* bias_bf16, void* out_bf16, int64_t M, int64_t N, int64_t K,
                void* workspace, int64_t workspace_bytes, bsp_stream_t stream)
{
    if (M < 0 || N < 0 || K <= 0) return BSP_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BSP_OK;
    const int64_t need = fp8r_linear_workspace_bytes(M, K);
    if (need < 0) return static_cast<int>(need);
    if (!workspace || workspace_bytes < need) return BSP_ERR_INVALID_ARG;
    if (!bsp::aligned16(workspace)) return BSP_ERR_MISALIGNED;
    auto* aq = static_cast<uint8_t*>(workspace);
    auto* as = reinterpret_cast<float*>(aq + bsp::align_up(M * K));
    int st = fp8r_quantize_rows(x_bf16, M, K, aq, as, stream);
    if (st != BSP_OK) return st;
    // launched as a programmatic dependent of the quantizer (as every GEMM launch is),
    // fetching its first weight stages while the quantizer finishes
    return bsp::gemm_after_quantizer(false, aq, nullptr, as, w_e4m3, nullptr, w_row_scale,
                                     bias_bf16, out_bf16, M, N, K, stream);
}

}  // extern "C"
