/*
 * bsp_testing.h -- test hooks of libbsp.so (not part of the compute path).
 *
 * The pages describe no failure handling; these hooks exist so the bounded waits
 * inside the GEMM kernels can be exercised without faulting or hanging a GPU.
 */
#ifndef BSP_TESTING_H_
#define BSP_TESTING_H_

#include <stdint.h>

#include "bsp.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * bsp_testing_gemm_stall -- runs the nvfp4 (scheme 1) or fp8r (scheme 0) GEMM with
 * the producer stopping after `stop_after_stages` K-stages, so the MMA thread's
 * wait on the next stage can never complete.  Every wait in the kernel is bounded
 * by `wait_limit_ms` (1..10000); the kernel then records BSP_ERR_TIMEOUT in the
 * device status word, waits for the copies and MMAs it already issued, frees its
 * tensor memory and exits, leaving the context usable.  Arguments are those of
 * nvfp4_gemm / fp8r_gemm (a_sf / w_sf ignored for fp8r; no bias).  The output is
 * left partially written.  Read the outcome with bsp_last_device_status().
 */
int bsp_testing_gemm_stall(int scheme, const uint8_t* a, const uint8_t* a_sf,
                           const float* a_scale, const uint8_t* w, const uint8_t* w_sf,
                           const float* w_scale, void* out_bf16, int64_t M, int64_t N,
                           int64_t K, int64_t stop_after_stages, int64_t wait_limit_ms,
                           bsp_stream_t stream);

/*
 * bsp_testing_set_gemm_kernel -- selects the GEMM kernel of later nvfp4_gemm /
 * fp8r_gemm calls in this process: 0 = automatic (default), 1 = CTA-pair kernel
 * (256 x 256 tiles, tcgen05 cta_group::2), 2 = single-CTA kernel (128 x 256 or
 * 128 x 128 tiles).  Both compute the same results; this exists so the tests can
 * cover each.  Returns the previous choice, or BSP_ERR_INVALID_ARG.
 */
int bsp_testing_set_gemm_kernel(int choice);

/*
 * bsp_testing_set_quant_kernel -- selects the kernel of later nvfp4_quantize_act calls in
 * this process: 0 = by input size (default), 1 = grid-stride kernel (each thread loads its
 * blocks directly), 2 = staged kernel (one CTA per SM streaming its range through a
 * shared-memory ring filled by bulk copies).  Both give identical codes and scales; this
 * exists so the tests can cover each.  Returns the previous choice, or
 * BSP_ERR_INVALID_ARG.
 */
int bsp_testing_set_quant_kernel(int choice);

/*
 * bsp_testing_cvt_range -- writes out[i] = the quantizers' conversion of the fp32 whose
 * bit pattern is first + i, for i in [0, n): kind 0 = E2M1 code (cvt.rn.satfinite.e2m1x2,
 * the low nibble), kind 1 = E4M3 byte (cvt.rn.satfinite.e4m3x2).  first + n <= 2^32.
 * An exhaustive pin of the conversions walks all 2^32 patterns in ranges.  Returns
 * BSP_ERR_INVALID_ARG on a bad kind or range.
 */
int bsp_testing_cvt_range(int kind, uint32_t first, int64_t n, uint8_t* out,
                          bsp_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BSP_TESTING_H_ */
