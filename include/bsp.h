/*
 * bsp.h -- C ABI of libbsp.so: the block-scaled precision linear on B200 (sm_100a).
 *
 * The operation is the quantized linear layer Y = X * W^T (+ bias) of a
 * rectified-flow image transformer in the two storage schemes defined on the
 * "BFL (fp8r / nvfp4)" page (Diffusers quantization doc, format bullets):
 *
 *   nvfp4 (ModelOpt layout): `weight` packed E2M1, two values per byte;
 *          `weight_scale` E4M3, one per block of 16 elements along K;
 *          `weight_scale_2` fp32 global scale; `input_scale` fp32 calibrated
 *          activation scale.
 *   fp8r : `weight` E4M3 with one fp32 `weight_scale` per row; activations are
 *          quantized to E4M3 per row at run time.
 *
 * The same page's "Kernels" table pairs each scheme with a fused path: for nvfp4,
 * an activation quantizer followed by a block-scaled FP4 GEMM; for fp8r, a
 * row-scaled FP8 GEMM.  These entry points are that pair of calls for each scheme.
 *
 * Conventions for every call
 *   - All pointers are DEVICE pointers unless stated otherwise, owned by the caller.
 *     The library makes no allocation and keeps no per-call state: what one call
 *     computes depends only on its arguments.  It does keep a little process-wide
 *     state: per device, a status word written by kernels whose bounded wait ran out
 *     (read and cleared by bsp_last_device_status), cached device properties and
 *     kernel attributes, and nvfp4_linear_noalloc's fixed 128 MiB buffer and its cached
 *     address; process-wide, the wait limit (bsp_set_wait_limit_ms) and the kernel
 *     choices that the bsp_testing_set_* hooks of bsp_testing.h switch.  Every tensor
 *     is contiguous row-major.  All work is enqueued asynchronously on `stream`
 *     (NULL = the legacy default stream) of the CURRENT device; nothing synchronises
 *     the host.
 *   - Tensor pointers must be 16-byte aligned (BSP_ERR_MISALIGNED otherwise).
 *   - Argument errors are detected on the host before any launch and returned as a
 *     negative bsp_status; nothing is enqueued in that case.  A zero-sized problem
 *     (M == 0, or N == 0 for a GEMM) returns BSP_OK and enqueues nothing; its
 *     pointers may then be NULL.
 *   - Launch failures return BSP_ERR_CUDA.  Faults found by the kernels themselves
 *     (a bounded wait that ran out) are recorded in a per-device status word and
 *     reported by bsp_last_device_status().
 *   - Only compute capability 10.0 (B200, sm_100a) is supported
 *     (BSP_ERR_UNSUPPORTED_DEVICE otherwise).  There is no fallback path.
 *
 * Number formats
 *   E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
 *         {0, 0.5, 1, 1.5, 2, 3, 4, 6}.  Packed two per byte: element 2j in bits 0-3,
 *         element 2j+1 in bits 4-7.
 *   E4M3: the "fn" variant (bias 7, no infinities, max 448, 0x7F/0xFF are NaN).
 *   bf16 in and out.  Rounding everywhere is to nearest, ties to even; encoders
 *   saturate (E2M1 at +-6, E4M3 at +-448) and keep the sign.
 *
 * Scale-factor layouts for NVFP4 block scales (one E4M3 byte per 16 elements):
 *   BSP_SF_LINEAR: [rows][K/16] row-major.
 *   BSP_SF_MMA   : the tiled layout the tensor cores read.  Rows are grouped in
 *                  tiles of 128 and block-columns in tiles of 4; tile (rt, ct) is
 *                  512 contiguous bytes at offset (rt * ceil(K/64) + ct) * 512, and
 *                  inside it row r, block-column c sits at
 *                  (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4).
 *                  Its size is nvfp4_sf_bytes(rows, K, BSP_SF_MMA) (rows padded to
 *                  a multiple of 128); padding bytes are never read for results.
 */
#ifndef BSP_H_
#define BSP_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* bsp_stream_t; /* same handle as cudaStream_t */

typedef enum {
    BSP_OK = 0,
    BSP_ERR_INVALID_ARG = -1,       /* null pointer, bad enum, negative size        */
    BSP_ERR_UNSUPPORTED_SHAPE = -2, /* a size outside the documented constraints    */
    BSP_ERR_MISALIGNED = -3,        /* a tensor pointer not 16-byte aligned         */
    BSP_ERR_UNSUPPORTED_DEVICE = -4,/* current device is not compute capability 10.0 */
    BSP_ERR_CUDA = -5,              /* a CUDA runtime call or launch failed          */
    BSP_ERR_TIMEOUT = -6            /* a kernel's bounded wait ran out (device side) */
} bsp_status;

typedef enum { BSP_SF_LINEAR = 0, BSP_SF_MMA = 1 } bsp_sf_layout;

/*
 * nvfp4_quantize_act -- NVFP4 activation quantizer ("BFL (fp8r / nvfp4)", Kernels
 * table: the activations of an nvfp4 linear are quantized before the FP4 GEMM; the
 * format bullet gives block 16, E4M3 block scales and the fp32 `input_scale`).
 *
 *   x_bf16        [M][K] bf16.
 *   global_scale  device pointer to ONE fp32: the decode-side global scale g
 *                 (`input_scale` for activations, `weight_scale_2` for weights).
 *   codes         out [M][K/2] bytes, packed E2M1.
 *   scales        out E4M3 block scales in `layout` (nvfp4_sf_bytes(M, K, layout)).
 * Per block b of 16 elements along K (every step one IEEE binary32 operation):
 *   s_b = amax_b / (6 g) (0 when 6 g is 0) ; scales[b] = E4M3(s_b) ; d = e4m3(scales[b]) * g ;
 *   d == 0 -> all 16 codes 0 ; else code_i = E2M1(x_i * (1/d)), 1/d clamped to FLT_MAX.
 * Constraints: K % 16 == 0; BSP_SF_MMA also needs K % 64 == 0.
 */
int nvfp4_quantize_act(const void* x_bf16, int64_t M, int64_t K, const float* global_scale,
                       uint8_t* codes, uint8_t* scales, int layout, bsp_stream_t stream);

/*
 * nvfp4_gemm -- block-scaled FP4 GEMM with the dequantisation fused into the
 * epilogue ("BFL (fp8r / nvfp4)", Kernels table: the nvfp4 fused GEMM).
 *
 *   a_codes [M][K/2], a_sf (BSP_SF_MMA, rows = M), a_global (device, 1 fp32 = input_scale)
 *   w_codes [N][K/2], w_sf (BSP_SF_MMA, rows = N), w_global (device, 1 fp32 = weight_scale_2)
 *   bias_bf16  [N] bf16 or NULL.
 *   out_bf16   [M][N] bf16.
 *   Y[m][n] = bf16( acc[m][n] * (a_global * w_global) + bias[n] ),
 *   acc = sum_k e2m1(a)*e4m3(sa) * e2m1(w)*e4m3(sw), accumulated in fp32 on the
 *   tensor cores.
 * Constraints: K % 64 == 0, K >= 64; N % 8 == 0.  Any M >= 0.
 * Launch: with programmatic stream serialisation (also fp8r_gemm and nvfp4_gemm_quant).
 * The kernel reads its inputs and writes its output only after the preceding grid on
 * the stream has completed, so this is safe after any kernel; after the library's own
 * quantizer, which triggers early, the GEMM's prologue overlaps the quantizer's tail.
 */
int nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
               const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
               const void* bias_bf16, void* out_bf16, int64_t M, int64_t N, int64_t K,
               bsp_stream_t stream);

/*
 * nvfp4_gemm_quant -- nvfp4_gemm whose output is handed straight to the next nvfp4
 * linear: instead of writing Y in bf16, the epilogue quantizes bf16(Y) exactly as
 * nvfp4_quantize_act would (same block-16 arithmetic, global scale out_global) and
 * writes the codes and MMA-layout scales ("BFL (fp8r / nvfp4)", Kernels table: every
 * nvfp4 linear quantizes its activations; in an MLP the second linear's activations
 * are the first one's output).  Bit-identical to nvfp4_gemm followed by
 * nvfp4_quantize_act(Y, out_global, BSP_SF_MMA), without the bf16 round trip.
 *   out_global  device fp32: the next layer's input_scale.
 *   out_codes   [M][N/2] bytes, packed E2M1 ; out_sf  nvfp4_sf_bytes(M, N, BSP_SF_MMA)
 *               bytes (padding rows of the last 128-row tile are not written).
 * Other arguments as nvfp4_gemm.  Constraints: those of nvfp4_gemm and N % 64 == 0.
 * Always runs the CTA-pair kernel.
 */
int nvfp4_gemm_quant(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
                     const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
                     const void* bias_bf16, const float* out_global, uint8_t* out_codes,
                     uint8_t* out_sf, int64_t M, int64_t N, int64_t K, bsp_stream_t stream);

/*
 * nvfp4_linear -- the nvfp4 linear forward in one call ("BFL (fp8r / nvfp4)", Kernels
 * table: the activations are quantized at run time, then the fused FP4 GEMM runs):
 * nvfp4_quantize_act(x, input_scale) into `workspace` (BSP_SF_MMA scales), then
 * nvfp4_gemm against the pre-quantized weights.  The GEMM is launched with
 * programmatic stream serialisation, so its prologue overlaps the end of the
 * quantizer; it reads no input before the quantizer has completed.  Results are
 * bit-identical to the two separate calls.
 *
 *   x_bf16        [M][K] bf16 activations.
 *   input_scale   device pointer to one fp32: the activation global scale g.
 *   w_codes, w_sf, w_scale   the quantized weight: [N][K/2] codes, BSP_SF_MMA scales
 *                 (rows = N), device fp32 weight_scale_2.
 *   bias_bf16     [N] bf16 or NULL.   out_bf16  [M][N] bf16.
 *   workspace     caller-owned device buffer of at least
 *                 nvfp4_linear_workspace_bytes(M, K) bytes, 16-byte aligned.  It receives
 *                 the quantized activations (codes, then scales at a 256-byte boundary;
 *                 after them, at the next 256-byte boundary, 8 KB that
 *                 nvfp4_linear_dynamic uses for per-CTA maxima), is overwritten by every
 *                 call, and must not be in use by another call that can run at the same
 *                 time (another stream).
 * Constraints: K % 64 == 0, K >= 64, N % 8 == 0 (those of the two calls).
 * Errors: BSP_ERR_INVALID_ARG when workspace is NULL or workspace_bytes too small;
 * otherwise as nvfp4_quantize_act and nvfp4_gemm.
 */
int nvfp4_linear(const void* x_bf16, const float* input_scale, const uint8_t* w_codes,
                 const uint8_t* w_sf, const float* w_scale, const void* bias_bf16,
                 void* out_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                 int64_t workspace_bytes, bsp_stream_t stream);

/*
 * nvfp4_linear_dynamic -- nvfp4_linear with the activation global scale computed from
 * this call's activations instead of a calibrated constant ("BFL (fp8r / nvfp4)",
 * nvfp4 bullet: `input_scale` is an fp32 activation scale; here g = amax(x) / (448*6),
 * the global-scale convention used for the weights, the same value nvfp4_global_scale(x)
 * gives), then the nvfp4_linear path with it.  Two launches precede the GEMM: a pass over
 * x leaving one maximum of |x| per CTA in the workspace, and the quantizer, whose CTAs
 * reduce those maxima to g themselves; CTA 0 writes g to *input_scale_out, which the GEMM
 * then reads.  input_scale_out is a device fp32 the caller owns (4-byte aligned); it holds
 * g when the call's work completes.  Other arguments, workspace rules and errors as
 * nvfp4_linear.  Costs one more read of x than nvfp4_linear.
 */
int nvfp4_linear_dynamic(const void* x_bf16, float* input_scale_out, const uint8_t* w_codes,
                         const uint8_t* w_sf, const float* w_scale, const void* bias_bf16,
                         void* out_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                         int64_t workspace_bytes, bsp_stream_t stream);

/* Workspace bytes nvfp4_linear / nvfp4_linear_dynamic need for an [M][K] activation
 * (codes, padding to 256 bytes, MMA-layout scales, padding to 256 bytes, 8 KB of per-CTA
 * maxima); negative on bad arguments. */
int64_t nvfp4_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * nvfp4_linear_noalloc -- nvfp4_linear without a caller workspace and without any
 * allocation.  The pages have no counterpart: this is a deployment variant of
 * nvfp4_linear for callers that must not allocate device memory after start-up (a
 * serving loop with a fixed memory plan, C code without an allocator): cudaMalloc /
 * cudaFree can synchronise the device and fail under memory pressure.
 *
 * Arguments and results: those of nvfp4_linear minus workspace / workspace_bytes;
 * results are bit-identical to nvfp4_linear.  The quantized activations go to one
 * buffer of nvfp4_linear_noalloc_max_bytes() bytes (128 MiB) per device, compiled
 * into the library (a file-scope __device__ array).
 * Footprint: the buffer takes 128 MiB of device memory on every device where its
 * module is loaded, until the context is destroyed, even in a process that never
 * calls this function: at context creation under CUDA_MODULE_LOADING=EAGER, or at
 * the first call of this function on the device under lazy loading (the default).
 * Its address is looked up on the first call on each device (which may load the
 * module), so make that first call outside any stream capture; a lookup that fails
 * returns BSP_ERR_CUDA, leaves no pending CUDA error, and is retried by the next call.
 * Nothing in it needs to start at zero (each call writes what it reads).
 * Errors: BSP_ERR_UNSUPPORTED_SHAPE when nvfp4_linear_workspace_bytes(M, K) exceeds
 * the buffer; otherwise as nvfp4_linear.
 * Concurrency: the buffer is shared by all calls on a device, so calls that can run
 * at the same time (different streams, unordered host threads) race on it and
 * corrupt each other's results; calls ordered on one stream are safe.
 */
int nvfp4_linear_noalloc(const void* x_bf16, const float* input_scale, const uint8_t* w_codes,
                         const uint8_t* w_sf, const float* w_scale, const void* bias_bf16,
                         void* out_bf16, int64_t M, int64_t N, int64_t K, bsp_stream_t stream);

/* Size in bytes of nvfp4_linear_noalloc's per-device buffer (the largest workspace it
 * accepts). */
int64_t nvfp4_linear_noalloc_max_bytes(void);

/*
 * fp8r_quantize_rows -- per-row E4M3 quantizer ("BFL (fp8r / nvfp4)", fp8r bullet:
 * activations are quantized to E4M3 per row at run time; weights use one fp32 scale
 * per row).
 *   x_bf16 [M][K] bf16 ; q_e4m3 out [M][K] ; row_scale out [M] fp32.
 *   s_m = amax_m / 448 ; s_m == 0 -> q = 0 ; else q = E4M3(x * (1/s_m)), 1/s_m
 *   clamped to FLT_MAX.
 * Constraints: K % 8 == 0.
 */
int fp8r_quantize_rows(const void* x_bf16, int64_t M, int64_t K, uint8_t* q_e4m3,
                       float* row_scale, bsp_stream_t stream);

/*
 * fp8r_gemm -- row-scaled FP8 GEMM ("BFL (fp8r / nvfp4)", Kernels table: the fp8r
 * fused GEMM with per-row scales).
 *   a_e4m3 [M][K], a_row_scale [M]; w_e4m3 [N][K], w_row_scale [N]; bias [N] or NULL.
 *   Y[m][n] = bf16( (acc[m][n] * sA[m]) * sW[n] + bias[n] ), acc in fp32 on the
 *   tensor cores.
 * Constraints: K % 16 == 0, K >= 16; N % 8 == 0.  Any M >= 0.
 */
int fp8r_gemm(const uint8_t* a_e4m3, const float* a_row_scale, const uint8_t* w_e4m3,
              const float* w_row_scale, const void* bias_bf16, void* out_bf16, int64_t M,
              int64_t N, int64_t K, bsp_stream_t stream);

/*
 * fp8r_linear -- the fp8r linear forward in one call ("BFL (fp8r / nvfp4)", fp8r bullet
 * and Kernels table: activations quantized to E4M3 per row at run time, then the
 * row-scaled FP8 GEMM): fp8r_quantize_rows(x) into `workspace`, then fp8r_gemm (launched
 * as the quantizer's programmatic dependent).  Results are bit-identical to the two calls.
 *   x_bf16 [M][K] bf16 ; w_e4m3 [N][K] ; w_row_scale [N] fp32 ; bias [N] bf16 or NULL ;
 *   out_bf16 [M][N].
 *   workspace  caller-owned device buffer of at least fp8r_linear_workspace_bytes(M, K)
 *              bytes, 16-byte aligned (codes, then the row scales at a 256-byte boundary);
 *              fully rewritten by each call; not shared by calls that can run at the same
 *              time.
 * Constraints: those of fp8r_quantize_rows and fp8r_gemm.  Errors as those two, and
 * BSP_ERR_INVALID_ARG for a missing or too small workspace.
 */
int fp8r_linear(const void* x_bf16, const uint8_t* w_e4m3, const float* w_row_scale,
                const void* bias_bf16, void* out_bf16, int64_t M, int64_t N, int64_t K,
                void* workspace, int64_t workspace_bytes, bsp_stream_t stream);

/* Workspace bytes fp8r_linear needs for an [M][K] activation; negative on bad arguments. */
int64_t fp8r_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * nvfp4_global_scale -- g = amax(X) / (448 * 6) over n bf16 values, written to the
 * device fp32 at `global_scale_out` (the nvfp4 `weight_scale_2` / `input_scale`
 * convention: a decode-side multiplier that maps the largest block scale to the
 * E4M3 maximum).  Enqueues a clear of the output, an atomic max over the input and a
 * final divide; no scratch memory.  Constraints: n % 8 == 0.
 */
int nvfp4_global_scale(const void* x_bf16, int64_t n, float* global_scale_out,
                       bsp_stream_t stream);

/*
 * nvfp4_dequantize -- decode NVFP4 to bf16: the weight decode of the dequantise-only
 * fallback ("BFL (fp8r / nvfp4)", closing paragraph of the "Kernels" section: weights are
 * dequantized back to bf16 and the GEMM runs in bf16 on activations that are not
 * quantized, so results differ slightly from the fused path).  Per element, in binary32
 * with round to nearest even and no flush to zero:
 *     out = bf16_rne( (e2m1(code) * e4m3(scale)) * g )
 * (the first product is exact).  Not on the fused hot path; provided for comparison and
 * for callers that need bf16 weights.
 *   codes         [rows][K/2] packed E2M1 (element 2j in the low nibble)
 *   scales        E4M3 block scales in `layout` (BSP_SF_LINEAR [rows][K/16] or BSP_SF_MMA)
 *   global_scale  device fp32, 1 element (weight_scale_2 or input_scale)
 *   out_bf16      [rows][K] bf16, caller-owned
 * Constraints: K % 16 == 0 (K % 64 == 0 for BSP_SF_MMA); codes and out 16-byte aligned,
 * global_scale 4-byte aligned; scale bytes finite (a NaN scale gives NaN elements).
 * Errors: BSP_ERR_INVALID_ARG, BSP_ERR_UNSUPPORTED_SHAPE, BSP_ERR_MISALIGNED,
 * BSP_ERR_UNSUPPORTED_DEVICE, BSP_ERR_CUDA.  Asynchronous on `stream`; no allocation.
 */
int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int layout,
                     const float* global_scale, int64_t rows, int64_t K, void* out_bf16,
                     bsp_stream_t stream);

/*
 * nvfp4_sf_convert -- re-lay block scales between BSP_SF_LINEAR and BSP_SF_MMA
 * (rows x K/16 bytes; padding of an MMA-layout destination is written as 0).
 * Constraints: K % 64 == 0.  src and dst must not overlap.
 */
int nvfp4_sf_convert(const uint8_t* src, uint8_t* dst, int64_t rows, int64_t K, int from,
                     int to, bsp_stream_t stream);

/* Bytes of a scale array of `rows` x K/16 in `layout`; negative on bad arguments. */
int64_t nvfp4_sf_bytes(int64_t rows, int64_t K, int layout);

/*
 * bsp_last_device_status -- synchronises `stream`, returns and clears the status
 * word the kernels of the current device write (BSP_OK, or BSP_ERR_TIMEOUT when a
 * bounded wait inside a GEMM ran out).  BSP_ERR_CUDA if the synchronisation fails.
 */
int bsp_last_device_status(bsp_stream_t stream);

/* Bounded-wait limit of the GEMM kernels in milliseconds (default 2000, also set by
 * the BSP_WAIT_LIMIT_MS environment variable at first use): the longest any one wait on a
 * pipeline stage or tile may take.  (The fp8r kernel's last-tile helpers wait once for the
 * whole GEMM's issue; that wait is bounded by the larger of this limit and 60 s.)  Returns
 * the old value. */
int64_t bsp_set_wait_limit_ms(int64_t ms);

/* Human-readable name of a bsp_status value. */
const char* bsp_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int bsp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSP_H_ */
