// bsp_internal.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "bsp.h"

namespace bsp {

// Devices the library keeps per-device state for (ids 0 .. kMaxDevices - 1; check_device
// refuses others before any of that state is touched).
constexpr int kMaxDevices = 64;

// Returns BSP_OK when the current device is compute capability 10.0; caches per device.
int check_device(int* device_out, int* num_sms_out);

// Device address of the current device's status word (int[2]: code, where).
int* device_status_ptr(int device);

// Bounded-wait limit for kernels, in nanoseconds.
uint64_t wait_limit_ns();

// nvfp4_gemm (nvf4) / fp8r_gemm launched right after the library's activation quantizer
// wrote `a` (and `a_sf`): same results, but the weight operand's first stages are fetched
// while that quantizer finishes (the quantizer never writes the weights).
int gemm_after_quantizer(bool nvf4, const uint8_t* a, const uint8_t* a_sf, const float* a_scale,
                         const uint8_t* w, const uint8_t* w_sf, const float* w_scale,
                         const void* bias_bf16, void* out_bf16, int64_t M, int64_t N, int64_t K,
                         bsp_stream_t stream);

// nvfp4_quantize_act with an optional per-call global scale: when `partials` is not null,
// g is reduced from the `npartials` per-CTA maxima of |x| there (fp32 bit patterns) and
// published at `gout`; `global_scale` is then unused.
int quantize_act_impl(const void* x_bf16, int64_t M, int64_t K, const float* global_scale,
                      uint8_t* codes, uint8_t* scales, int layout, bsp_stream_t stream,
                      const uint32_t* partials, int npartials, float* gout);

// Slots of per-CTA maxima the dynamic path keeps in the linear workspace.
constexpr int kDynamicPartials = 2048;

// amax pass into `partials`, then the quantizer reducing them (MMA scale layout).
int dynamic_quantize_front(const void* x_bf16, int64_t M, int64_t K, uint32_t* partials,
                           float* g_out, uint8_t* codes, uint8_t* scales, bsp_stream_t stream);

// Launch `kernel`; with `pdl` the launch allows programmatic stream serialisation, so
// the grid may start (prologue: barriers, TMEM, tensor-map prefetch, or just being
// scheduled) while the preceding grid in the stream finishes.  Every kernel launched
// this way executes griddep_wait() before its first read of an input or write of an
// output.
template <typename... Params, typename... Args>
cudaError_t launch_kernel(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem,
                          cudaStream_t s, bool pdl, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(block, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status()
{
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
}

}  // namespace bsp
