// linear_noalloc.cu -- nvfp4_linear_noalloc: nvfp4_linear with its workspace taken
// from a fixed buffer compiled into the library instead of from the caller.
//
// Who needs it: a caller that must not allocate device memory once it is running,
// and cannot hand in a workspace either -- for example a serving loop with a memory
// plan fixed at start-up, or C code linked against the library that has no allocator
// of its own.  cudaMalloc / cudaFree can synchronise the device and can fail under
// memory pressure, so such callers keep them off the hot path.  This entry point
// performs no allocation of any kind: no cudaMalloc, no cudaFree, no torch tensor.
//
// The buffer is g_linear_scratch below: kNoallocScratchBytes (128 MiB) per device, a
// file-scope __device__ array.  Its device address is looked up with
// cudaGetSymbolAddress on the first call made on each device and cached; that lookup
// loads this file's module if it is not loaded yet, so make the first call on each
// device outside any stream capture.  Problems whose workspace
// (nvfp4_linear_workspace_bytes(M, K)) exceeds the buffer are rejected with
// BSP_ERR_UNSUPPORTED_SHAPE.  Nothing in the buffer has to start at zero: every
// byte the GEMM reads is written first by the quantizer of the same call.
//
// There is ONE buffer per device, shared by every call on that device: two calls that
// can run at the same time (different streams, or different host threads on streams
// that are not ordered) race on it and corrupt each other's results.  Calls on one
// stream are ordered and safe.
#include <cstdint>
#include <mutex>

#include "bsp_internal.h"

namespace bsp {
namespace {

constexpr int64_t kNoallocScratchBytes = int64_t{128} << 20;

__device__ __align__(256) uint8_t g_linear_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::once_flag g_scratch_once[kMaxDevices];
void* g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

}  // namespace
}  // namespace bsp

extern "C" {

int64_t nvfp4_linear_noalloc_max_bytes(void) { return bsp::kNoallocScratchBytes; }

int nvfp4_linear_noalloc(const void* x_bf16, const float* input_scale, const uint8_t* w_codes,
                         const uint8_t* w_sf, const float* w_scale, const void* bias_bf16,
                         void* out_bf16, int64_t M, int64_t N, int64_t K, bsp_stream_t stream)
{
    using namespace bsp;
    if (M < 0 || N < 0 || K <= 0) return BSP_ERR_INVALID_ARG;
    if (K % 64 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return BSP_OK;
    const int64_t need = nvfp4_linear_workspace_bytes(M, K);
    if (need < 0) return static_cast<int>(need);
    if (need > kNoallocScratchBytes) return BSP_ERR_UNSUPPORTED_SHAPE;
    int dev = 0;
    int st = check_device(&dev, nullptr);
    if (st != BSP_OK) return st;
    if (dev < 0 || dev >= kMaxDevices) return BSP_ERR_UNSUPPORTED_DEVICE;
    std::call_once(g_scratch_once[dev], [dev] {
        g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_addr[dev], g_linear_scratch);
    });
    if (g_scratch_err[dev] != cudaSuccess || g_scratch_addr[dev] == nullptr) return BSP_ERR_CUDA;
    return nvfp4_linear(x_bf16, input_scale, w_codes, w_sf, w_scale, bias_bf16, out_bf16, M, N,
                        K, g_scratch_addr[dev], kNoallocScratchBytes, stream);
}

}  // extern "C"
