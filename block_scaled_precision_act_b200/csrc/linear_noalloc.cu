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
// file-scope __device__ array.  It occupies 128 MiB of device memory on every device
// where this file's module is loaded, from the load until the context is destroyed,
// whether or not this entry point is ever called there: with eager module loading
// (CUDA_MODULE_LOADING=EAGER) the load happens when the library's context is created;
// with lazy loading (the default) it happens at the first cudaGetSymbolAddress below.
// Its device address is looked up with cudaGetSymbolAddress on the first successful
// call made on each device and cached; that lookup may load the module, so make the
// first call on each device outside any stream capture.  A lookup that fails (for
// example inside a capture) is not cached: the call returns BSP_ERR_CUDA, the runtime
// error it raised is cleared, and the next call tries again.  Problems whose workspace
// (nvfp4_linear_workspace_bytes(M, K)) exceeds the buffer are rejected with
// BSP_ERR_UNSUPPORTED_SHAPE.  Nothing in the buffer has to start at zero: every
// byte the GEMM reads is written first by the quantizer of the same call.
//
// There is ONE buffer per device, shared by every call on that device: two calls that
// can run at the same time (different streams, or different host threads on streams
// that are not ordered) race on it and corrupt each other's results.  Calls on one
// stream are ordered and safe.
#include <atomic>
#include <cstdint>
#include <mutex>

#include "bsp_internal.h"

namespace bsp {
namespace {

constexpr int64_t kNoallocScratchBytes = int64_t{128} << 20;

__device__ __align__(256) uint8_t g_linear_scratch[kNoallocScratchBytes];

std::atomic<void*> g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the current device's buffer (the caller made `dev` current), or
// nullptr when the lookup failed; a failure leaves no pending runtime error behind.
void* scratch_address(int dev)
{
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p != nullptr) return p;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (p != nullptr) return p;
    if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return nullptr;
    }
    g_scratch_addr[dev].store(p, std::memory_order_release);
    return p;
}

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
    void* scratch = scratch_address(dev);
    if (scratch == nullptr) return BSP_ERR_CUDA;
    return nvfp4_linear(x_bf16, input_scale, w_codes, w_sf, w_scale, bias_bf16, out_bf16, M, N,
                        K, scratch, kNoallocScratchBytes, stream);
}

}  // extern "C"
