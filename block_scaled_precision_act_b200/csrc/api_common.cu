// api_common.cu -- device checks, the per-device status word, status strings.
#include <atomic>
#include <cstdlib>
#include <mutex>

#include "bsp_internal.h"

namespace {

// Written by kernels when a bounded wait runs out: {status code, wait site}.
__device__ int g_bsp_status[2];

using bsp::kMaxDevices;
std::once_flag g_dev_once[kMaxDevices];
int g_dev_ok[kMaxDevices];
int g_dev_sms[kMaxDevices];
int* g_dev_status[kMaxDevices];

std::atomic<int64_t> g_wait_limit_ms{-1};

void probe_device(int dev)
{
    int major = 0, minor = 0, sms = 0;
    g_dev_ok[dev] = BSP_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    if (major != 10 || minor != 0) {
        g_dev_ok[dev] = BSP_ERR_UNSUPPORTED_DEVICE;
        return;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bsp_status) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    g_dev_status[dev] = static_cast<int*>(p);
    g_dev_sms[dev] = sms;
    g_dev_ok[dev] = BSP_OK;
}

}  // namespace

namespace bsp {

int check_device(int* device_out, int* num_sms_out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return BSP_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return BSP_ERR_UNSUPPORTED_DEVICE;
    std::call_once(g_dev_once[dev], probe_device, dev);
    if (device_out) *device_out = dev;
    if (num_sms_out) *num_sms_out = g_dev_sms[dev];
    return g_dev_ok[dev];
}

int* device_status_ptr(int device) { return g_dev_status[device]; }

uint64_t wait_limit_ns()
{
    int64_t ms = g_wait_limit_ms.load();
    if (ms < 0) {
        const char* e = std::getenv("BSP_WAIT_LIMIT_MS");
        int64_t v = e ? std::atoll(e) : 0;
        ms = v > 0 ? v : 2000;
        int64_t expected = -1;
        g_wait_limit_ms.compare_exchange_strong(expected, ms);
        ms = g_wait_limit_ms.load();
    }
    return static_cast<uint64_t>(ms) * 1000000ull;
}

}  // namespace bsp

extern "C" {

int64_t bsp_set_wait_limit_ms(int64_t ms)
{
    const int64_t old = static_cast<int64_t>(bsp::wait_limit_ns() / 1000000ull);
    if (ms > 0) g_wait_limit_ms.store(ms);
    return old;
}

int bsp_last_device_status(bsp_stream_t stream)
{
    int dev = 0;
    int st = bsp::check_device(&dev, nullptr);
    if (st != BSP_OK) return st;
    int host[2] = {0, 0};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(host, bsp::device_status_ptr(dev), sizeof(host),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return BSP_ERR_CUDA;
    }
    if (host[0] != 0) {
        const int zero[2] = {0, 0};
        if (cudaMemcpyAsync(bsp::device_status_ptr(dev), zero, sizeof(zero),
                            cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess) {
            cudaGetLastError();
            return BSP_ERR_CUDA;
        }
    }
    return host[0];
}

const char* bsp_status_string(int status)
{
    switch (status) {
        case BSP_OK: return "BSP_OK";
        case BSP_ERR_INVALID_ARG: return "BSP_ERR_INVALID_ARG";
        case BSP_ERR_UNSUPPORTED_SHAPE: return "BSP_ERR_UNSUPPORTED_SHAPE";
        case BSP_ERR_MISALIGNED: return "BSP_ERR_MISALIGNED";
        case BSP_ERR_UNSUPPORTED_DEVICE: return "BSP_ERR_UNSUPPORTED_DEVICE";
        case BSP_ERR_CUDA: return "BSP_ERR_CUDA";
        case BSP_ERR_TIMEOUT: return "BSP_ERR_TIMEOUT";
        default: return "BSP_ERR_UNKNOWN";
    }
}

int bsp_version(void) { return 200; }

int64_t nvfp4_sf_bytes(int64_t rows, int64_t K, int layout)
{
    if (rows < 0 || K < 0 || K % 16 != 0) return BSP_ERR_INVALID_ARG;
    const int64_t nb = K / 16;
    if (layout == BSP_SF_LINEAR) return rows * nb;
    if (layout == BSP_SF_MMA) return ((rows + 127) / 128) * ((nb + 3) / 4) * 512;
    return BSP_ERR_INVALID_ARG;
}

}  // extern "C"
