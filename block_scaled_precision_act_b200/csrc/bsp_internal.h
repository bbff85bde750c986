// bsp_internal.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "bsp.h"

namespace bsp {

// Returns BSP_OK when the current device is compute capability 10.0; caches per device.
int check_device(int* device_out, int* num_sms_out);

// Device address of the current device's status word (int[2]: code, where).
int* device_status_ptr(int device);

// Bounded-wait limit for kernels, in nanoseconds.
uint64_t wait_limit_ns();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status()
{
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
}

}  // namespace bsp
