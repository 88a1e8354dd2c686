// host_common.h -- host-side helpers shared by the entry points: status
// mapping, argument checks, device properties.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "nvfp4.h"

namespace nvfp4 {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Multiprocessor count and compute capability of the current device, cached
// per device ordinal.
struct DeviceInfo {
    int sms = 0;
    int major = 0;
    int minor = 0;
};

nvfp4_status current_device_info(DeviceInfo* info);

// Device address of the library's status word (set by kernels whose bounded
// waits gave up), looked up once per device; nullptr on a CUDA error.
int* device_status_ptr();

// The block-scaled FP4 tensor-core path needs an sm_100 device.
inline nvfp4_status require_sm100(DeviceInfo* info) {
    nvfp4_status st = current_device_info(info);
    if (st != NVFP4_OK) return st;
    return info->major == 10 ? NVFP4_OK : NVFP4_ERR_DEVICE;
}

}  // namespace nvfp4
