// host_common.h -- host-side helpers shared by the entry points: status
// mapping, argument checks, device properties.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "nvfp4.h"

namespace nvfp4 {

// Device ordinals the per-device caches below can hold.
constexpr int kMaxDevices = 64;

// Ordinal of the calling thread's current device, or NVFP4_ERR_CUDA when it
// cannot be read or lies beyond the caches.
inline nvfp4_status current_device(int* dev) {
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

// One-time, per-device set-up that several host threads may reach at once
// (cached device properties, symbol addresses, kernel attributes).  The first
// caller runs `init` under a lock; a success is published with release order,
// so a later caller that sees it (acquire) also sees everything `init` wrote.
// A failed `init` is not recorded and runs again on the next call.
class PerDeviceOnce {
  public:
    template <class F>
    nvfp4_status run(int dev, F&& init) {
        if (done_[dev].load(std::memory_order_acquire)) return NVFP4_OK;
        std::lock_guard<std::mutex> lock(mu_);
        if (done_[dev].load(std::memory_order_relaxed)) return NVFP4_OK;
        const nvfp4_status st = init();
        if (st == NVFP4_OK) done_[dev].store(true, std::memory_order_release);
        return st;
    }

  private:
    std::atomic<bool> done_[kMaxDevices] = {};
    std::mutex mu_;
};

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// True when [p, p + pn) and [q, q + qn) share a byte (either may be null).
inline bool overlaps(const void* p, size_t pn, const void* q, size_t qn) {
    if (!p || !q) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + qn && b < a + pn;
}

// Bytes spanned by a row-major [rows, cols] matrix with row stride ld, all
// counted in elements of elem_bytes (0 when empty).  Callers have bounded
// rows and ld with extent_too_large first.
inline size_t extent_bytes(int64_t rows, int64_t ld, int64_t cols, int64_t elem_bytes) {
    if (rows <= 0 || cols <= 0) return 0;
    return static_cast<size_t>(((rows - 1) * ld + cols) * elem_bytes);
}

// True when `rows` rows `ld` elements apart, of elem_bytes each, would span
// more than 2^48 bytes -- more than any device address space.  Checked before
// any stride or size arithmetic on caller values (rows, ld >= 0), so that
// none of it can overflow int64.
inline bool extent_too_large(int64_t rows, int64_t ld, int64_t elem_bytes) {
    constexpr int64_t kMaxBytes = int64_t(1) << 48;
    if (rows <= 0 || ld <= 0) return false;
    return ld > kMaxBytes / elem_bytes || rows > kMaxBytes / (ld * elem_bytes);
}

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
