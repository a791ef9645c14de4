// echo_host.h -- host-side helpers shared by the plans: config checks,
// the device guard, CUDA error mapping.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "echo.h"

namespace echo {

// Checks every field of *c (shared by both kinds of plan).
echo_status validate_config(const echo_config *c);

// Restores the caller's current device on scope exit.
struct DeviceGuard {
    int prev = -1;
    cudaError_t err = cudaSuccess;
    explicit DeviceGuard(int dev) {
        err = cudaGetDevice(&prev);
        if (err == cudaSuccess && prev != dev) err = cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

inline echo_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return ECHO_OK;
    if (e == cudaErrorMemoryAllocation) return ECHO_ERR_OOM;
    return ECHO_ERR_CUDA;
}

inline bool aligned16(const void *ptr) { return ((uintptr_t)ptr & 15u) == 0; }
inline bool aligned4(const void *ptr) { return ((uintptr_t)ptr & 3u) == 0; }

// Whether st is capturing into a CUDA graph (false if the query fails: the
// launches that follow then report the error).
inline bool capturing(cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return cs != cudaStreamCaptureStatusNone;
}

}  // namespace echo

#define ECHO_TRY(expr)                                     \
    do {                                                   \
        cudaError_t e_ = (expr);                           \
        if (e_ != cudaSuccess) return echo::from_cuda(e_); \
    } while (0)
