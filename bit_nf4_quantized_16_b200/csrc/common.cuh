// Shared host-side plumbing of the QLoRA library: status handling, argument
// checks, device properties and the device error word.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qlora.h"

namespace qlora {

// Kernel-side error codes written into the device error word.
enum DeviceError : int {
    kDevOk = 0,
    kDevTimeout = 1,   // a bounded mbarrier wait gave up
};

// Device address of this device's error word (set-up on first use).
int *device_error_word();

// Number of SMs and compute capability of the current device (cached).
struct DeviceInfo {
    int device;
    int sms;
    int major, minor;
    size_t smem_optin;
};
qlora_status device_info(DeviceInfo *out);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define QLORA_CUDA_TRY(expr)                                  \
    do {                                                      \
        cudaError_t err__ = (expr);                           \
        if (err__ != cudaSuccess) return QLORA_ERR_CUDA;      \
    } while (0)

#define QLORA_TRY(expr)                                       \
    do {                                                      \
        qlora_status st__ = (expr);                           \
        if (st__ != QLORA_OK) return st__;                    \
    } while (0)

// Launch-error check after a kernel launch.
inline qlora_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// Checks shared by every entry point that takes a quantized weight.
qlora_status check_weight(const qlora_nf4_weight *w);

// Brackets one kernel launch for qlora_timing_read (events only while timing
// is enabled) and counts it for qlora_launch_count.
class LaunchScope {
  public:
    LaunchScope(int kind, cudaStream_t s);
    ~LaunchScope();

  private:
    int kind_;
    cudaStream_t s_;
    cudaEvent_t start_ = nullptr;
};

}  // namespace qlora
