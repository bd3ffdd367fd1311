// Shared host-side plumbing of the QLoRA library: status handling, argument
// checks, device properties and the device error word.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/qlora.h"

namespace qlora {

constexpr int kMaxDevices = 64;

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

// Launch with programmatic stream serialization (kernels of the linear path):
// the kernel's set-up overlaps the tail of the kernel before it, and the kernel
// waits (griddepcontrol.wait) before reading anything that kernel produced.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args &&...args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// 2-D row-major tensor map: `inner` elements per row (contiguous), `rows` rows,
// `pitch_bytes` between rows; box = box_inner x box_rows elements.
qlora_status make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw);

// Checks shared by every entry point that takes a quantized weight.
qlora_status check_weight(const qlora_nf4_weight *w);

// Per-device one-time set-up (kernel attributes, occupancy queries): the first
// successful run of `fn` on a device happens under a lock; later calls on that
// device return at once.  The results of `fn` are published by the release
// store of the done flag.
class PerDeviceOnce {
  public:
    template <typename F>
    qlora_status run(int device, F &&fn)
    {
        if (device < 0 || device >= kMaxDevices) return QLORA_ERR_CUDA;
        if (done_[device].load(std::memory_order_acquire)) return QLORA_OK;
        std::lock_guard<std::mutex> lock(mu_);
        if (done_[device].load(std::memory_order_relaxed)) return QLORA_OK;
        const qlora_status st = fn();
        if (st == QLORA_OK) done_[device].store(true, std::memory_order_release);
        return st;
    }

  private:
    std::mutex mu_;
    std::atomic<bool> done_[kMaxDevices] = {};
};

// Failure-detection test hook (qlora_debug_inject_stall): true, once, for the
// first launch of kernel family `kind` after the hook was armed; *timeout_ns
// then receives the armed wait limit.
bool take_stall_injection(int kind, uint64_t *timeout_ns);

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
