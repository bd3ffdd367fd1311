// Paged optimizer for the LoRA adapters on sm_100a.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs", Introduction item (3) and
// section "Method" (opening paragraph): the optimizer states live in NVIDIA
// unified memory, so that the driver evicts them to CPU RAM when the GPU runs
// short of memory and pages them back when the update step touches them; the
// mbrenndoerfer.com essay, section "Paged Optimizers", describes the same
// mechanism (CPU memory as a buffer for the optimizer states during memory
// spikes).  The pages name no optimizer; the update is Adam with decoupled
// weight decay (AdamW), whose two states per parameter (first and second
// moment) are what gets paged.
//
// Pieces:
//   qlora_paged_alloc / qlora_paged_free   unified (managed) allocations for the states
//   qlora_paged_prefetch                   explicit migration to the GPU or to the host
//   qlora_adamw_step                       one fused AdamW update over a flat parameter vector:
//                                          reads grad, param, m, v; writes param, m, v and an
//                                          optional bf16 copy of the parameters (the adapters
//                                          the linear layer reads); 30 bytes per parameter.
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "sm100.cuh"

namespace qlora {
namespace {

struct AdamWArgs {
    float *p;
    __nv_bfloat16 *p16;   // nullable
    const float *g;
    float *m;
    float *v;
    int64_t n;
    float decay;          // 1 - lr * weight_decay
    float beta1, one_minus_beta1;
    float beta2, one_minus_beta2;
    float step_size;      // lr / (1 - beta1^t)
    float bc2_sqrt;       // sqrt(1 - beta2^t)
    float eps;
};

__device__ __forceinline__ float adamw_one(float p, float g, float &m, float &v, const AdamWArgs &a)
{
    p = __fmul_rn(p, a.decay);
    m = __fmaf_rn(a.beta1, m, __fmul_rn(a.one_minus_beta1, g));
    v = __fmaf_rn(a.beta2, v, __fmul_rn(a.one_minus_beta2, __fmul_rn(g, g)));
    const float denom = __fadd_rn(__fdiv_rn(__fsqrt_rn(v), a.bc2_sqrt), a.eps);
    return __fsub_rn(p, __fmul_rn(a.step_size, __fdiv_rn(m, denom)));
}

__device__ __forceinline__ float4 ld_stream_f4(const float *p)
{
    float4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

// Four parameters per thread and step; the grid covers the vector in a few
// waves.  Managed pages that live on the host migrate on first touch.
__global__ void __launch_bounds__(256) adamw_kernel(const AdamWArgs a)
{
    sm100::pdl_wait();   // the gradients come from the kernels before this one
    sm100::pdl_trigger();
    const int64_t n4 = a.n / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 g = ld_stream_f4(a.g + 4 * i);
        float4 p = *reinterpret_cast<const float4 *>(a.p + 4 * i);
        float4 m = *reinterpret_cast<const float4 *>(a.m + 4 * i);
        float4 v = *reinterpret_cast<const float4 *>(a.v + 4 * i);
        p.x = adamw_one(p.x, g.x, m.x, v.x, a);
        p.y = adamw_one(p.y, g.y, m.y, v.y, a);
        p.z = adamw_one(p.z, g.z, m.z, v.z, a);
        p.w = adamw_one(p.w, g.w, m.w, v.w, a);
        *reinterpret_cast<float4 *>(a.p + 4 * i) = p;
        *reinterpret_cast<float4 *>(a.m + 4 * i) = m;
        *reinterpret_cast<float4 *>(a.v + 4 * i) = v;
        if (a.p16) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(p.x, p.y), hi = __floats2bfloat162_rn(p.z, p.w);
            uint2 w;
            w.x = *reinterpret_cast<uint32_t *>(&lo);
            w.y = *reinterpret_cast<uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(a.p16 + 4 * i) = w;
        }
    }
    // the last n % 4 parameters
    const int64_t t = 4 * n4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t < a.n) {
        float m = a.m[t], v = a.v[t];
        const float p = adamw_one(a.p[t], a.g[t], m, v, a);
        a.p[t] = p;
        a.m[t] = m;
        a.v[t] = v;
        if (a.p16) a.p16[t] = __float2bfloat16_rn(p);
    }
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" qlora_status qlora_paged_alloc(size_t bytes, void **ptr)
{
    if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
    *ptr = nullptr;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    void *p = nullptr;
    if (cudaMallocManaged(&p, bytes, cudaMemAttachGlobal) != cudaSuccess) return QLORA_ERR_CUDA;
    // zero on the host: the pages start out in CPU memory and move to the GPU
    // when a prefetch or the first update touches them
    memset(p, 0, bytes);
    *ptr = p;
    return QLORA_OK;
}

extern "C" qlora_status qlora_paged_free(void *ptr)
{
    if (!ptr) return QLORA_OK;
    return cudaFree(ptr) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

extern "C" qlora_status qlora_paged_prefetch(const void *ptr, size_t bytes, int to_device, void *stream)
{
    if (!ptr || (to_device != 0 && to_device != 1)) return QLORA_ERR_INVALID_ARG;
    if (bytes == 0) return QLORA_OK;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    const int dst = to_device ? dev.device : cudaCpuDeviceId;
    QLORA_CUDA_TRY(cudaMemPrefetchAsync(ptr, bytes, dst, static_cast<cudaStream_t>(stream)));
    return QLORA_OK;
}

extern "C" qlora_status qlora_adamw_step(float *param, void *param_bf16, const float *grad, float *exp_avg,
                                         float *exp_avg_sq, int64_t n, const qlora_adamw_hparams *h, void *stream)
{
    if (!param || !grad || !exp_avg || !exp_avg_sq || !h) return QLORA_ERR_INVALID_ARG;
    if (n < 0 || h->step < 1) return QLORA_ERR_INVALID_ARG;
    if (!(h->lr >= 0.0f) || !(h->beta1 >= 0.0f && h->beta1 < 1.0f) || !(h->beta2 >= 0.0f && h->beta2 < 1.0f) ||
        !(h->eps > 0.0f) || !(h->weight_decay >= 0.0f))
        return QLORA_ERR_INVALID_ARG;
    if (!aligned16(param) || !aligned16(grad) || !aligned16(exp_avg) || !aligned16(exp_avg_sq) ||
        (param_bf16 && (reinterpret_cast<uintptr_t>(param_bf16) & 7u)))
        return QLORA_ERR_ALIGNMENT;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    if (n == 0) return QLORA_OK;
    AdamWArgs a;
    a.p = param;
    a.p16 = static_cast<__nv_bfloat16 *>(param_bf16);
    a.g = grad;
    a.m = exp_avg;
    a.v = exp_avg_sq;
    a.n = n;
    // the scalars of step t, formed in double and rounded once
    const double t = (double)h->step;
    a.decay = (float)(1.0 - (double)h->lr * (double)h->weight_decay);
    a.beta1 = h->beta1;
    a.one_minus_beta1 = (float)(1.0 - (double)h->beta1);
    a.beta2 = h->beta2;
    a.one_minus_beta2 = (float)(1.0 - (double)h->beta2);
    a.step_size = (float)((double)h->lr / (1.0 - pow((double)h->beta1, t)));
    a.bc2_sqrt = (float)sqrt(1.0 - pow((double)h->beta2, t));
    a.eps = h->eps;
    const int64_t n4 = (n + 3) / 4;
    int64_t grid = (n4 + 255) / 256;
    const int64_t cap = (int64_t)dev.sms * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        LaunchScope ls(QLORA_KERNEL_OPTIMIZER, s);
        QLORA_CUDA_TRY(launch_pdl(adamw_kernel, dim3((unsigned)grid), dim3(256), 0, s, a));
    }
    return launch_status();
}
