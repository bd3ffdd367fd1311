// QLoRA linear layer (forward and backward): placeholder entry points until
// the tcgen05 kernels land.
#include "common.cuh"

extern "C" size_t qlora_linear_workspace_bytes(int64_t, int64_t, int64_t, int32_t) { return 0; }

extern "C" qlora_status qlora_linear_fwd(const qlora_nf4_weight *, const void *, int64_t, const void *,
                                         const void *, int32_t, float, void *, qlora_dtype, float *, void *,
                                         size_t, void *)
{
    return QLORA_ERR_UNSUPPORTED;
}

extern "C" qlora_status qlora_linear_bwd(const qlora_nf4_weight *, const void *, const void *, int64_t,
                                         const void *, const void *, int32_t, float, const float *, void *,
                                         qlora_dtype, float *, float *, void *, size_t, void *)
{
    return QLORA_ERR_UNSUPPORTED;
}
