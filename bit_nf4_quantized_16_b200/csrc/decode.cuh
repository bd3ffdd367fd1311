// Forward pass of the QLoRA linear for a handful of tokens (decode shape):
// split-contraction GEMV over the packed weight plus a finalize kernel.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace qlora {

// Largest token count served by the decode kernels.
constexpr int kDecodeMaxTokens = 16;

// Workspace the decode forward needs (fp32 partial products of every split).
size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K, int r, int sms);

// Y = X W'^T + (s Xa A^T) B^T for 1 <= M <= kDecodeMaxTokens (Xa = X, or the
// dropped-out input under LoRA dropout); H_save (nullable) receives s Xa A^T in
// fp32; f16: the fp16 compute dtype (X, Xa, A, B fp16; y_dtype QLORA_FP16 or
// QLORA_FP32).  Arguments already validated by the caller.
qlora_status run_decode_fwd(const qlora_nf4_weight *w, const void *X, const void *Xa, int64_t M, const void *A,
                            const void *B, int r, float scale, void *Y, qlora_dtype y_dtype, float *H_save, void *ws,
                            size_t ws_bytes, const DeviceInfo &dev, cudaStream_t s, bool f16 = false);

}  // namespace qlora
