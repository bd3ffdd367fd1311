// Expansion of packed 4-bit codes to bf16: the arithmetic of dequantization
// ("QLoRA: Efficient Finetuning of Quantized LLMs", section "Method": the
// stored weight is dequantized to BFloat16 before the 16-bit matmul), shared
// by the stand-alone dequantizer and the fused GEMM's producer warps so that
// both produce the same bits.
//
// Per block of 64 weights: c1' = fmaf(E4M3value(code2), c2, mean); per weight:
// w = bf16_RNE(RN32(q[code] * c1')) (fp16_RNE for the fp16 compute dtype).
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace qlora {
namespace nf4 {

__device__ __forceinline__ float e4m3_to_float(uint8_t code)
{
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
    return __half2float(__half(h));
}

// c1' = RN32(E4M3value(e) * c2 + mean), one rounding
__device__ __forceinline__ float block_scale(uint8_t e, float c2, float mean)
{
    return __fmaf_rn(e4m3_to_float(e), c2, mean);
}

// Two binary32 values rounded to nearest-even bf16, lo in bits 0-15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Two binary32 values rounded to nearest-even binary16, lo in bits 0-15.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// The 16-bit compute type's pair packing: bf16 (default) or fp16.
template <bool F16>
__device__ __forceinline__ uint32_t pack16x2(float lo, float hi)
{
    if constexpr (F16)
        return pack_f16x2(lo, hi);
    else
        return pack_bf16x2(lo, hi);
}

// (a, b) * (s, s), each lane an IEEE round-to-nearest-even product.
__device__ __forceinline__ void mul2(float a, float b, float s, float &ra, float &rb)
{
    uint64_t x, y, ss;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a), "f"(b));
    asm("mov.b64 %0, {%1, %1};" : "=l"(ss) : "f"(s));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(x), "l"(ss));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(ra), "=f"(rb) : "l"(y));
}

// Codebook value at byte offset `off` (= 4 * code) of a 16-float table in
// shared memory.
__device__ __forceinline__ float lut_at(const float *lut, uint32_t off)
{
    return *reinterpret_cast<const float *>(reinterpret_cast<const char *>(lut) + off);
}

// 8 consecutive codes (one 32-bit word, element 0 in bits 0-3) -> 8 bf16 (or,
// with F16, fp16: the fp16 compute dtype) in a 16-byte vector (element 0 in
// the lowest 16 bits).  The byte offsets of the even and the odd codes are
// formed once per word; each element then costs one byte extraction and one
// shared-memory load.  kPairMul: the products as paired f32x2 multiplies (half
// the multiply instructions) or as scalar ones (no register pairing); both
// are IEEE round-to-nearest products, so the bits are the same.
template <bool F16 = false, bool kPairMul = true>
__device__ __forceinline__ uint4 expand8(uint32_t word, const float *lut, float c1p)
{
    const uint32_t ev = (word << 2) & 0x3C3C3C3Cu;   // byte k: 4 * code of element 2k
    const uint32_t od = (word >> 2) & 0x3C3C3C3Cu;   // byte k: 4 * code of element 2k+1
    float q[8];
    q[0] = lut_at(lut, ev & 0xFFu);
    q[1] = lut_at(lut, od & 0xFFu);
    q[2] = lut_at(lut, __byte_perm(ev, 0u, 0x4441));
    q[3] = lut_at(lut, __byte_perm(od, 0u, 0x4441));
    q[4] = lut_at(lut, __byte_perm(ev, 0u, 0x4442));
    q[5] = lut_at(lut, __byte_perm(od, 0u, 0x4442));
    q[6] = lut_at(lut, ev >> 24);
    q[7] = lut_at(lut, od >> 24);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float lo, hi;
        if constexpr (kPairMul) {
            mul2(q[2 * i], q[2 * i + 1], c1p, lo, hi);
        } else {
            lo = __fmul_rn(q[2 * i], c1p);
            hi = __fmul_rn(q[2 * i + 1], c1p);
        }
        o[i] = pack16x2<F16>(lo, hi);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace nf4
}  // namespace qlora
