// NF4 + double-quantization codec kernels for sm_100a.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs", section "Method":
//   - "4-bit NormalFloat Quantization", step (3): each block of 64 weights is
//     rescaled by its absolute maximum into [-1, 1] and rounded to the nearest
//     value of the 16-entry table (NF4, or any strictly increasing 16-value
//     table with one zero, such as the Int4 one);
//   - "Double Quantization": the per-block 32-bit constants are quantized
//     again (8-bit floats, groups of 256, mean subtracted);
//   - storage vs. compute type: the weight is dequantized to BFloat16 when
//     used.
//
// Three kernels, all streaming passes (bf16 input through per-warp TMA rings,
// 16- and 32-byte global accesses elsewhere):
//   quantize_blocks_kernel  W -> packed codes, c1 (workspace), exact mean
//   dq_encode_kernel        c1, mean -> code2 (E4M3), c2
//   dequantize_kernel       packed, code2, c2, mean -> bf16 W'
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "debug.cuh"
#include "exact_mean.cuh"
#include "nf4_expand.cuh"
#include "sm100.cuh"

namespace qlora {

namespace {

constexpr int kThreads = 256;
constexpr int kDeqUnroll = 4;   // words per thread in flight (dequantize)

// ---- small device helpers ----------------------------------------------------

// 32-byte store (sm_100).
__device__ __forceinline__ void st_v8(void *p, uint4 a, uint4 b)
{
    asm volatile("st.global.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
                 "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void *p)
{
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// ---- pass 1: absmax, codes, exact-mean buckets -----------------------------------

struct QuantParams {
    const void *W;             // bf16 or fp32, numel elements
    uint8_t *packed;           // numel / 2 bytes
    float *c1;                 // nblocks floats (workspace)
    unsigned long long *acc;   // 256 buckets (workspace, zero on entry)
    unsigned int *ticket;      // CTA arrival counter (workspace, zero on entry)
    float *mean_out;           // 1 float
    uint32_t nwords;           // numel / 8: one word = 8 codes = 32 bits
    int64_t nblocks;
    uint32_t mkey[15];         // keys of the round-down midpoints, ascending
    CUtensorMap tm_w;          // bf16 input as [nblocks][64], box 64 x 32, 128-byte swizzle
    int *err;                  // device error word (a bounded wait gave up)
    uint64_t timeout_ns;
    int stall_inject;          // failure-detection test hook: warp 0 of CTA 0 skips its first copy (bf16)
};

// bf16 input: every warp streams its 32 blocks (4 KB) per step through a
// two-stage shared-memory ring filled by TMA (lane 0 issues the copy of the
// next step before the current one is processed).
constexpr int kQStages = 2;
constexpr uint32_t kQStageBytes = 32 * 128;
// Quantizer: one CTA of 24 warps per SM (the per-warp TMA rings take 193 KB);
// registers capped at 64 per thread so that a dequantizer CTA of another stream
// still fits beside it.  Measured on B200 against 10 warps x 2 CTAs and 8 warps
// x 2 CTAs per SM: fastest alone (3.62 TB/s on 22016 x 8192), slightly less
// overlap between independent tensors on several streams.
constexpr int kQThreads = 768;
constexpr uint32_t kQDynSmem = (kQThreads / 32) * kQStages * kQStageBytes + 1024;

// Code lookup.  The 15 midpoints between neighbouring codebook values are
// rounded down to binary32, so "n > midpoint_j" holds exactly when n is nearer
// to value j+1 than to value j (a tie stays with the lower index), and the
// code is the number of midpoints below n.
// Keys: the order-preserving integer key of n (bits | 2^31 for n >= +0, ~bits
// for n <= -0) splits into an 11-bit interval index and a 21-bit offset; each
// interval that scaled elements reach (|n| <= 1, plus rounding) holds at most
// one midpoint (the host checks this).  The table is indexed by the top 11 RAW
// bits of n (sign, exponent, two mantissa bits), which name one interval; its
// entry plus the raw bits of n gives, through the carry out of the low 21
// bits, the code in bits 28..31 (bits 21..27 of the entry are ones so that the
// carry reaches bit 28):
//  - n >= +0: offset = low21(bits) grows with n; with j midpoints below the
//    interval and midpoint m inside it, the entry adds 2^21-1 - low21(key_m),
//    so the carry is [n > m] and the nibble j + [n > m];
//  - n <= -0: low21(bits) grows as n falls, so the entry yields 15 - code
//    (the nibble rises with |n| as the code falls): its top is 15 - j, or
//    14 - j and 1 + low21(key_m) added when m lies inside; the packed word's
//    nibbles of negative elements are complemented afterwards, from the input
//    sign bits (eight at a time with byte permutes).
// Entry i holds its value minus i << 21, so the sum's top bits depend only on
// the entry.  Per element: a shift (the index), a shared load, an add and a
// funnel shift that moves the nibble into the packed word.
// Every CTA builds the table once: thread t < 256 fills the entries of the
// key-ordered intervals 8t..8t+7, walking the sorted midpoint keys once.
constexpr int kLutShift = 21;
constexpr uint32_t kLutEntries = 1u << (32 - kLutShift);       // 2048
constexpr uint32_t kLutLow = (1u << kLutShift) - 1;

__device__ __forceinline__ void build_code_lut(uint32_t *lut, const uint32_t *mkey_smem)
{
    constexpr uint32_t kPer = kLutEntries / 256;
    constexpr uint32_t kHalf = kLutEntries / 2;
    const uint32_t first = threadIdx.x * kPer;
    uint32_t j = 0;
    while (j < 15 && mkey_smem[j] < (first << kLutShift)) j++;
#pragma unroll
    for (uint32_t t = 0; t < kPer; t++) {
        const uint32_t idx = first + t;    // interval of the order-preserving key
        while (j < 15 && mkey_smem[j] < (idx << kLutShift)) j++;
        const bool inside = j < 15 && (mkey_smem[j] >> kLutShift) == idx;
        const uint32_t low_m = inside ? mkey_smem[j] & kLutLow : 0u;
        uint32_t raw, top, inc;
        if (idx >= kHalf) {                // n >= +0: key = bits | 2^31
            raw = idx - kHalf;
            top = j;
            inc = inside ? kLutLow - low_m : 0u;
        } else {                           // n <= -0: key = ~bits
            raw = (kLutEntries - 1) - idx;
            top = inside ? 14 - j : 15 - j;
            inc = inside ? low_m + 1 : 0u;
        }
        lut[raw] = (((top << 7) | 0x7Fu) << kLutShift) + inc - (raw << kLutShift);
    }
}

// Table entry plus the raw bits of n: the code of n (15 - code for n <= -0)
// in bits 28..31.
__device__ __forceinline__ uint32_t code_top(const uint32_t *lut, float n)
{
    const uint32_t b = __float_as_uint(n);
    return lut[b >> kLutShift] + b;
}

// 8 nibbles of 8 consecutive values (already multiplied by r), element 0 in
// bits 0-3, those of negative elements still complemented: each funnel shift
// moves the word up one nibble and brings in the next lower element's nibble.
__device__ __forceinline__ uint32_t codes8(const uint32_t *lut, const float (&n)[8])
{
    uint32_t word = code_top(lut, n[7]) >> 28;
#pragma unroll
    for (int e = 6; e >= 0; e--) word = __funnelshift_l(code_top(lut, n[e]), word, 4);
    return word;
}

// Byte permute whose selector nibbles with bit 3 set replicate the sign bit
// of the chosen byte (0x00 or 0xFF).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Nibble mask of the negative elements among 8 elements given as 16-bit
// pairs u0..u3 (element 2j in the low half of uj): 0xF at nibble e where
// element e has its sign bit set.
__device__ __forceinline__ uint32_t neg_nibbles16(uint32_t u0, uint32_t u1, uint32_t u2, uint32_t u3)
{
    const uint32_t x = prmt(u0, u1, 0xFDB9);   // byte k: sign of element k (0..3)
    const uint32_t y = prmt(u2, u3, 0xFDB9);   // elements 4..7
    const uint32_t even = prmt(x, y, 0x6420);  // elements 0, 2, 4, 6
    const uint32_t odd = prmt(x, y, 0x7531);   // elements 1, 3, 5, 7
    return (even & 0x0F0F0F0Fu) | (odd & 0xF0F0F0F0u);
}

// The same for 8 binary32 elements (sign in byte 3 of each word).
__device__ __forceinline__ uint32_t neg_nibbles32(const uint4 &v0, const uint4 &v1)
{
    const uint32_t even = prmt(prmt(v0.x, v0.z, 0xFFFB), prmt(v1.x, v1.z, 0xFFFB), 0x5410);
    const uint32_t odd = prmt(prmt(v0.y, v0.w, 0xFFFB), prmt(v1.y, v1.w, 0xFFFB), 0x5410);
    return (even & 0x0F0F0F0Fu) | (odd & 0xF0F0F0F0u);
}

// Magnitude maximum of two bf16 (F16: fp16) pairs, lane by lane
// (max.xorsign.abs: the result's magnitude is max(|a|, |b|); its sign bit is
// meaningless and masked off by the caller).
template <bool F16>
__device__ __forceinline__ uint32_t maxabs16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    if constexpr (F16)
        asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    else
        asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// One lane per block of 64 weights, 32 consecutive blocks per warp and step:
// the loads of a warp cover 4 KB (bf16) of contiguous input and its stores 1 KB
// of packed codes; the block absmax, the reciprocal and the block constant are
// lane-local.  A lane's 8 (bf16) or 16 (fp32) 16-byte loads are issued
// together; fp32 input is read twice (the second time from L1).
// kIn: 0 bf16 input, 1 fp32 input, 2 fp16 input (bf16 and fp16 stream
// through the TMA rings).
template <int kIn>
__global__ void __maxnreg__(64) quantize_blocks_kernel(const __grid_constant__ QuantParams p)
{
    constexpr bool kF32In = kIn == 1;
    constexpr bool kF16In = kIn == 2;
    static_assert(kQThreads >= 256, "the first 256 threads build the code table and own the buckets");
    __shared__ __align__(16) uint32_t lut[kLutEntries];
    __shared__ unsigned long long s_acc[256];
    __shared__ uint32_t s_mkey[16];
    __shared__ bool s_last;
    __shared__ int s_lohi[8][2];
    const uint32_t lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t nwarps = (int64_t)gridDim.x * (kQThreads / 32);
    // warp w of CTA c is global warp w * gridDim.x + c: the steps a few warps
    // take beyond an equal share are spread over all SMs instead of landing
    // on the first CTAs
    const int64_t first = ((int64_t)warp * gridDim.x + blockIdx.x) * 32;
    // bf16: this warp's TMA ring (stages of 32 rows x 128 B, 128-byte swizzle);
    // the first copy is issued before the code table is built
    extern __shared__ uint8_t q_dyn[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(q_dyn) + 1023) & ~uintptr_t(1023)) +
                    warp * kQStages * kQStageBytes;
    __shared__ uint64_t s_bar[kQThreads / 32][kQStages];
    // Set-up that reads no memory another kernel writes (barriers, the code
    // table from the parameters) runs before the dependency wait: launched with
    // programmatic serialization, it overlaps the tail of the kernel before
    // (for a quantize call, the kernel that reset its reduction slots).
    if (!kF32In && lane == 0) {
        for (int st = 0; st < kQStages; st++) sm100::mbar_init(&s_bar[warp][st], 1);
        sm100::fence_barrier_init();
    }
    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < 15; j++) s_mkey[j] = p.mkey[j];
    }
    if (threadIdx.x < 256) s_acc[threadIdx.x] = 0;
    __syncthreads();
    if (threadIdx.x < 256) build_code_lut(lut, s_mkey);
    // the input, the reduction slots and the outputs from here on; the
    // double-quantization kernel after this one may become resident now and
    // wait for this grid's completion
    sm100::pdl_wait();
    sm100::pdl_trigger();
    if (!kF32In && lane == 0) {
        const bool skip = p.stall_inject && blockIdx.x == 0 && warp == 0;
        if (first < p.nblocks && !skip) {
            sm100::mbar_arrive_expect_tx(&s_bar[warp][0], kQStageBytes);
            sm100::tma_load_2d(ring, &p.tm_w, &s_bar[warp][0], 0, (int32_t)first);
        }
    }
    __syncthreads();
    uint32_t it = 0;
    for (int64_t b0 = first; b0 < p.nblocks; b0 += nwarps * 32, it++) {
        const int64_t b = b0 + lane;
        const bool act = b < p.nblocks;
        uint32_t words[8];
        float cv;
        if (!kF32In) {
            const int st = it & 1;
            const int64_t nb = b0 + nwarps * 32;
            if (lane == 0 && nb < p.nblocks) {
                // the other stage was read by every lane in the previous step
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive_expect_tx(&s_bar[warp][st ^ 1], kQStageBytes);
                sm100::tma_load_2d(ring + (st ^ 1) * kQStageBytes, &p.tm_w, &s_bar[warp][st ^ 1], 0, (int32_t)nb);
            }
            const bool landed = sm100::mbar_wait_bounded(&s_bar[warp][st], (it >> 1) & 1, p.timeout_ns);
            if (!__all_sync(0xffffffffu, landed)) {
                // a copy did not arrive: record it and stop; the copy of the next
                // step (if issued) is waited for below, bounded, before leaving
                if (lane == 0) {
                    atomicExch(p.err, 1);
                    if (nb < p.nblocks) sm100::mbar_wait_bounded(&s_bar[warp][st ^ 1], ((it + 1) >> 1) & 1, p.timeout_ns);
                }
                break;
            }
            // row `lane` of the stage: 16-byte chunk c sits at c ^ (lane & 7)
            const uint8_t *row = ring + st * kQStageBytes + lane * 128;
            uint4 v[8];
#pragma unroll
            for (int i = 0; i < 8; i++) v[i] = *reinterpret_cast<const uint4 *>(row + ((i ^ (lane & 7)) << 4));
            // block absmax: magnitudes of the 64 values in two lanes of bf16
            // pairs, then the larger half; magnitude bit patterns compare like
            // the values
            uint32_t m0 = maxabs16x2<kF16In>(v[0].x, v[0].y), m1 = maxabs16x2<kF16In>(v[0].z, v[0].w);
#pragma unroll
            for (int i = 1; i < 8; i++) {
                m0 = maxabs16x2<kF16In>(m0, maxabs16x2<kF16In>(v[i].x, v[i].y));
                m1 = maxabs16x2<kF16In>(m1, maxabs16x2<kF16In>(v[i].z, v[i].w));
            }
            const uint32_t m = maxabs16x2<kF16In>(m0, m1) & 0x7FFF7FFFu;
            const uint32_t mh = __vmaxu2(m, m >> 16) & 0xFFFFu;   // larger half
            cv = kF16In ? __half2float(__ushort_as_half((unsigned short)mh)) : __uint_as_float(mh << 16);
            // zero block (absmax below the smallest normal): r = 0 sends every
            // element to n = +-0, whose code is the codebook's zero
            const float r = cv < 1.17549435e-38f ? 0.0f : __frcp_rn(cv);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                float n[8];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    if constexpr (kF16In) {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&u[j]));
                        nf4::mul2(f.x, f.y, r, n[2 * j], n[2 * j + 1]);
                    } else {
                        nf4::mul2(__uint_as_float(u[j] << 16), __uint_as_float(u[j] & 0xFFFF0000u), r, n[2 * j],
                                  n[2 * j + 1]);
                    }
                }
                words[i] = codes8(lut, n) ^ neg_nibbles16(u[0], u[1], u[2], u[3]);
            }
        } else {
            const uint4 *src = static_cast<const uint4 *>(p.W) + 16 * b;  // 64 fp32 = 16 x 16 B
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const uint4 v = act && QLORA_IN(b, p.nblocks) ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
                m = fmaxf(fmaxf(m, fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y)))),
                          fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w))));
            }
            cv = m;
            const float r = cv < 1.17549435e-38f ? 0.0f : __frcp_rn(cv);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const uint4 v0 = act ? __ldg(src + 2 * i) : make_uint4(0, 0, 0, 0);
                const uint4 v1 = act ? __ldg(src + 2 * i + 1) : make_uint4(0, 0, 0, 0);
                float n[8];
                nf4::mul2(__uint_as_float(v0.x), __uint_as_float(v0.y), r, n[0], n[1]);
                nf4::mul2(__uint_as_float(v0.z), __uint_as_float(v0.w), r, n[2], n[3]);
                nf4::mul2(__uint_as_float(v1.x), __uint_as_float(v1.y), r, n[4], n[5]);
                nf4::mul2(__uint_as_float(v1.z), __uint_as_float(v1.w), r, n[6], n[7]);
                words[i] = codes8(lut, n) ^ neg_nibbles32(v0, v1);
            }
        }
        if (act && QLORA_IN(b, p.nblocks)) {
            st_v8(reinterpret_cast<uint4 *>(p.packed) + 2 * b, make_uint4(words[0], words[1], words[2], words[3]),
                  make_uint4(words[4], words[5], words[6], words[7]));   // 64 codes = 32 B
            p.c1[b] = cv;
        }
        if (!kF32In) __syncwarp();   // every lane has read its row before the stage is refilled
        // exact-mean buckets: one shared atomic per distinct exponent in the warp
        uint32_t bucket, sig;
        exact_mean_split(__float_as_uint(cv), &bucket, &sig);
        bool pending = act;
        for (;;) {
            const unsigned pend = __ballot_sync(0xffffffffu, pending);
            if (!pend) break;
            const int leader = __ffs(pend) - 1;
            const uint32_t lb = __shfl_sync(0xffffffffu, bucket, leader);
            const bool mine = pending && bucket == lb;
            const uint32_t sum = __reduce_add_sync(0xffffffffu, mine ? sig : 0u);   // < 32 * 2^24
            if ((int)lane == leader) atomicAdd(&s_acc[lb], (unsigned long long)sum);
            pending = pending && !mine;
        }
    }
    __syncthreads();
    if (threadIdx.x < 256) {
        const unsigned long long v = s_acc[threadIdx.x];
        if (v) atomicAdd(&p.acc[threadIdx.x], v);
    }
    // the last CTA to finish turns the buckets into the mean.  The barrier
    // orders this CTA's bucket atomics before thread 0's fence, which is
    // cumulative over them, and the fence before the ticket.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(p.ticket, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        // the first 256 threads own the buckets
        const unsigned long long mine = threadIdx.x < 256 ? atomicAdd(&p.acc[threadIdx.x], 0ull) : 0ull;
        if (threadIdx.x < 256) s_acc[threadIdx.x] = mine;
        // lowest and highest non-zero bucket (1..254)
        const bool nz = mine != 0 && threadIdx.x >= 1 && threadIdx.x <= 254;
        const unsigned bal = __ballot_sync(0xffffffffu, nz);
        if ((threadIdx.x & 31) == 0 && threadIdx.x < 256) {
            s_lohi[threadIdx.x >> 5][0] = bal ? (int)(threadIdx.x + __ffs(bal) - 1) : 256;
            s_lohi[threadIdx.x >> 5][1] = bal ? (int)(threadIdx.x + 31 - __clz(bal)) : -1;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int lo = 256, hi = -1;
            for (int w = 0; w < 8; w++) {
                lo = min(lo, s_lohi[w][0]);
                hi = max(hi, s_lohi[w][1]);
            }
            *p.mean_out = __uint_as_float(exact_mean_bits_range(s_acc, (uint64_t)p.nblocks, lo, hi));
        }
    }
}

// ---- pass 2: double quantization of the block constants ----------------------------

struct DqParams {
    const float *c1;
    const float *mean;
    uint8_t *code2;
    float *c2;
    int64_t nblocks;
    int64_t ngroups;
};

// E4M3 code (saturating, round to nearest even) of RN32(d / c2) for c2 > 0.
// Fast path: q = RN32(d * RN32(1/c2)) lies within 3 units in the last place
// of RN32(d / c2) (two roundings of relative size 2^-24 each); E4M3 rounding
// is monotone, so when the values 4 units below and above q encode to the
// same code, that code is the one of RN32(d / c2).  Otherwise (q within a few
// units of an E4M3 rounding boundary, about once in 10^5 values) the quotient
// is formed with the IEEE division, as it is for c2 < 2^-100 (rc2 = 0 then).
__device__ __forceinline__ uint8_t e4m3_of_quotient(float d, float c2, float rc2)
{
    if (rc2 == 0.0f)   // c2 below 2^-100: the reciprocal could overflow; divide
        return (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(d, c2), __NV_SATFINITE, __NV_E4M3);
    const float q = __fmul_rn(d, rc2);
    const uint32_t b = __float_as_uint(q);
    const uint32_t mag = b & 0x7FFFFFFFu;
    float lo = q, hi = q;
    if (mag >= 4u) {   // |q| far below every E4M3 boundary otherwise
        lo = __uint_as_float(b - 4u);
        hi = __uint_as_float(b + 4u);
    }
    const __nv_fp8x2_storage_t two = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
    const uint8_t e_lo = (uint8_t)(two & 0xFF), e_hi = (uint8_t)(two >> 8);
    if (e_lo == e_hi) return e_lo;
    return (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(d, c2), __NV_SATFINITE, __NV_E4M3);
}

// One warp per group of 256 constants, 8 consecutive ones per lane (two
// 16-byte loads).
__global__ void __launch_bounds__(kThreads) dq_encode_kernel(DqParams p)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // resident while the quantizer runs; c1 and the mean are read after it completed
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const float mu = *p.mean;
    for (int64_t g = (int64_t)blockIdx.x * (kThreads / 32) + warp; g < p.ngroups;
         g += (int64_t)gridDim.x * (kThreads / 32)) {
        const int64_t b0 = g * QLORA_GROUP + lane * 8;
        float c[8];
        if (b0 + 8 <= p.nblocks) {
            const float4 v0 = *reinterpret_cast<const float4 *>(p.c1 + b0);
            const float4 v1 = *reinterpret_cast<const float4 *>(p.c1 + b0 + 4);
            c[0] = v0.x; c[1] = v0.y; c[2] = v0.z; c[3] = v0.w;
            c[4] = v1.x; c[5] = v1.y; c[6] = v1.z; c[7] = v1.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) c[i] = b0 + i < p.nblocks ? p.c1[b0 + i] : mu;   // d = 0 past the end
        }
        float d[8];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            d[i] = __fsub_rn(c[i], mu);
            amax = fmaxf(amax, fabsf(d[i]));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = __fdiv_rn(amax, 448.0f);
        if (lane == 0 && QLORA_IN(g, p.ngroups)) p.c2[g] = s;
        const float rs = s >= 0x1p-100f ? __frcp_rn(s) : 0.0f;
        uint8_t e[8];
#pragma unroll
        for (int i = 0; i < 8; i++) e[i] = s == 0.0f ? (uint8_t)0 : e4m3_of_quotient(d[i], s, rs);
        if (b0 + 8 <= p.nblocks && QLORA_IN(b0 + 7, p.nblocks)) {
            uint2 v;
            v.x = e[0] | (e[1] << 8) | (e[2] << 16) | ((uint32_t)e[3] << 24);
            v.y = e[4] | (e[5] << 8) | (e[6] << 16) | ((uint32_t)e[7] << 24);
            *reinterpret_cast<uint2 *>(p.code2 + b0) = v;
        } else {
            for (int i = 0; i < 8; i++)
                if (b0 + i < p.nblocks) p.code2[b0 + i] = e[i];
        }
    }
}

// ---- dequantize -------------------------------------------------------------------

struct DeqParams {
    const uint8_t *packed;
    const uint8_t *code2;
    const float *c2;
    const float *mean;
    __nv_bfloat16 *out;
    int64_t nwords;
    float q[16];
};

template <bool F16>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(DeqParams p)
{
    __shared__ float lut[16];
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < 16; i++) lut[i] = p.q[i];   // static indices keep p in the parameter bank
    }
    __syncthreads();
    sm100::pdl_wait();   // the quantized weight may come from the kernel before this one
    sm100::pdl_trigger();
    const float mu = *p.mean;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t w0 = (int64_t)blockIdx.x * kThreads + threadIdx.x; w0 < p.nwords; w0 += stride * kDeqUnroll) {
        uint32_t word[kDeqUnroll];
        float c1p[kDeqUnroll];
#pragma unroll
        for (int u = 0; u < kDeqUnroll; u++) {
            int64_t w = w0 + u * stride;
            word[u] = 0;
            c1p[u] = 0.0f;
            if (w < p.nwords) {
                word[u] = ld_stream_u32(p.packed + 4 * w);
                int64_t b = w >> 3;
                if (QLORA_IN(b, (p.nwords + 7) / 8) && QLORA_IN(b / QLORA_GROUP, (p.nwords / 8 + QLORA_GROUP - 1) / QLORA_GROUP))
                    c1p[u] = nf4::block_scale(p.code2[b], p.c2[b / QLORA_GROUP], mu);
            }
        }
#pragma unroll
        for (int u = 0; u < kDeqUnroll; u++) {
            int64_t w = w0 + u * stride;
            if (w >= p.nwords || !QLORA_IN(w, p.nwords)) continue;
            *reinterpret_cast<uint4 *>(p.out + 8 * w) = nf4::expand8<F16>(word[u], lut, c1p[u]);
        }
    }
}

// ---- host helpers ----------------------------------------------------------------

// Binary32 nearest below-or-equal to a double.
float round_down_f32(double d)
{
    float f = (float)d;
    if ((double)f > d) f = nextafterf(f, -INFINITY);
    return f;
}

uint32_t host_sortable_key(float f)
{
    uint32_t b;
    memcpy(&b, &f, 4);
    uint32_t s = (uint32_t)((int32_t)b >> 31);
    return b ^ (s | 0x80000000u);
}

// Midpoint keys for the code lookup; rejects tables the lookup cannot serve.
qlora_status midpoint_keys(const float q[16], uint32_t out[15])
{
    for (int j = 0; j < 15; j++) {
        if (!(q[j] < q[j + 1])) return QLORA_ERR_INVALID_ARG;
        double sum = (double)q[j] + (double)q[j + 1];
        if (sum - (double)q[j + 1] != (double)q[j]) return QLORA_ERR_UNSUPPORTED;  // inexact sum
        float m = round_down_f32(sum / 2.0);
        if (m == 0.0f) m = 0.0f;  // +0, never -0
        out[j] = host_sortable_key(m);
        // two midpoints in one key interval: only an interval that scaled
        // elements reach (|n| <= 1, plus rounding) must hold at most one
        const uint32_t iv = out[j] >> kLutShift;
        if (j > 0 && iv == (out[j - 1] >> kLutShift) && iv >= (host_sortable_key(-1.0001f) >> kLutShift) &&
            iv <= (host_sortable_key(1.0001f) >> kLutShift))
            return QLORA_ERR_UNSUPPORTED;
    }
    return QLORA_OK;
}

// Tensor map of a bf16 input, error word, timeout and the kernel's dynamic
// shared-memory limit (once per device).
qlora_status prepare_quantize(QuantParams &qp, const void *W, qlora_dtype w_dtype, int64_t numel,
                              const DeviceInfo &dev)
{
    qp.err = device_error_word();
    if (!qp.err) return QLORA_ERR_CUDA;
    qp.timeout_ns = 2000000000ull;
    qp.stall_inject = 0;
    if (w_dtype == QLORA_BF16 || w_dtype == QLORA_FP16) {
        QLORA_TRY(make_map(&qp.tm_w,
                           w_dtype == QLORA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, W,
                           64, (uint64_t)(numel / 64), 128, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B));
        static PerDeviceOnce attr;
        QLORA_TRY(attr.run(dev.device, []() -> qlora_status {
            QLORA_CUDA_TRY(cudaFuncSetAttribute(quantize_blocks_kernel<0>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, kQDynSmem));
            QLORA_CUDA_TRY(cudaFuncSetAttribute(quantize_blocks_kernel<2>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, kQDynSmem));
            return QLORA_OK;
        }));
        qp.stall_inject = take_stall_injection(QLORA_KERNEL_QUANTIZE, &qp.timeout_ns) ? 1 : 0;
    }
    return QLORA_OK;
}

// Resets the quantizer's reduction slots (bucket sums and the CTA ticket) at
// the start of a call; a kernel rather than a memset so that the quantizer's
// set-up can overlap it under programmatic dependent launch.
__global__ void __launch_bounds__(64) reset_slots_kernel(unsigned long long *acc, unsigned int *ticket)
{
    sm100::pdl_wait();   // the previous call on this workspace may still read the slots
    sm100::pdl_trigger();
    for (int i = threadIdx.x; i < 256; i += 64) acc[i] = 0ull;
    if (threadIdx.x == 0) *ticket = 0u;
}

// The quantizer for the input type w_dtype.
cudaError_t launch_quantize(qlora_dtype w_dtype, int grid, cudaStream_t s, const QuantParams &qp)
{
    if (w_dtype == QLORA_FP32) return launch_pdl(quantize_blocks_kernel<1>, dim3(grid), dim3(kQThreads), 0, s, qp);
    if (w_dtype == QLORA_FP16)
        return launch_pdl(quantize_blocks_kernel<2>, dim3(grid), dim3(kQThreads), kQDynSmem, s, qp);
    return launch_pdl(quantize_blocks_kernel<0>, dim3(grid), dim3(kQThreads), kQDynSmem, s, qp);
}

int grid_for(int64_t work_items, int items_per_cta, int max_ctas)
{
    int64_t g = (work_items + items_per_cta - 1) / items_per_cta;
    if (g > max_ctas) g = max_ctas;
    return g < 1 ? 1 : (int)g;
}

}  // namespace

// Workspace layout for the quantizer: [acc 256 u64][ticket u32 + pad to 16][c1 floats]
static constexpr size_t kAccBytes = 256 * sizeof(unsigned long long) + 16;

// The reduction slots and the arrival ticket start at zero on every call.
static qlora_status reset_slots(void *ws, cudaStream_t s)
{
    {
        LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
        QLORA_CUDA_TRY(launch_pdl(reset_slots_kernel, dim3(1), dim3(64), 0, s,
                                  static_cast<unsigned long long *>(ws),
                                  reinterpret_cast<unsigned int *>(static_cast<char *>(ws) +
                                                                   256 * sizeof(unsigned long long))));
    }
    return launch_status();
}

}  // namespace qlora

using namespace qlora;

extern "C" size_t qlora_quantize_workspace_bytes(int64_t rows, int64_t cols)
{
    if (rows <= 0 || cols <= 0) return kAccBytes;
    int64_t nblocks = rows * cols / QLORA_BLOCK;
    return kAccBytes + (size_t)((nblocks * 4 + 15) / 16 * 16);
}

extern "C" qlora_status qlora_quantize_nf4_dq(const void *W, qlora_dtype w_dtype, const qlora_nf4_weight *out,
                                              void *workspace, size_t workspace_bytes, void *stream)
{
    if (!W || !out || !workspace) return QLORA_ERR_INVALID_ARG;
    if (w_dtype != QLORA_BF16 && w_dtype != QLORA_FP32 && w_dtype != QLORA_FP16) return QLORA_ERR_INVALID_ARG;
    QLORA_TRY(check_weight(out));
    if (!aligned16(W) || !aligned16(workspace)) return QLORA_ERR_ALIGNMENT;
    if (workspace_bytes < qlora_quantize_workspace_bytes(out->rows, out->cols)) return QLORA_ERR_WORKSPACE;
    if (out->rows * out->cols / 8 >= ((int64_t)1 << 31)) return QLORA_ERR_SHAPE;   // 32-bit word indices
    uint32_t mkey[15];
    QLORA_TRY(midpoint_keys(out->codebook, mkey));
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t numel = out->rows * out->cols;
    const int64_t nblocks = numel / QLORA_BLOCK;
    char *ws = static_cast<char *>(workspace);
    QLORA_TRY(reset_slots(ws, s));

    QuantParams qp;
    qp.W = W;
    qp.packed = out->packed;
    qp.acc = reinterpret_cast<unsigned long long *>(ws);
    qp.ticket = reinterpret_cast<unsigned int *>(ws + 256 * sizeof(unsigned long long));
    qp.c1 = reinterpret_cast<float *>(ws + kAccBytes);
    qp.mean_out = out->mean;
    qp.nwords = (uint32_t)(numel / 8);
    qp.nblocks = nblocks;
    memcpy(qp.mkey, mkey, sizeof(mkey));
    QLORA_TRY(prepare_quantize(qp, W, w_dtype, numel, dev));
    int grid = grid_for(qp.nblocks, kQThreads * 2, dev.sms);
    {
        LaunchScope ls(QLORA_KERNEL_QUANTIZE, s);
        QLORA_CUDA_TRY(launch_quantize(w_dtype, grid, s, qp));
    }
    QLORA_TRY(launch_status());

    DqParams dp;
    dp.c1 = qp.c1;
    dp.mean = out->mean;
    dp.code2 = out->code2;
    dp.c2 = out->c2;
    dp.nblocks = nblocks;
    dp.ngroups = (nblocks + QLORA_GROUP - 1) / QLORA_GROUP;
    {
        LaunchScope ls(QLORA_KERNEL_DQ_ENCODE, s);
        QLORA_CUDA_TRY(launch_pdl(dq_encode_kernel, dim3(grid_for(dp.ngroups, kThreads / 32, dev.sms * 8)),
                                  dim3(kThreads), 0, s, dp));
    }
    return launch_status();
}

extern "C" qlora_status qlora_dequantize_nf4_dq_ex(const qlora_nf4_weight *w, void *out, qlora_dtype out_dtype,
                                                   void *stream)
{
    if (!w || !out) return QLORA_ERR_INVALID_ARG;
    if (out_dtype != QLORA_BF16 && out_dtype != QLORA_FP16) return QLORA_ERR_INVALID_ARG;
    void *out_bf16 = out;
    QLORA_TRY(check_weight(w));
    if (!aligned16(out_bf16)) return QLORA_ERR_ALIGNMENT;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    DeqParams p;
    p.packed = w->packed;
    p.code2 = w->code2;
    p.c2 = w->c2;
    p.mean = w->mean;
    p.out = static_cast<__nv_bfloat16 *>(out_bf16);
    p.nwords = w->rows * w->cols / 8;
    memcpy(p.q, w->codebook, sizeof(p.q));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        LaunchScope ls(QLORA_KERNEL_DEQUANTIZE, s);
        QLORA_CUDA_TRY(launch_pdl(out_dtype == QLORA_FP16 ? dequantize_kernel<true> : dequantize_kernel<false>,
                                  dim3(grid_for(p.nwords, kThreads * kDeqUnroll, dev.sms * 8)), dim3(kThreads), 0, s,
                                  p));
    }
    return launch_status();
}

extern "C" qlora_status qlora_dequantize_nf4_dq(const qlora_nf4_weight *w, void *out_bf16, void *stream)
{
    return qlora_dequantize_nf4_dq_ex(w, out_bf16, QLORA_BF16, stream);
}

// ---- quantization without allocation ------------------------------------------------
//
// Same kernels and results as qlora_quantize_nf4_dq, but the scratch memory
// (reduction slots and the first-level constants c1) lives in a fixed
// module-level device array instead of a caller-provided workspace.  For
// callers that cannot hand over device memory at quantization time: a process
// whose memory is already fully reserved for a pool or cache, or code that
// quantizes weights while other streams are busy and must not call cudaMalloc
// or cudaFree, which synchronize the device.  The array is shared by every
// call on a device, so calls that overlap in time (two streams, two host
// threads) race on it; the caller must order them.

namespace qlora {
namespace {

constexpr size_t kStaticAccBytes = 2304;   // kAccBytes rounded up to 256 bytes
static_assert(kStaticAccBytes >= kAccBytes, "reduction slots must fit");
constexpr size_t kStaticScratchBytes = kStaticAccBytes + (size_t)QLORA_NOALLOC_MAX_BLOCKS * 4;

// [acc 256 u64][ticket][pad][c1: QLORA_NOALLOC_MAX_BLOCKS floats], about 4 MiB per device
static __device__ __align__(256) unsigned char g_quant_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = kMaxDevices;
unsigned char *g_scratch_ptr[kMaxScratchDevices] = {};
std::mutex g_scratch_mutex;

// Device address of this device's scratch array; the first call per device
// looks it up (with that device current) and caches it.
qlora_status static_scratch(int device, unsigned char **out)
{
    if (device < 0 || device >= kMaxScratchDevices) return QLORA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[device]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_quant_scratch) != cudaSuccess || !p) return QLORA_ERR_CUDA;
        g_scratch_ptr[device] = static_cast<unsigned char *>(p);
    }
    *out = g_scratch_ptr[device];
    return QLORA_OK;
}

}  // namespace
}  // namespace qlora

extern "C" qlora_status qlora_quantize_nf4_dq_noalloc(const void *W, qlora_dtype w_dtype,
                                                      const qlora_nf4_weight *out, void *stream)
{
    if (!W || !out) return QLORA_ERR_INVALID_ARG;
    if (w_dtype != QLORA_BF16 && w_dtype != QLORA_FP32 && w_dtype != QLORA_FP16) return QLORA_ERR_INVALID_ARG;
    QLORA_TRY(check_weight(out));
    if (!aligned16(W)) return QLORA_ERR_ALIGNMENT;
    // larger than the fixed scratch (compared before multiplying)
    if (out->rows > (int64_t)QLORA_NOALLOC_MAX_BLOCKS * QLORA_BLOCK / out->cols) return QLORA_ERR_SHAPE;
    const int64_t numel = out->rows * out->cols;
    const int64_t nblocks = numel / QLORA_BLOCK;
    if (nblocks > QLORA_NOALLOC_MAX_BLOCKS) return QLORA_ERR_SHAPE;
    uint32_t mkey[15];
    QLORA_TRY(midpoint_keys(out->codebook, mkey));
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    unsigned char *ws = nullptr;
    QLORA_TRY(static_scratch(dev.device, &ws));

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    QLORA_TRY(reset_slots(ws, s));

    QuantParams qp;
    qp.W = W;
    qp.packed = out->packed;
    qp.acc = reinterpret_cast<unsigned long long *>(ws);
    qp.ticket = reinterpret_cast<unsigned int *>(ws + 256 * sizeof(unsigned long long));
    qp.c1 = reinterpret_cast<float *>(ws + kStaticAccBytes);
    qp.mean_out = out->mean;
    qp.nwords = (uint32_t)(numel / 8);
    qp.nblocks = nblocks;
    memcpy(qp.mkey, mkey, sizeof(mkey));
    QLORA_TRY(prepare_quantize(qp, W, w_dtype, numel, dev));
    const int grid = grid_for(qp.nblocks, kQThreads * 2, dev.sms);
    {
        LaunchScope ls(QLORA_KERNEL_QUANTIZE, s);
        QLORA_CUDA_TRY(launch_quantize(w_dtype, grid, s, qp));
    }
    QLORA_TRY(launch_status());

    DqParams dp;
    dp.c1 = qp.c1;
    dp.mean = out->mean;
    dp.code2 = out->code2;
    dp.c2 = out->c2;
    dp.nblocks = nblocks;
    dp.ngroups = (nblocks + QLORA_GROUP - 1) / QLORA_GROUP;
    {
        LaunchScope ls(QLORA_KERNEL_DQ_ENCODE, s);
        QLORA_CUDA_TRY(launch_pdl(dq_encode_kernel, dim3(grid_for(dp.ngroups, kThreads / 32, dev.sms * 8)),
                                  dim3(kThreads), 0, s, dp));
    }
    return launch_status();
}
