// Exactly rounded mean of non-negative binary32 values, from per-exponent
// integer sums.
//
// Double quantization subtracts the mean of the first-level constants before
// quantizing them ("QLoRA: Efficient Finetuning of Quantized LLMs", section
// "Method", paragraph "Double Quantization").  The mean used here is the
// binary32 number nearest to the exact arithmetic mean (ties to even), which
// does not depend on summation order: kernels add the significands of values
// that share an exponent field into 64-bit integer buckets, in any order,
// and this routine turns the buckets into the rounded mean.
//
// A non-negative binary32 v with exponent field E and fraction F equals
// m * 2^(max(E,1) - 150) with m = F + (E > 0 ? 2^23 : 0).  Bucket j (1..254)
// holds the sum of m over values with max(E,1) == j; bucket 0 is unused.
// Each bucket stays below 2^56 as long as fewer than 2^32 values are summed.
//
// Written for both host and device so the same code is unit-tested on CPU.
#pragma once
#include <stdint.h>

#ifndef QLORA_HD
#if defined(__CUDACC__)
#define QLORA_HD __host__ __device__ __forceinline__
#else
#define QLORA_HD inline
#endif
#endif

namespace qlora {

// Bucket index and significand of a finite non-negative binary32 bit pattern.
QLORA_HD void exact_mean_split(uint32_t bits, uint32_t *bucket, uint32_t *sig)
{
    uint32_t E = bits >> 23;
    uint32_t F = bits & 0x7FFFFFu;
    *bucket = E ? E : 1u;
    *sig = E ? (F | 0x800000u) : F;
}

// Count of leading zero bits of a non-zero 64-bit value.
QLORA_HD int clz64(uint64_t v)
{
#if defined(__CUDA_ARCH__)
    return __clzll((long long)v);
#else
    return __builtin_clzll(v);
#endif
}

// Fast path: all non-zero buckets lie within 61 consecutive exponents, so the
// exact sum fits one 128-bit integer T (units of 2^(lo-150)); the quotient
// T / count is normalized to at least 26 bits before rounding.  Returns false
// when the fast path does not apply.
QLORA_HD bool exact_mean_bits_narrow(const unsigned long long *bucket, uint64_t count, int lo, int hi,
                                     uint32_t *out)
{
    if (hi - lo > 60) return false;
    unsigned __int128 T = 0;
    for (int j = lo; j <= hi; j++) T += (unsigned __int128)bucket[j] << (j - lo);
    int b = lo - 150;                                   // value = T * 2^b / count
    // normalize so that the quotient has at least 26 significant bits
    const unsigned __int128 need = (unsigned __int128)count << 26;
    while (T < need) {
        T <<= 1;
        b -= 1;
    }
    // Q = T / count by long division in 32-bit digits (count < 2^32), which
    // avoids a generic 128-bit division
    uint32_t qd[4];
    uint64_t rem = 0;
    for (int i = 3; i >= 0; i--) {
        const uint64_t cur = (rem << 32) | (uint32_t)(T >> (32 * i));
        qd[i] = (uint32_t)(cur / count);
        rem = cur % count;
    }
    const unsigned __int128 Q = ((unsigned __int128)(((uint64_t)qd[3] << 32) | qd[2]) << 64) |
                                (((uint64_t)qd[1] << 32) | qd[0]);
    // position of the most significant set bit (Q >= 2^26 after normalization)
    const uint64_t qhi = (uint64_t)(Q >> 64), qlo = (uint64_t)Q;
    int p = qhi ? 127 - clz64(qhi) : 63 - clz64(qlo);
    // least significant kept bit: 2^(p+b-23) for a normal result, 2^-149 below
    int L = p + b - 23;
    if (L < -149) L = -149;
    const int t = L - b;                                // quotient bits dropped (>= 2)
    uint32_t mant;
    bool up;
    if (t > 127) {
        mant = 0;
        up = false;                                     // far below 2^-150: rounds to 0
    } else {
        mant = (uint32_t)(Q >> t);
        const bool round_bit = (Q >> (t - 1)) & 1;
        const unsigned __int128 low_mask = (((unsigned __int128)1) << (t - 1)) - 1;
        const bool sticky = (Q & low_mask) != 0 || rem != 0;
        up = round_bit && (sticky || (mant & 1u));
    }
    if (up) mant += 1;
    // value = mant * 2^L; the same formula covers subnormals (L = -149) and a
    // carry into the next binade
    *out = ((uint32_t)(L + 149) << 23) + mant;
    return true;
}

QLORA_HD uint32_t exact_mean_bits_range(const unsigned long long *bucket, uint64_t count, int lo, int hi);

// Binary32 bit pattern of RN(sum_j bucket[j] * 2^(j-150) / count).
// bucket has 256 entries; count >= 1 and < 2^32.
QLORA_HD uint32_t exact_mean_bits(const unsigned long long *bucket, uint64_t count)
{
    int lo = 256, hi = -1;
#pragma unroll 8
    for (int j = 1; j < 255; j++) {
        if (bucket[j]) {
            lo = j < lo ? j : lo;
            hi = j;
        }
    }
    return exact_mean_bits_range(bucket, count, lo, hi);
}

// The same, given the lowest (lo) and highest (hi) non-zero bucket in 1..254
// (hi < 0 when every bucket is zero).
QLORA_HD uint32_t exact_mean_bits_range(const unsigned long long *bucket, uint64_t count, int lo, int hi)
{
    if (hi < 0) return 0u;
    uint32_t fast;
    if (exact_mean_bits_narrow(bucket, count, lo, hi, &fast)) return fast;

    // 1. exact sum as an integer in units of 2^-149: sum_j bucket[j] << (j-1)
    //    held in ten 32-bit digits (320 bits, least significant first).
    uint32_t dig[10];
    for (int i = 0; i < 10; i++) dig[i] = 0;
    bool any = false;
    for (int j = 1; j < 255; j++) {
        unsigned long long v = bucket[j];
        if (v == 0) continue;
        any = true;
        int sh = j - 1;
        int d0 = sh >> 5, b0 = sh & 31;
        // v << b0 spans at most three digits (v < 2^64, b0 < 32)
        uint64_t lo = (uint64_t)(uint32_t)v << b0;               // bits 0..63
        uint64_t hi = (uint64_t)(uint32_t)(v >> 32) << b0;        // bits 32..95
        uint32_t part[4];
        part[0] = (uint32_t)lo;
        uint64_t mid = (lo >> 32) + (uint32_t)hi;
        part[1] = (uint32_t)mid;
        uint64_t top = (mid >> 32) + (hi >> 32);
        part[2] = (uint32_t)top;
        part[3] = (uint32_t)(top >> 32);
        uint64_t carry = 0;
        for (int i = 0; i < 4 || carry; i++) {
            int d = d0 + i;
            if (d >= 10) break;
            uint64_t s = (uint64_t)dig[d] + (i < 4 ? part[i] : 0u) + carry;
            dig[d] = (uint32_t)s;
            carry = s >> 32;
        }
    }
    if (!any) return 0u;

    // 2. long division by count, most significant digit first
    uint32_t quo[10];
    uint64_t rem = 0;
    for (int i = 9; i >= 0; i--) {
        uint64_t cur = (rem << 32) | dig[i];
        quo[i] = (uint32_t)(cur / count);
        rem = cur % count;
    }

    // 3. position p of the most significant set bit of the quotient
    int p = -1;
    for (int i = 9; i >= 0 && p < 0; i--) {
        if (quo[i]) {
            int lz = 0;
            uint32_t t = quo[i];
            while (!(t & 0x80000000u)) { t <<= 1; lz++; }
            p = 32 * i + 31 - lz;
        }
    }
    // the mean is (quo + rem/count) * 2^-149; quo == 0 means it is below the
    // smallest subnormal: round on rem/count alone
    auto bit_at = [&](int k) -> uint32_t {
        return (k < 0 || k >= 320) ? 0u : ((quo[k >> 5] >> (k & 31)) & 1u);
    };
    auto any_below = [&](int k) -> bool {          // any quotient bit in [0, k)
        for (int i = 0; i < 10; i++) {
            int lo = 32 * i;
            if (lo >= k) break;
            uint32_t w = quo[i];
            int n = k - lo;
            if (n < 32) w &= (1u << n) - 1u;
            if (w) return true;
        }
        return false;
    };

    if (p < 0) {
        // 0 < mean < 2^-149: nearest of 0 and 2^-149; a tie goes to 0 (even)
        return (2 * rem > count) ? 1u : 0u;
    }
    // keep bits [s, p] as the significand, s = max(p - 23, 0)
    int s = p >= 23 ? p - 23 : 0;
    uint32_t mant = 0;
    for (int k = p; k >= s; k--) mant = (mant << 1) | bit_at(k);
    bool up;
    if (s > 0) {
        // dropped part = bits [0, s) of the quotient plus rem/count
        uint32_t round_bit = bit_at(s - 1);
        bool sticky = any_below(s - 1) || rem != 0;
        up = round_bit && (sticky || (mant & 1u));
    } else {
        // every quotient bit is kept; the fraction rem/count decides
        up = (2 * rem > count) || (2 * rem == count && (mant & 1u));
    }
    if (up) mant += 1;
    if (p < 23) return mant;                        // subnormal (mant <= 2^23)
    // value = mant * 2^(s - 149) with mant in [2^23, 2^24]
    return ((uint32_t)(p - 23) << 23) + mant;
}

}  // namespace qlora
