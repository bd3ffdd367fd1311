/*
 * Oracle: plain CPU restatement of the NF4 + double-quantization codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; it exists so that tests and the CPU baseline can check the
 * CUDA path against an independent, slow, obviously-correct implementation.
 *
 * Source of every step: "QLoRA: Efficient Finetuning of Quantized LLMs"
 * (inquiringlines.com/papers/2305.14314), section "Method":
 *   - storage/compute data types ("whenever a QLORA weight tensor is used, we
 *     dequantize the tensor to BFloat16")      -> oracle_dequantize
 *   - "4-bit NormalFloat Quantization", step (3): rescale each block by its
 *     absolute maximum into [-1, 1], then quantize to the nearest value of
 *     the 16-entry data type
 *                                              -> oracle_quantize_blocks
 *   - "Double Quantization": the 32-bit block constants (blocksize 64) are
 *     themselves quantized                      -> oracle_dq_encode
 * The second-level format (8-bit float, 256 constants per group, mean
 * subtracted) is not on the page; the readings used are:
 *   - 8-bit float = OCP E4M3 ("fn": bias 7, no infinity, max 448),
 *   - the mean is one fp32 value per tensor (computed by the Python side of
 *     the oracle as the exactly rounded arithmetic mean, then passed in),
 *   - each group is scaled so that its largest |c1 - mean| maps to 448.
 *
 * Every fp32 operation below is a single IEEE-754 binary32 operation with
 * round-to-nearest-even (x86-64 SSE, compiled with -ffp-contract=off so that
 * no multiply-add is fused behind our back); fmaf() is glibc's correctly
 * rounded fused multiply-add.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---- scalar helpers --------------------------------------------------- */

/* bf16 = upper 16 bits of binary32, rounded to nearest, ties to even.
 * Inputs are finite (the codec never produces NaN from finite inputs). */
uint16_t oracle_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* Value of an OCP E4M3 ("e4m3fn") code straight from the format definition:
 * 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0 is
 * subnormal (m * 2^-9); codes 0x7F / 0xFF are NaN and never produced here. */
double oracle_e4m3_value(uint8_t code)
{
    int s = code >> 7, E = (code >> 3) & 15, m = code & 7;
    double mag = (E == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), E - 10);
    return s ? -mag : mag;
}

/* Nearest E4M3 code to t by exhaustive search over the 127 finite
 * magnitudes; an exact tie goes to the code with even mantissa (the IEEE
 * round-half-to-even rule); |t| beyond 448 saturates to 448; the sign bit is
 * t's sign bit, so a negative value that rounds to zero gives 0x80. */
uint8_t oracle_e4m3_encode(float t)
{
    double mag = fabs((double)t);
    if (mag > 448.0) mag = 448.0; /* saturate: 448 is the largest finite value */
    int best = 0;
    double best_d = mag; /* distance to code 0 (value 0) */
    for (int c = 1; c <= 0x7E; c++) {
        double d = fabs(mag - oracle_e4m3_value((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(best | (signbit(t) ? 0x80 : 0));
}

/* ---- quantize, first level ---------------------------------------------- */

/* For each block b of 64 consecutive values x[64b .. 64b+63]:
 *   c1_b   = max |x|                                   (exact)
 *   zero block (c1_b below the smallest normal fp32, 2^-126): every code is
 *   the index of the codebook's zero.
 *   otherwise r = RN32(1 / c1_b), n = RN32(x * r) and the code is the index
 *   of the codebook value nearest to n, found by trying all 16; on an exact
 *   tie the lower index wins.  The distances are taken in double precision,
 *   which is exact whenever two candidates are close to a tie (all operands
 *   are binary32 numbers of similar magnitude there).
 * codes[] receives one code per element (0..15). */
void oracle_quantize_blocks(const float *x, int64_t nblocks, const float q[16],
                            float *c1, uint8_t *codes)
{
    int zero_idx = 0;
    for (int j = 0; j < 16; j++)
        if (q[j] == 0.0f) zero_idx = j;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; b++) {
        const float *xb = x + 64 * b;
        float amax = 0.0f;
        for (int i = 0; i < 64; i++) {
            float a = fabsf(xb[i]);
            if (a > amax) amax = a;
        }
        c1[b] = amax;
        uint8_t *cb = codes + 64 * b;
        if (amax < 0x1p-126f) {
            for (int i = 0; i < 64; i++) cb[i] = (uint8_t)zero_idx;
            continue;
        }
        float r = 1.0f / amax;
        for (int i = 0; i < 64; i++) {
            float n = xb[i] * r;
            int best = 0;
            double best_d = fabs((double)n - (double)q[0]);
            for (int j = 1; j < 16; j++) {
                double d = fabs((double)n - (double)q[j]);
                if (d < best_d) {
                    best = j;
                    best_d = d;
                }
            }
            cb[i] = (uint8_t)best;
        }
    }
}

/* Two 4-bit codes per byte: element 2j in bits 0-3, element 2j+1 in bits 4-7. */
void oracle_pack_nibbles(const uint8_t *codes, int64_t n, uint8_t *packed)
{
    for (int64_t j = 0; j < n / 2; j++)
        packed[j] = (uint8_t)((codes[2 * j] & 15) | ((codes[2 * j + 1] & 15) << 4));
}

void oracle_unpack_nibbles(const uint8_t *packed, int64_t n, uint8_t *codes)
{
    for (int64_t j = 0; j < n / 2; j++) {
        codes[2 * j] = packed[j] & 15;
        codes[2 * j + 1] = packed[j] >> 4;
    }
}

/* ---- quantize, second level (double quantization) ------------------------ */

/* Groups of `group` consecutive c1 (the last one may be short).  Per group g:
 *   d     = RN32(c1 - mu)
 *   amax  = max |d|
 *   c2_g  = RN32(amax / 448)
 *   e     = 0 for every member if c2_g == 0, else E4M3(RN32(d / c2_g)).      */
void oracle_dq_encode(const float *c1, int64_t nblocks, int32_t group, float mu,
                      float *c2, uint8_t *e)
{
    int64_t ngroups = (nblocks + group - 1) / group;
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < ngroups; g++) {
        int64_t lo = g * group, hi = lo + group < nblocks ? lo + group : nblocks;
        float amax = 0.0f;
        for (int64_t b = lo; b < hi; b++) {
            float d = fabsf(c1[b] - mu);
            if (d > amax) amax = d;
        }
        float s = amax / 448.0f;
        c2[g] = s;
        for (int64_t b = lo; b < hi; b++) {
            if (s == 0.0f) {
                e[b] = 0;
            } else {
                float d = c1[b] - mu;
                e[b] = oracle_e4m3_encode(d / s);
            }
        }
    }
}

/* ---- dequantize ----------------------------------------------------------- */

/* Per block b (group g = b / group):
 *   c1'  = fmaf(E4M3value(e_b), c2_g, mu)          (one rounding)
 *   w    = bf16_RNE( RN32(q[code] * c1') )          per element.            */
void oracle_dequantize(const uint8_t *packed, const uint8_t *e, const float *c2,
                       float mu, const float q[16], int64_t nblocks, int32_t group,
                       uint16_t *w)
{
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; b++) {
        float ev = (float)oracle_e4m3_value(e[b]);
        float c1p = fmaf(ev, c2[b / group], mu);
        for (int i = 0; i < 64; i++) {
            int64_t idx = 64 * b + i;
            uint8_t byte = packed[idx / 2];
            int code = (idx & 1) ? (byte >> 4) : (byte & 15);
            float v = q[code] * c1p;
            w[idx] = oracle_bf16_rne(v);
        }
    }
}

/* The products RN32(q[code] * c1') before the 16-bit rounding: the fp16
 * compute dtype rounds these to binary16 (the caller does that). */
void oracle_dequantize_f32(const uint8_t *packed, const uint8_t *e, const float *c2,
                           float mu, const float q[16], int64_t nblocks, int32_t group,
                           float *w)
{
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; b++) {
        float ev = (float)oracle_e4m3_value(e[b]);
        float c1p = fmaf(ev, c2[b / group], mu);
        for (int i = 0; i < 64; i++) {
            int64_t idx = 64 * b + i;
            uint8_t byte = packed[idx / 2];
            int code = (idx & 1) ? (byte >> 4) : (byte & 15);
            w[idx] = q[code] * c1p;
        }
    }
}

