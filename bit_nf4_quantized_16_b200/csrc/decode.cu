// QLoRA forward for a handful of tokens (M <= 16) on sm_100a: the decode
// shape, where the product is bound by streaming the packed 4-bit weight
// from HBM (0.516 B per weight against 2 M FLOP).
//
//   Y = X W'^T + H B^T,  H = s X A^T
//
// ("QLoRA: Efficient Finetuning of Quantized LLMs", section "Method": the
// 4-bit weight is dequantized to BFloat16 and multiplied in 16-bit; the LoRA
// term x_out = (W + BA) x_in from the mbrenndoerfer.com essay, section
// "Low-Rank Adaptation (LoRA)").
//
// decode_gemv_kernel: each warp owns 16 rows of W (or of A) and a range of the
// contraction.  Every lane streams the packed codes of its two rows with
// 16-byte loads (32 codes = 32 consecutive k per row), expands them with the
// dequantizer's arithmetic (w = bf16(RN32(q[code] * c1')), bit-identical)
// straight into the A fragments of mma.sync m16n8k16, and multiplies them with
// X.  One byte of packed codes is one A register (two neighbouring k), so the
// expansion looks up both codebook values of a byte at once in a 256-entry
// pair table in shared memory.  The block constants c1' of a warp's 16 rows
// are decoded once per 12 steps into shared memory.  The
// contraction index is permuted the same way on both operands (a fragment's
// k slots map to the lane's 32 consecutive k), so no shared-memory transpose
// is needed; the tensor cores only replace the 2 M FMAs per weight that CUDA
// cores could not keep up with at 16 tokens.  Rows of A (the LoRA down
// projection) run through the same loop without expansion.  Partial products
// of each contraction split are written in fp32.
//
// decode_finalize_kernel: sums the splits in a fixed order (deterministic),
// forms H = s X A^T (fp32, optionally saved for the backward pass), adds
// H B^T and stores Y in bf16 or fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "debug.cuh"
#include "decode.cuh"
#include "nf4_expand.cuh"
#include "sm100.cuh"

namespace qlora {
namespace {

constexpr int kDecWarps = 8;                    // 16 rows each: 128 rows per CTA
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecRows = 16 * kDecWarps;
constexpr int kDecCtasPerSm = 2;   // resident CTAs per SM (registers: the prefetched steps)

struct DecodeParams {
    const uint8_t *packed;
    const uint8_t *code2;
    const float *c2;
    const float *mean;
    float q[16];
    const __nv_bfloat16 *X;   // [M][K]
    const __nv_bfloat16 *Xa;  // [M][K]: input of the adapter rows (X, or the dropped-out input under LoRA dropout)
    const __nv_bfloat16 *A;   // [r][K]
    int64_t N, K, kblocks;
    int M, r;
    int row_tiles;            // CTAs along the rows of W; the CTAs after them take the rows of A
    int dblk_per_split;       // 128-wide contraction steps per split
    int n_dblk;               // total 128-wide steps (the last may hold only 64)
    float *part;              // [splits][M][N]: partial products of W
    float *part_h;            // [kAPieces][M][r]: partial products of A
};

// The rows of A are bf16 already (4x the bytes of a packed row): their whole
// contraction is cut into kAPieces ranges, one warp per (16 rows, range), all
// in the CTAs of split 0.
constexpr int kAPieces = 8;
// 128-wide steps of W in flight per warp (fewer with two token tiles, whose
// accumulators and X fragments take the registers)
template <int NT>
constexpr int prefetch_depth() { return NT == 1 ? 4 : 3; }
// 128-wide steps whose block constants a warp decodes at once (a multiple of
// both prefetch depths): 24 blocks of each of its 16 rows.
constexpr int kScaleSteps = 12;
constexpr int kScaleBlocks = 2 * kScaleSteps;
constexpr int kScaleStride = kScaleBlocks + 1;   // odd row stride: a warp's reads hit distinct banks

// Pair table: entry e (one byte of packed codes, the lower k in its low
// nibble) holds (q[e & 15], q[e >> 4]).  Each entry is a 256-byte row of 32
// copies, one 8-byte slot per lane, so the 32 lookups of a warp never share a
// bank whatever their entries.  Then the block constants: per warp 16 rows x
// kScaleStride floats.
constexpr uint32_t kPairTableBytes = 256 * 32 * 8;   // 64 KB
constexpr uint32_t kScaleBytes = kDecWarps * 16 * kScaleStride * 4;
// X of the CTA's current kPrefetch steps, double-buffered: (8 NT) token rows
// of 128 kPrefetch bf16 (24 KB for two token tiles)
template <int NT>
constexpr uint32_t x_stage_bytes() { return 2u * (8 * NT) * (128 * prefetch_depth<NT>()) * 2; }
template <int NT>
constexpr uint32_t dec_smem_bytes() { return kPairTableBytes + kScaleBytes + (NT == 2 ? x_stage_bytes<2>() : 0u); }

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Two dequantized weights (one byte of codes, the lower k in the low half):
// the shared-memory offset [lane slot, entry] is one byte permute of the code
// word and lane8 (= 8 * lane).  Same products and rounding as nf4::expand8.
template <bool F16, int kByte>
__device__ __forceinline__ uint32_t expand_pair(uint32_t word, uint32_t lane8, const char *tab, float c1p)
{
    const uint32_t off = __byte_perm(word, lane8, 0x5504u | (kByte << 4));   // lane8 + 256 * byte
    const float2 qv = *reinterpret_cast<const float2 *>(tab + off);
    float lo, hi;
    nf4::mul2(qv.x, qv.y, c1p, lo, hi);
    return nf4::pack16x2<F16>(lo, hi);
}

template <bool F16>
__device__ __forceinline__ uint4 expand8_pairs(uint32_t word, uint32_t lane8, const char *tab, float c1p)
{
    return make_uint4(expand_pair<F16, 0>(word, lane8, tab, c1p), expand_pair<F16, 1>(word, lane8, tab, c1p),
                      expand_pair<F16, 2>(word, lane8, tab, c1p), expand_pair<F16, 3>(word, lane8, tab, c1p));
}

__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_cached_v4(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// D += A B, m16n8k16, bf16 (or, F16, fp16) inputs, fp32 accumulators.
template <bool F16>
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    if constexpr (F16)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 128-wide step of this lane's two rows: packed codes.  Loads only:
// nothing computed from a loaded value until the step is used, so issuing the
// next step's loads never waits for them.
struct WStage {
    uint4 pg, pg8;
};

// Fragment layout (lane = 4 g + c): A regs {a0a1, a2a3, a4a5, a6a7} hold rows
// g, g+8, g, g+8 at k slots {2c, 2c+1}, {2c, 2c+1}, {2c+8, 2c+9}, {2c+8, 2c+9};
// B regs {b0b1, b2b3} hold token g at the same two slot pairs.  Slot pair
// {2c, 2c+1} of step t is real k = base + 32 c + 4 t + {0, 1}, pair {2c+8,
// 2c+9} is + {2, 3}: lane c's 32 consecutive k feed 8 steps, four per step.
// mma.sync is warp-collective: every lane calls this; lanes whose k is past the
// end pass kin = false and multiply zeros.
template <int NT, bool F16>
__device__ __forceinline__ void mma_step(float (&acc)[NT][2][4], const uint4 (&ea)[4], const uint4 (&eb)[4],
                                         const __nv_bfloat16 *const (&xrow)[NT], const bool (&xok)[NT], int64_t k,
                                         bool kin, [[maybe_unused]] const __nv_bfloat16 *xbase,
                                         [[maybe_unused]] int64_t xlen)
{
#pragma unroll
    for (int w = 0; w < 4; w++) {
#pragma unroll
        for (int t = 0; t < NT; t++) {
            const uint4 xb = (xok[t] && kin && QLORA_IN((xrow[t] - xbase) + k + 8 * w + 7, xlen))
                                 ? ld_cached_v4(xrow[t] + k + 8 * w) : make_uint4(0, 0, 0, 0);
            mma_bf16_16816<F16>(acc[t][0], ea[w].x, eb[w].x, ea[w].y, eb[w].y, xb.x, xb.y);
            mma_bf16_16816<F16>(acc[t][1], ea[w].z, eb[w].z, ea[w].w, eb[w].w, xb.z, xb.w);
        }
    }
}

// mma_step with X from the staged chunk: xs_row[t] is token 8t+g's row of the
// chunk; 16-byte unit u of a row sits at u ^ (bit 3 of u) ^ (2 * (token & 1)),
// so the 8 lanes of each quarter-warp (two tokens, four k slices 64 bytes
// apart) read 8 distinct bank groups.  jb = 16 * (step in chunk) + 4 c, sw the
// lane's swizzle bits.
template <int NT, bool F16>
__device__ __forceinline__ void mma_step_xs(float (&acc)[NT][2][4], const uint4 (&ea)[4], const uint4 (&eb)[4],
                                            const char *const (&xs_row)[NT], const bool (&xok)[NT], int jb, int sw,
                                            bool kin)
{
#pragma unroll
    for (int w = 0; w < 4; w++) {
#pragma unroll
        for (int t = 0; t < NT; t++) {
            const uint4 xb = (xok[t] && kin) ? *reinterpret_cast<const uint4 *>(xs_row[t] + ((jb + (w ^ sw)) << 4))
                                             : make_uint4(0, 0, 0, 0);
            mma_bf16_16816<F16>(acc[t][0], ea[w].x, eb[w].x, ea[w].y, eb[w].y, xb.x, xb.y);
            mma_bf16_16816<F16>(acc[t][1], ea[w].z, eb[w].z, ea[w].w, eb[w].w, xb.z, xb.w);
        }
    }
}

// F16: the fp16 compute dtype (fp16 X, A and expansion).
template <int NT, bool F16>
__global__ void __launch_bounds__(kDecThreads, kDecCtasPerSm) decode_gemv_kernel(const __grid_constant__ DecodeParams p)
{
    extern __shared__ __align__(16) char dec_smem[];
    __shared__ float s_q[16];
    const bool w_rows = (int)blockIdx.x < p.row_tiles;
    if (w_rows) {
        // the pair table depends on the parameters only: built before the
        // dependency wait, overlapping the previous kernel's tail
        if (threadIdx.x < 16) s_q[threadIdx.x] = p.q[threadIdx.x];
        __syncthreads();
        float2 *tab = reinterpret_cast<float2 *>(dec_smem);
        for (int i = threadIdx.x; i < 256 * 32; i += kDecThreads) {
            const int e = i >> 5;   // a warp writes one entry's 32 slots
            tab[i] = make_float2(s_q[e & 15], s_q[e >> 4]);
        }
        __syncthreads();
    }
    sm100::pdl_wait();
    sm100::pdl_trigger();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int sp = blockIdx.y;
    int d0 = sp * p.dblk_per_split;
    int d1 = min(d0 + p.dblk_per_split, p.n_dblk);

    float acc[NT][2][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int i = 0; i < 4; i++) acc[t][0][i] = acc[t][1][i] = 0.0f;
    const __nv_bfloat16 *xrow[NT];
    bool xok[NT];
#pragma unroll
    for (int t = 0; t < NT; t++) {
        const int tok = 8 * t + g;
        xok[t] = tok < p.M;
        xrow[t] = p.X + (int64_t)(xok[t] ? tok : 0) * p.K;
    }

    if (!w_rows) {
        // ---- rows of A: warp task = (16-row group, piece of the contraction)
        if (sp != 0) return;
#pragma unroll
        for (int t = 0; t < NT; t++) xrow[t] = p.Xa + (int64_t)(xok[t] ? 8 * t + g : 0) * p.K;
        const int groups = (p.r + 15) / 16;
        const int task = ((int)blockIdx.x - p.row_tiles) * kDecWarps + warp;
        const int grp = task % groups, qtr = task / groups;
        if (qtr >= kAPieces) return;
        const int qper = (p.n_dblk + kAPieces - 1) / kAPieces;
        d0 = qtr * qper;
        d1 = min(p.n_dblk, d0 + qper);
        const int64_t rg = 16 * grp + g, rg8 = rg + 8;
        const bool ok_g = rg < p.r, ok_g8 = rg8 < p.r;
        for (int d = d0; d < d1; d++) {
            const int64_t k = (int64_t)d * 128 + 32 * c;
            const bool k_ok = k < p.K;
            uint4 ea[4], eb[4];
#pragma unroll
            for (int w = 0; w < 4; w++) {
                ea[w] = (ok_g && k_ok && QLORA_IN(rg * p.K + k + 8 * w + 7, (int64_t)p.r * p.K))
                            ? ld_cached_v4(p.A + rg * p.K + k + 8 * w) : make_uint4(0, 0, 0, 0);
                eb[w] = (ok_g8 && k_ok && QLORA_IN(rg8 * p.K + k + 8 * w + 7, (int64_t)p.r * p.K))
                            ? ld_cached_v4(p.A + rg8 * p.K + k + 8 * w) : make_uint4(0, 0, 0, 0);
            }
            mma_step<NT, F16>(acc, ea, eb, xrow, xok, k, k_ok, p.Xa, (int64_t)p.M * p.K);
        }
        float *part = p.part_h + (int64_t)qtr * p.M * p.r;
#pragma unroll
        for (int t = 0; t < NT; t++) {
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int tok = 8 * t + 2 * c + (i & 1);
                const int64_t row = (i < 2) ? rg : rg8;
                if (tok < p.M && row < p.r && QLORA_IN(((int64_t)qtr * p.M + tok) * p.r + row, (int64_t)kAPieces * p.M * p.r))
                    part[(int64_t)tok * p.r + row] = __fadd_rn(acc[t][0][i], acc[t][1][i]);
            }
        }
        return;
    }

    // ---- rows of W: packed codes streamed kPrefetch steps ahead
    constexpr int kPrefetch = prefetch_depth<NT>();
    static_assert(kScaleSteps % kPrefetch == 0, "block constants are refilled at a prefetch boundary");
    // X staged in shared memory once per CTA (two token tiles: measured faster
    // than every warp loading it through L1) or loaded by each warp (one tile)
    constexpr bool kStageX = NT == 2;
    const int64_t row0 = (int64_t)blockIdx.x * kDecRows + 16 * warp;
    // with staged X a warp past the last row still takes part in the CTA's
    // chunk barriers
    const bool wrow = row0 < p.N;
    if (!kStageX && !wrow) return;
    const int64_t rg = row0 + g, rg8 = row0 + g + 8;
    const bool ok_g = rg < p.N, ok_g8 = rg8 < p.N;
    const float mu = *p.mean;
    const int64_t half_k = p.K / 2;
    const char *tab = dec_smem;
    const uint32_t lane8 = 8u * (uint32_t)lane;
    float *sc = reinterpret_cast<float *>(dec_smem + kPairTableBytes) + warp * 16 * kScaleStride;
    auto load = [&](int d, WStage &st) {
        const int64_t k = (int64_t)d * 128 + 32 * c;
        const bool in = d < d1 && k < p.K;
        const uint4 z = make_uint4(0, 0, 0, 0);
        // (checked only where the access happens)
        const bool ld_g = in && ok_g && QLORA_IN(rg * half_k + k / 2 + 15, p.N * half_k);
        const bool ld_g8 = in && ok_g8 && QLORA_IN(rg8 * half_k + k / 2 + 15, p.N * half_k);
        st.pg = ld_g ? ld_stream_v4(p.packed + rg * half_k + k / 2) : z;
        st.pg8 = ld_g8 ? ld_stream_v4(p.packed + rg8 * half_k + k / 2) : z;
    };
    // c1' of the warp's 16 rows for the blocks of steps d .. d+kScaleSteps-1,
    // one row at a time: lane j < 24 takes block 2d + j, so each load
    // instruction reads one contiguous run of a row's block codes (and mostly
    // one group scale); blocks past the row's end (the upper half of a final
    // 64-wide step) get 0
    auto fill_scales = [&](int d) {
        const int64_t blk = 2 * (int64_t)d + lane;
        [[maybe_unused]] const int64_t nblk = p.N * p.kblocks;
        __syncwarp();   // every lane has read the previous range
        if (lane < kScaleBlocks) {
#pragma unroll
            for (int r = 0; r < 16; r++) {
                const int64_t row = row0 + r;
                const int64_t b = row * p.kblocks + blk;
                const bool ok = row < p.N && blk < p.kblocks && QLORA_IN(b, nblk) && QLORA_IN(b >> 8, (nblk + 255) / 256);
                sc[r * kScaleStride + lane] = ok ? nf4::block_scale(__ldg(p.code2 + b), __ldg(p.c2 + (b >> 8)), mu) : 0.0f;
            }
        }
        __syncwarp();
    };
    // X of steps d .. d+kPrefetch-1 into buffer buf, by all threads of the CTA
    constexpr int kXUnits = 16 * kPrefetch;               // 16-byte units per token row
    constexpr uint32_t kXRowBytes = 16 * kXUnits;
    constexpr uint32_t kXBufBytes = 8 * NT * kXRowBytes;
    char *xs = dec_smem + kPairTableBytes + kScaleBytes;
    auto stage_x = [&](int d, int buf) {
        char *dst = xs + buf * kXBufBytes;
        const int64_t kb = (int64_t)d * 128;
        const int64_t kend = min((int64_t)d1 * 128, p.K);
        for (int idx = threadIdx.x; idx < 8 * NT * kXUnits; idx += kDecThreads) {
            const int row = idx / kXUnits, u = idx % kXUnits;
            const int64_t k = kb + 8 * u;
            if (row < p.M && k < kend && QLORA_IN(row * p.K + k + 7, (int64_t)p.M * p.K))
                cp_async16(dst + row * kXRowBytes + ((u ^ ((u >> 3) & 1) ^ ((row & 1) << 1)) << 4), p.X + row * p.K + k);
        }
        cp_async_commit();
    };
    const int sw = (c >> 1) ^ ((g & 1) << 1);
    WStage st[kPrefetch];
#pragma unroll
    for (int i = 0; i < kPrefetch; i++) load(d0 + i, st[i]);
    if constexpr (kStageX) stage_x(d0, 0);
    for (int d = d0, ci = 0; d < d1; d += kPrefetch, ci++) {
        if constexpr (kStageX) {
            cp_async_wait_all();
            __syncthreads();   // this chunk's X is visible; every warp is done with the previous chunk
            if (d + kPrefetch < d1) stage_x(d + kPrefetch, (ci + 1) & 1);
            if (!wrow) continue;
        }
        const char *xs_row[NT];
#pragma unroll
        for (int t = 0; t < NT; t++) xs_row[t] = xs + (ci & 1) * kXBufBytes + (8 * t + g) * kXRowBytes;
        if ((d - d0) % kScaleSteps == 0) fill_scales(d);
        const float *sc_d = sc + 2 * ((d - d0) % kScaleSteps) + (c >> 1);
#pragma unroll
        for (int i = 0; i < kPrefetch; i++) {
            if (d + i < d1) {
                const int64_t k = (int64_t)(d + i) * 128 + 32 * c;
                const bool kin = k < p.K;   // false only for the upper half of a final 64-wide step
                {
                    const float sg = sc_d[g * kScaleStride + 2 * i];
                    const float sg8 = sc_d[(g + 8) * kScaleStride + 2 * i];
                    uint4 ea[4], eb[4];
                    ea[0] = expand8_pairs<F16>(st[i].pg.x, lane8, tab, sg);
                    ea[1] = expand8_pairs<F16>(st[i].pg.y, lane8, tab, sg);
                    ea[2] = expand8_pairs<F16>(st[i].pg.z, lane8, tab, sg);
                    ea[3] = expand8_pairs<F16>(st[i].pg.w, lane8, tab, sg);
                    eb[0] = expand8_pairs<F16>(st[i].pg8.x, lane8, tab, sg8);
                    eb[1] = expand8_pairs<F16>(st[i].pg8.y, lane8, tab, sg8);
                    eb[2] = expand8_pairs<F16>(st[i].pg8.z, lane8, tab, sg8);
                    eb[3] = expand8_pairs<F16>(st[i].pg8.w, lane8, tab, sg8);
                    if constexpr (kStageX)
                        mma_step_xs<NT, F16>(acc, ea, eb, xs_row, xok, 16 * i + 4 * c, sw, kin);
                    else
                        mma_step<NT, F16>(acc, ea, eb, xrow, xok, k, kin, p.X, (int64_t)p.M * p.K);
                }
                load(d + i + kPrefetch, st[i]);
            }
        }
    }

    // acc[t] = {(row g, token 8t+2c), (row g, 8t+2c+1), (row g+8, 8t+2c), (row g+8, 8t+2c+1)}
    float *part = p.part + (int64_t)sp * p.M * p.N;
#pragma unroll
    for (int t = 0; t < NT; t++) {
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int tok = 8 * t + 2 * c + (i & 1);
            const int64_t row = (i < 2) ? rg : rg8;
            if (tok < p.M && row < p.N && QLORA_IN(((int64_t)sp * p.M + tok) * p.N + row, (int64_t)gridDim.y * p.M * p.N))
                part[(int64_t)tok * p.N + row] = __fadd_rn(acc[t][0][i], acc[t][1][i]);
        }
    }
}

// Up to 8 split partials of token m at outputs n, splits s0 .. s0+7.
__device__ __forceinline__ void load_splits8(float (&v)[8], const float *part, int s0, int splits, int m, int M,
                                             int64_t N, int64_t n)
{
#pragma unroll
    for (int i = 0; i < 8; i++)
        v[i] = s0 + i < splits ? __ldcg(part + ((int64_t)(s0 + i) * M + m) * N + n) : 0.0f;
}

// One CTA per 256 outputs n (all tokens): the H rows of every token from the
// A partials (fixed order) in shared memory, B[n] in registers, then
// y[m][n] = sum of the W splits + H[m] . B[n].  The chain of dependent
// memory waits is kept short: B[n] is read before the dependency wait (it is
// not written by the GEMV; everything before the GEMV in the stream completed
// before the GEMV let this kernel start, and the loads go through L2 only),
// and the first token's split partials are in flight during the H reduction.
// y_type: QLORA_BF16, QLORA_FP32 or QLORA_FP16; b_f16: B holds fp16 (the fp16
// compute dtype) instead of bf16.
__global__ void __launch_bounds__(256) decode_finalize_kernel(const float *part, const float *part_h, int splits,
                                                            int M, int64_t N, int r, float scale,
                                                            const __nv_bfloat16 *B, int b_f16, void *Y, int y_type,
                                                            float *H_save)
{
    __shared__ float h[kDecodeMaxTokens * 128];
    const int64_t n = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const bool has_row = n < N;
    uint4 bv[16];   // B[n][0 .. r), r <= 128
    const __nv_bfloat16 *bn = B + (has_row ? n : 0) * r;
#pragma unroll
    for (int j = 0; j < 16; j++)
        bv[j] = (has_row && 8 * j < r) ? __ldcg(reinterpret_cast<const uint4 *>(bn + 8 * j)) : make_uint4(0, 0, 0, 0);
    sm100::pdl_wait();
    sm100::pdl_trigger();
    float v[8];
    load_splits8(v, part, 0, has_row ? splits : 0, 0, M, N, n);
    for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
        if (!QLORA_IN(i, kDecodeMaxTokens * 128)) break;
        float hv = 0.0f;
#pragma unroll
        for (int s = 0; s < kAPieces; s++) hv = __fadd_rn(hv, part_h[(int64_t)s * M * r + i]);
        hv = __fmul_rn(scale, hv);
        h[i] = hv;
        if (H_save && blockIdx.x == 0) H_save[i] = hv;
    }
    __syncthreads();
    if (!has_row) return;
    for (int m = 0; m < M; m++) {
        // eight splits' loads ahead of their in-order additions
        float y = 0.0f;
        for (int s0 = 0; s0 < splits; s0 += 8) {
            if (m > 0 || s0 > 0) load_splits8(v, part, s0, splits, m, M, N, n);
#pragma unroll
            for (int i = 0; i < 8; i++)
                if (s0 + i < splits) y = __fadd_rn(y, v[i]);
        }
        const float *hm = h + m * r;
        float l = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; j++) {
            if (8 * j >= r) break;
            const uint32_t w[4] = {bv[j].x, bv[j].y, bv[j].z, bv[j].w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                float b0, b1;
                if (b_f16) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
                    b0 = f.x;
                    b1 = f.y;
                } else {
                    b0 = __uint_as_float(w[i] << 16);
                    b1 = __uint_as_float(w[i] & 0xFFFF0000u);
                }
                l = __fmaf_rn(hm[8 * j + 2 * i], b0, l);
                l = __fmaf_rn(hm[8 * j + 2 * i + 1], b1, l);
            }
        }
        y = __fadd_rn(y, l);
        if (y_type == QLORA_FP32)
            static_cast<float *>(Y)[(int64_t)m * N + n] = y;
        else if (y_type == QLORA_FP16)
            static_cast<__half *>(Y)[(int64_t)m * N + n] = __float2half_rn(y);
        else
            static_cast<__nv_bfloat16 *>(Y)[(int64_t)m * N + n] = __float2bfloat16_rn(y);
    }
}

int ceil_div_i(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

struct DecodePlan {
    int row_tiles, a_ctas, n_dblk, splits, per;
    size_t part_bytes, part_h_bytes;
};

DecodePlan decode_plan(int64_t M, int64_t N, int64_t K, int r, int sms)
{
    DecodePlan d;
    d.row_tiles = ceil_div_i(N, kDecRows);
    d.a_ctas = ceil_div_i((int64_t)((r + 15) / 16) * kAPieces, kDecWarps);
    d.n_dblk = ceil_div_i(K, 128);
    // about four CTAs per SM in all (two waves at two resident per SM: measured
    // faster than one or one and a half), at least two 128-wide steps per split
    int want = ceil_div_i((int64_t)4 * sms, d.row_tiles + d.a_ctas);
    want = std::max(1, std::min(want, std::max(1, d.n_dblk / 2)));
    d.per = ceil_div_i(d.n_dblk, want);
    d.splits = ceil_div_i(d.n_dblk, d.per);
    d.part_bytes = ((size_t)d.splits * M * N * 4 + 255) / 256 * 256;
    d.part_h_bytes = (size_t)kAPieces * M * r * 4;
    return d;
}

}  // namespace

size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K, int r, int sms)
{
    const DecodePlan d = decode_plan(M, N, K, r, sms);
    return d.part_bytes + d.part_h_bytes;
}

qlora_status run_decode_fwd(const qlora_nf4_weight *w, const void *X, const void *Xa, int64_t M, const void *A,
                            const void *B, int r, float scale, void *Y, qlora_dtype y_dtype, float *H_save, void *ws,
                            size_t ws_bytes, const DeviceInfo &dev, cudaStream_t s, bool f16)
{
    if (M < 1 || M > kDecodeMaxTokens) return QLORA_ERR_SHAPE;
    const DecodePlan d = decode_plan(M, w->rows, w->cols, r, dev.sms);
    if (ws_bytes < d.part_bytes + d.part_h_bytes) return QLORA_ERR_WORKSPACE;
    DecodeParams p;
    p.packed = w->packed;
    p.code2 = w->code2;
    p.c2 = w->c2;
    p.mean = w->mean;
    for (int i = 0; i < 16; i++) p.q[i] = w->codebook[i];
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.Xa = static_cast<const __nv_bfloat16 *>(Xa);
    p.A = static_cast<const __nv_bfloat16 *>(A);
    p.N = w->rows;
    p.K = w->cols;
    p.kblocks = w->cols / QLORA_BLOCK;
    p.M = (int)M;
    p.r = r;
    p.row_tiles = d.row_tiles;
    p.dblk_per_split = d.per;
    p.n_dblk = d.n_dblk;
    p.part = static_cast<float *>(ws);
    p.part_h = reinterpret_cast<float *>(static_cast<char *>(ws) + d.part_bytes);
    const dim3 grid(d.row_tiles + d.a_ctas, d.splits);
    static PerDeviceOnce attr;
    QLORA_TRY(attr.run(dev.device, []() -> qlora_status {
        QLORA_CUDA_TRY(cudaFuncSetAttribute(decode_gemv_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            dec_smem_bytes<1>()));
        QLORA_CUDA_TRY(cudaFuncSetAttribute(decode_gemv_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            dec_smem_bytes<1>()));
        QLORA_CUDA_TRY(cudaFuncSetAttribute(decode_gemv_kernel<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            dec_smem_bytes<2>()));
        QLORA_CUDA_TRY(cudaFuncSetAttribute(decode_gemv_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            dec_smem_bytes<2>()));
        return QLORA_OK;
    }));
    {
        LaunchScope ls(QLORA_KERNEL_FWD_FUSED, s);
        if (M <= 8)
            QLORA_CUDA_TRY(launch_pdl(f16 ? decode_gemv_kernel<1, true> : decode_gemv_kernel<1, false>, grid,
                                      dim3(kDecThreads), dec_smem_bytes<1>(), s, p));
        else
            QLORA_CUDA_TRY(launch_pdl(f16 ? decode_gemv_kernel<2, true> : decode_gemv_kernel<2, false>, grid,
                                      dim3(kDecThreads), dec_smem_bytes<2>(), s, p));
    }
    {
        LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
        QLORA_CUDA_TRY(launch_pdl(decode_finalize_kernel, dim3(ceil_div_i(w->rows, 256)), dim3(256), 0, s,
                                  (const float *)p.part, (const float *)p.part_h, d.splits, (int)M,
                                  (int64_t)w->rows, r, scale, static_cast<const __nv_bfloat16 *>(B), f16 ? 1 : 0, Y,
                                  (int)y_dtype, H_save));
    }
    return launch_status();
}

}  // namespace qlora
