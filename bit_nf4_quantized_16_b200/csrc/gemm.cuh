// Warp-specialized tcgen05 GEMM for sm_100a, with an optional on-chip NF4
// dequantization producer for the B operand.
//
// D[128*MT x BN] tiles (MT = 1 or 2 accumulators of 128 rows that share one B
// tile, so every dequantized element feeds MT MMAs) accumulate in tensor
// memory (fp32); operands are staged in shared memory in the 128-byte-
// swizzled canonical layouts described in sm100.cuh.  Roles (one CTA per SM,
// persistent over output tiles):
//   warp 0       TMA producer: A tiles and either B tiles or packed NF4 tiles
//   warp 1       MMA issuer (one thread) and TMEM owner
//   warps 4..7   epilogue: TMEM -> registers -> global (bf16 / fp32)
//   warps 8..    dequantization producer (fused modes only): packed 4-bit
//                codes + double-quantized block constants -> bf16 B tile in
//                shared memory, exactly as the stand-alone dequantizer
//                ("QLoRA: Efficient Finetuning of Quantized LLMs", section
//                "Method": the stored weight is dequantized to BFloat16 and
//                multiplied in 16-bit); the bf16 weight never reaches HBM.
// Pipeline: a ring of kStages stages {A, B[, packed]} guarded by mbarriers
// full_a (TMA bytes landed), full_b (dequantized B written), empty (MMAs that
// read the stage completed); two TMEM accumulator buffers let the epilogue of
// one tile overlap the main loop of the next.  Every wait is bounded: on
// timeout the kernel records an error in the device error word and winds
// down instead of hanging.
//
// B operand modes:
//   kBTmaK    B[n][k] bf16, K contiguous (K-major), loaded by TMA
//   kBTmaMN   B[k][n] bf16, N contiguous (MN-major), loaded by TMA
//   kBNf4K    B = W' (dequantized weight [N][K]) used as B[n][k] (forward)
//   kBNf4MN   B = W' used as B[k=row of W][n=column of W] (input gradient:
//             the contraction runs over the rows of W; same shared-memory
//             bytes, described as MN-major)
// An optional second operand pair (A2, B2) adds `k_stages_lora` further
// 64-deep K steps to split 0 of every tile: the LoRA term of the layer.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "nf4_expand.cuh"
#include "sm100.cuh"

namespace qlora {

enum BMode : int { kBTmaK = 0, kBTmaMN = 1, kBNf4K = 2, kBNf4MN = 3 };
// Epilogues: kEpiBf16 stores the tile as bf16; kEpiF32 stores it as fp32,
// into plane `split` of a stack of partial products when the contraction is
// split (out + split * split_stride).  kEpiDropBf16 / kEpiDropF32 store
// drop_base + (kept ? drop_scale * acc : 0) (the adapter term of the input
// gradient under LoRA dropout, added to the frozen path's fp32 product; the
// mask holds bit c % 8 of byte (row * out_ld + c) / 8 per element).
enum Epi : int { kEpiBf16 = 0, kEpiF32 = 1, kEpiDropBf16 = 2, kEpiDropF32 = 3 };

struct GemmParams {
    CUtensorMap tm_a;    // main A operand
    CUtensorMap tm_b;    // main B operand, or packed NF4 codes (uint8 [N][K/2])
    CUtensorMap tm_a2;   // LoRA A operand (K-major)
    CUtensorMap tm_b2;   // LoRA B operand (same majorness as the main B)
    CUtensorMap tm_out;  // bf16 output, box 32 x 32, 64-byte swizzle (CTA-pair kernel's bf16 epilogue)
    // quantized weight constants (fused modes)
    const uint8_t *code2;
    const float *c2;
    const float *mean;
    int64_t kblocks;     // blocks per row of W (cols / 64)
    int64_t wrows;       // rows of W
    float q[16];         // codebook
    // tiling
    int m_tiles, n_tiles, splits;
    int k_stages_total;  // 64-deep main K steps over the full contraction
    int k_stages_split;  // main K steps per split (last split may have fewer)
    int k_stages_lora;   // extra LoRA K steps (split 0 only)
    int a_mn;            // A operand is MN-major
    int a2_x_step;       // x-coordinate advance of the LoRA A operand per 64-deep step
    // output (row-major, leading dimension out_ld elements)
    void *out;
    int64_t out_ld;
    int m_total, n_total;
    int64_t split_stride;  // elements between split planes (partial products)
    const uint8_t *drop_mask;  // kEpiDrop*: kept-input bit mask, [rows][out_ld / 8]
    const float *drop_base;    // kEpiDrop*: fp32 [rows][out_ld] added to the scaled tile
    float drop_scale;          // kEpiDrop*: 1 / (1 - p)
    int *err;            // device error word
    uint64_t timeout_ns; // limit of every pipeline wait
    uint64_t drain_ns;   // limit of the waits for copies and MMAs already in flight after an abort
    int stall_inject;    // failure-detection test hook: the first dequantization warp of CTA 0
                         // (of cluster 0) skips its first arrival, so the MMA's wait runs out
};

template <int BN, int kBMode, int MT>
struct GemmCfg {
    static constexpr bool kFused = kBMode >= kBNf4K;
    static constexpr int kDeqWarps = kFused ? 8 : 0;
    static constexpr int kThreads = 256 + 32 * kDeqWarps;
    static constexpr uint32_t kABytes = MT * 128 * 64 * 2;
    static constexpr uint32_t kBBytes = BN * 64 * 2;
    static constexpr uint32_t kPBytes = kFused ? BN * 32 : 0;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes + kPBytes;
    static constexpr int kMaxStages = (232448 - 2048) / kStageBytes;
    static constexpr int kStages = kMaxStages > 6 ? 6 : kMaxStages;
    static constexpr uint32_t kBarOff = kStages * kStageBytes;
    static constexpr uint32_t kSmemBytes = kBarOff + 512 + 1024;  // barriers etc. + alignment slack
    static constexpr uint32_t kAccCols = MT * BN;                  // one accumulator buffer
    static constexpr uint32_t kTmemCols = 2 * kAccCols < 32 ? 32 : 2 * kAccCols;
    static_assert(2 * kAccCols <= 512, "two accumulator buffers must fit in TMEM");
    static_assert(kStages >= 2, "shared memory too small for two stages");
    // dequantization: blocks per stage (BN rows x 1 block forward, 64 rows x
    // BN/64 blocks for the input gradient: BN blocks either way), threads per block
    static constexpr int kTPB = kFused ? (32 * kDeqWarps) / BN : 1;
};

namespace gemm_detail {

using nf4::block_scale;
using nf4::expand8;

__device__ __forceinline__ void record_timeout(const GemmParams &p, int *abort_flag)
{
    atomicExch(p.err, 1);
    *reinterpret_cast<volatile int *>(abort_flag) = 1;
}

}  // namespace gemm_detail

// F16: the fp16 compute dtype (fp16 operands, fp16 expansion and 16-bit
// outputs) instead of bf16.
template <int BN, int kBMode, int kEpi, int MT, bool F16 = false>
__global__ void __launch_bounds__(GemmCfg<BN, kBMode, MT>::kThreads, 1)
    qgemm_kernel(const __grid_constant__ GemmParams p)
{
    using Cfg = GemmCfg<BN, kBMode, MT>;
    using namespace sm100;
    using namespace gemm_detail;
    constexpr int S = Cfg::kStages;
    constexpr bool kFused = Cfg::kFused;
    constexpr int BM = 128 * MT;

    extern __shared__ uint8_t smem_raw[];
    __shared__ float lut[16];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_a = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
    uint64_t *full_b = full_a + S;
    uint64_t *empty = full_b + S;
    uint64_t *acc_full = empty + S;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto sA = [&](int s) { return smem + s * Cfg::kABytes; };
    auto sB = [&](int s) { return smem + S * Cfg::kABytes + s * Cfg::kBBytes; };
    auto sP = [&](int s) { return smem + S * (Cfg::kABytes + Cfg::kBBytes) + s * Cfg::kPBytes; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full_a[s], 1);
            mbar_init(&full_b[s], Cfg::kDeqWarps > 0 ? Cfg::kDeqWarps : 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
#pragma unroll
        for (int i = 0; i < 16; i++) lut[i] = p.q[i];
        fence_barrier_init();
        tma_prefetch_desc(&p.tm_a);
        tma_prefetch_desc(&p.tm_b);
        if (p.k_stages_lora > 0) {
            tma_prefetch_desc(&p.tm_a2);
            tma_prefetch_desc(&p.tm_b2);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // everything above overlaps the previous kernel's tail; inputs are read below
    pdl_wait();
    pdl_trigger();
    const uint32_t tmem_base = *tmem_slot;
    const int num_tiles = p.m_tiles * p.n_tiles * p.splits;
    volatile int *vabort = abort_flag;

    // tile index -> (m tile, n tile, split); consecutive indices walk M first
    auto decode = [&](int t, int &mt, int &nt, int &sp) {
        mt = t % p.m_tiles;
        t /= p.m_tiles;
        nt = t % p.n_tiles;
        sp = t / p.n_tiles;
    };
    auto stages_of = [&](int sp, int &k_begin, int &n_main) {
        k_begin = sp * p.k_stages_split;
        int e = k_begin + p.k_stages_split;
        if (e > p.k_stages_total) e = p.k_stages_total;
        n_main = e - k_begin;
    };

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        uint32_t it = 0;
        auto drain_loads = [&]() {
            // after an abort: wait (bounded) for the loads still in flight
            for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; j++)
                mbar_wait_bounded(&full_a[j % S], (j / S) & 1, p.drain_ns);
        };
        for (int t = blockIdx.x; t < num_tiles && !*vabort; t += gridDim.x) {
            int mt, nt, sp, kb0, nmain;
            decode(t, mt, nt, sp);
            stages_of(sp, kb0, nmain);
            const int nst = nmain + (sp == 0 ? p.k_stages_lora : 0);
            for (int ks = 0; ks < nst; ks++, it++) {
                const int s = it % S;
                const uint32_t use = it / S;
                if (!mbar_wait_bounded(&empty[s], (use & 1) ^ 1, p.timeout_ns)) {
                    record_timeout(p, abort_flag);
                    break;
                }
                if (*vabort) break;
                const int m0 = mt * BM, n0 = nt * BN;
                if (ks < nmain) {
                    const int k0 = (kb0 + ks) * 64;
                    mbar_arrive_expect_tx(&full_a[s], Cfg::kABytes + (kFused ? Cfg::kPBytes : Cfg::kBBytes));
                    if (!p.a_mn) {
                        tma_load_2d(sA(s), &p.tm_a, &full_a[s], k0, m0);                  // [BM rows][64]
                    } else {
#pragma unroll
                        for (int j = 0; j < 2 * MT; j++) tma_load_2d(sA(s) + 8192 * j, &p.tm_a, &full_a[s], m0 + 64 * j, k0);
                    }
                    if (kBMode == kBTmaK) {
                        tma_load_2d(sB(s), &p.tm_b, &full_a[s], k0, n0);
                    } else if (kBMode == kBTmaMN) {
#pragma unroll
                        for (int j = 0; j < BN / 64; j++) tma_load_2d(sB(s) + 8192 * j, &p.tm_b, &full_a[s], n0 + 64 * j, k0);
                    } else if (kBMode == kBNf4K) {
                        tma_load_2d(sP(s), &p.tm_b, &full_a[s], k0 / 2, n0);     // [BN rows][32 B]
                    } else {
                        tma_load_2d(sP(s), &p.tm_b, &full_a[s], n0 / 2, k0);     // [64 rows][BN/2 B]
                    }
                } else {
                    const int r0 = (ks - nmain) * 64;
                    mbar_arrive_expect_tx(&full_a[s], Cfg::kABytes + Cfg::kBBytes);
                    tma_load_2d(sA(s), &p.tm_a2, &full_a[s], (ks - nmain) * p.a2_x_step, m0);
                    if (kBMode == kBNf4MN || kBMode == kBTmaMN) {
#pragma unroll
                        for (int j = 0; j < BN / 64; j++) tma_load_2d(sB(s) + 8192 * j, &p.tm_b2, &full_a[s], n0 + 64 * j, r0);
                    } else {
                        tma_load_2d(sB(s), &p.tm_b2, &full_a[s], r0, n0);
                    }
                }
            }
        }
        if (*vabort) drain_loads();
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        constexpr bool kBMn = (kBMode == kBTmaMN || kBMode == kBNf4MN);
        const uint32_t idesc = idesc_bf16_f32(128, BN, p.a_mn, kBMn ? 1 : 0, F16);
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok && !*vabort; t += gridDim.x, local++) {
            int mt, nt, sp, kb0, nmain;
            decode(t, mt, nt, sp);
            stages_of(sp, kb0, nmain);
            const int nst = nmain + (sp == 0 ? p.k_stages_lora : 0);
            const uint32_t buf = local & 1, ause = local >> 1;
            if (!mbar_wait_bounded(&acc_empty[buf], (ause & 1) ^ 1, p.timeout_ns)) {
                record_timeout(p, abort_flag);
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + buf * Cfg::kAccCols;
            for (int ks = 0; ks < nst; ks++, it++) {
                const int s = it % S;
                const uint32_t use = it / S;
                if (!mbar_wait_bounded(&full_a[s], use & 1, p.timeout_ns) ||
                    (kFused && !mbar_wait_bounded(&full_b[s], use & 1, p.timeout_ns))) {
                    record_timeout(p, abort_flag);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(sA(s)), b_addr = smem_u32(sB(s));
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    const uint64_t bdesc = kBMn ? smem_desc_sw128(b_addr + 2048 * kk, 8192, 1024)
                                                : smem_desc_sw128(b_addr + 32 * kk, 16, 1024);
#pragma unroll
                    for (int m = 0; m < MT; m++) {
                        const uint32_t a_sub = a_addr + m * 16384;
                        const uint64_t adesc = p.a_mn ? smem_desc_sw128(a_sub + 2048 * kk, 8192, 1024)
                                                      : smem_desc_sw128(a_sub + 32 * kk, 16, 1024);
                        tc_mma_bf16(d_tmem + m * BN, adesc, bdesc, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc_commit(&empty[s]);
            }
            if (!ok) break;
            tc_commit(&acc_full[buf]);
        }
        if (*vabort) {
            // after an abort: wait (bounded) until the MMAs already issued finish
            tc_commit(drain);
            mbar_wait_bounded(drain, 0, p.drain_ns);
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------- epilogue ----------------
        const int q = warp & 3;
        uint32_t local = 0;
        for (int t = blockIdx.x; t < num_tiles && !*vabort; t += gridDim.x, local++) {
            int mt, nt, sp;
            decode(t, mt, nt, sp);
            const uint32_t buf = local & 1, ause = local >> 1;
            if (!mbar_wait_bounded(&acc_full[buf], ause & 1, p.timeout_ns)) {
                record_timeout(p, abort_flag);
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int m = 0; m < MT; m++) {
                const int row = mt * BM + m * 128 + 32 * q + lane;
                const bool row_ok = row < p.m_total;
#pragma unroll 1
                for (int c = 0; c < BN / 32; c++) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + buf * Cfg::kAccCols + m * BN + 32 * c, r);
                    tmem_ld_wait();
                    const int col0 = nt * BN + 32 * c;
                    if (!row_ok) continue;
                    if (kEpi == kEpiBf16) {
                        __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + (int64_t)row * p.out_ld + col0;
#pragma unroll
                        for (int g = 0; g < 4; g++) {
                            if (col0 + 8 * g >= p.n_total) break;
                            uint4 v;
                            v.x = nf4::pack16x2<F16>(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]));
                            v.y = nf4::pack16x2<F16>(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
                            v.z = nf4::pack16x2<F16>(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]));
                            v.w = nf4::pack16x2<F16>(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
                            *reinterpret_cast<uint4 *>(o + 8 * g) = v;
                        }
                    } else if (kEpi == kEpiDropBf16 || kEpi == kEpiDropF32) {
                        // out_ld % 32 == 0 and col0 % 32 == 0: the 32 mask bits of this
                        // chunk are one aligned 32-bit word; n_total % 32 == 0
                        if (col0 >= p.n_total) continue;
                        const int64_t flat = (int64_t)row * p.out_ld + col0;
                        const uint32_t bits = *reinterpret_cast<const uint32_t *>(p.drop_mask + flat / 8);
                        float v[32];
#pragma unroll
                        for (int g = 0; g < 8; g++) {
                            const float4 b4 = *reinterpret_cast<const float4 *>(p.drop_base + flat + 4 * g);
                            const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                            for (int i = 0; i < 4; i++) {
                                const int c = 4 * g + i;
                                const float t = ((bits >> c) & 1u) ? __fmul_rn(p.drop_scale, __uint_as_float(r[c])) : 0.0f;
                                v[c] = __fadd_rn(bb[i], t);
                            }
                        }
                        if (kEpi == kEpiDropBf16) {
                            __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + flat;
#pragma unroll
                            for (int g = 0; g < 4; g++) {
                                uint4 w;
                                w.x = nf4::pack16x2<F16>(v[8 * g + 0], v[8 * g + 1]);
                                w.y = nf4::pack16x2<F16>(v[8 * g + 2], v[8 * g + 3]);
                                w.z = nf4::pack16x2<F16>(v[8 * g + 4], v[8 * g + 5]);
                                w.w = nf4::pack16x2<F16>(v[8 * g + 6], v[8 * g + 7]);
                                *reinterpret_cast<uint4 *>(o + 8 * g) = w;
                            }
                        } else {
                            float *o = static_cast<float *>(p.out) + flat;
#pragma unroll
                            for (int g = 0; g < 8; g++)
                                *reinterpret_cast<float4 *>(o + 4 * g) = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                        }
                    } else {
                        float *o = static_cast<float *>(p.out) + (int64_t)sp * p.split_stride + (int64_t)row * p.out_ld + col0;
#pragma unroll
                        for (int g = 0; g < 8; g++) {
                            if (col0 + 4 * g >= p.n_total) break;
                            *reinterpret_cast<uint4 *>(o + 4 * g) = make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    } else if (kFused && warp >= 8) {
      if constexpr (kFused) {
        // ---------------- dequantization producer ----------------
        // A stage holds BN quantization blocks (64 consecutive k of one row of
        // W): forward stages are BN rows x 64 columns of W, input-gradient
        // stages are 64 rows x BN columns.  kTPB threads share a block, each
        // expanding 8 / kTPB words of 8 codes.  The block constant of the next
        // stage is fetched one stage ahead.
        constexpr int TPB = Cfg::kTPB;
        constexpr int WPT = 8 / TPB;   // words per thread
        const int dt = (warp - 8) * 32 + lane;
        const int blk = dt / TPB, part = dt % TPB;
        const float mu = *p.mean;
        uint32_t it = 0;
        for (int t = blockIdx.x; t < num_tiles && !*vabort; t += gridDim.x) {
            int mt, nt, sp, kb0, nmain;
            decode(t, mt, nt, sp);
            stages_of(sp, kb0, nmain);
            const int nst = nmain + (sp == 0 ? p.k_stages_lora : 0);
            auto block_of = [&](int ks, int64_t &n, int64_t &kb) {
                if (kBMode == kBNf4K) {
                    n = (int64_t)nt * BN + blk;
                    kb = kb0 + ks;
                } else {
                    n = (int64_t)(kb0 + ks) * 64 + (blk & 63);
                    kb = (int64_t)nt * (BN / 64) + (blk >> 6);
                }
            };
            auto load_raw = [&](int ks, uint8_t &e, float &c2) -> bool {
                int64_t n, kb;
                block_of(ks, n, kb);
                if (n >= p.wrows || kb >= p.kblocks) return false;
                const int64_t b = n * p.kblocks + kb;
                e = p.code2[b];
                c2 = p.c2[b >> 8];
                return true;
            };
            // block constants of the next kPre main stages, fetched ahead in a
            // register queue (q[0] = current stage)
            constexpr int kPre = 4;
            uint8_t qe[kPre];
            float qc2[kPre];
            bool qok[kPre];
#pragma unroll
            for (int i = 0; i < kPre; i++) qok[i] = i < nmain && load_raw(i, qe[i], qc2[i]);
            bool ok = true;
            for (int ks = 0; ks < nst; ks++, it++) {
                const int s = it % S;
                const uint32_t use = it / S;
                const float c1p = qok[0] ? block_scale(qe[0], qc2[0], mu) : 0.0f;
#pragma unroll
                for (int i = 0; i + 1 < kPre; i++) {
                    qe[i] = qe[i + 1];
                    qc2[i] = qc2[i + 1];
                    qok[i] = qok[i + 1];
                }
                qok[kPre - 1] = ks + kPre < nmain && load_raw(ks + kPre, qe[kPre - 1], qc2[kPre - 1]);
                if (!mbar_wait_bounded(&full_a[s], use & 1, p.timeout_ns)) {
                    record_timeout(p, abort_flag);
                    ok = false;
                    break;
                }
                if (ks < nmain) {
                    const uint8_t *pb = sP(s);
                    uint8_t *bb = sB(s);
                    uint32_t words[WPT];
                    int r;
                    uint8_t *dst;
                    // this thread's words part*WPT .. part*WPT+WPT-1 of the block's 8;
                    // 16-byte chunk h of the block holds words 4h..4h+3
                    auto load_words = [&](const uint8_t *row, auto chunk_pos) {
                        if constexpr (WPT == 8) {
#pragma unroll
                            for (int h = 0; h < 2; h++) {
                                const uint4 v = *reinterpret_cast<const uint4 *>(row + (chunk_pos(h) << 4));
                                words[4 * h + 0] = v.x; words[4 * h + 1] = v.y; words[4 * h + 2] = v.z; words[4 * h + 3] = v.w;
                            }
                        } else if constexpr (WPT == 4) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(row + (chunk_pos(part) << 4));
                            words[0] = v.x; words[1] = v.y; words[2] = v.z; words[3] = v.w;
                        } else {
                            static_assert(WPT == 2, "2, 4 or 8 words per thread");
                            const uint2 v = *reinterpret_cast<const uint2 *>(row + (chunk_pos(part >> 1) << 4) + ((part & 1) << 3));
                            words[0] = v.x; words[1] = v.y;
                        }
                    };
                    if (kBMode == kBNf4K) {
                        // packed tile [BN rows][32 B], 32-byte swizzle: chunk h at h ^ ((row >> 2) & 1)
                        r = blk;
                        const int sw = (r >> 2) & 1;
                        load_words(pb + r * 32, [&](int h) { return h ^ sw; });
                        dst = bb + r * 128;
                    } else {
                        // packed tile [64 rows][BN/2 B]: 128-byte swizzle (BN = 256) or
                        // 64-byte swizzle (BN = 128) of its 16-byte chunks
                        r = blk & 63;
                        const int c = blk >> 6;
                        load_words(pb + r * (BN / 2), [&](int h) {
                            const int chunk = 2 * c + h;
                            return BN == 256 ? (chunk ^ (r & 7)) : (chunk ^ ((r >> 1) & 3));
                        });
                        dst = bb + c * 8192 + r * 128;
                    }
                    const int dst_chunk0 = part * WPT;
#pragma unroll
                    for (int j = 0; j < WPT; j++)
                        *reinterpret_cast<uint4 *>(dst + (((dst_chunk0 + j) ^ (r & 7)) << 4)) = expand8<F16>(words[j], lut, c1p);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                const bool skip = p.stall_inject && blockIdx.x == 0 && warp == 8 && it == 0;
                if (lane == 0 && !skip) mbar_arrive(&full_b[s]);
            }
            if (!ok) break;
        }
      }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace qlora
