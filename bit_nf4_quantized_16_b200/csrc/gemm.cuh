// Warp-specialized tcgen05 GEMM for sm_100a, with an optional on-chip NF4
// dequantization producer for the B operand.
//
// D[128 x BN] tiles accumulate in tensor memory (fp32); operands are staged
// in shared memory in the 128-byte-swizzled canonical layouts described in
// sm100.cuh.  Roles (one CTA per SM, persistent over output tiles):
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
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "sm100.cuh"

namespace qlora {

enum BMode : int { kBTmaK = 0, kBTmaMN = 1, kBNf4K = 2, kBNf4MN = 3 };
enum Epi : int { kEpiBf16 = 0, kEpiF32 = 1 };

struct GemmParams {
    CUtensorMap tm_a;    // main A operand
    CUtensorMap tm_b;    // main B operand, or packed NF4 codes (uint8 [N][K/2])
    CUtensorMap tm_a2;   // LoRA A operand (K-major)
    CUtensorMap tm_b2;   // LoRA B operand (same majorness as the main B)
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
    // output (row-major, leading dimension out_ld elements)
    void *out;
    int64_t out_ld;
    int64_t split_stride;  // elements between split planes (partial outputs)
    int m_total, n_total;
    int *err;            // device error word
    uint64_t timeout_ns;
};

template <int BN, int kBMode>
struct GemmCfg {
    static constexpr int kStages = (kBMode >= kBNf4K) ? 4 : (BN >= 256 ? 4 : 6);
    static constexpr bool kFused = kBMode >= kBNf4K;
    static constexpr int kDeqWarps = kFused ? 8 : 0;
    static constexpr int kThreads = 256 + 32 * kDeqWarps;
    static constexpr uint32_t kABytes = 128 * 64 * 2;
    static constexpr uint32_t kBBytes = BN * 64 * 2;
    static constexpr uint32_t kPBytes = kFused ? BN * 32 : 0;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes + kPBytes;
    static constexpr uint32_t kBarOff = kStages * kStageBytes;
    static constexpr uint32_t kSmemBytes = kBarOff + 512 + 1024;  // barriers etc. + alignment slack
    static constexpr uint32_t kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;
};

namespace gemm_detail {

__device__ __forceinline__ float e4m3_to_float(uint8_t code)
{
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
    return __half2float(__half(h));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// 8 consecutive codes (one 32-bit word, element 0 in bits 0-3) -> 8 bf16 in a
// 16-byte vector: w = bf16(RN32(q[code] * c1p)).
__device__ __forceinline__ uint4 expand8(uint32_t word, const float *lut, float c1p)
{
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float lo = __fmul_rn(lut[(word >> (8 * i)) & 15u], c1p);
        float hi = __fmul_rn(lut[(word >> (8 * i + 4)) & 15u], c1p);
        o[i] = pack_bf16x2(lo, hi);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ float block_scale(const GemmParams &p, int64_t n, int64_t kb, float mu)
{
    if (n >= p.wrows || kb >= p.kblocks) return 0.0f;
    int64_t b = n * p.kblocks + kb;
    return __fmaf_rn(e4m3_to_float(p.code2[b]), p.c2[b >> 8], mu);
}

__device__ __forceinline__ void record_timeout(const GemmParams &p, int *abort_flag)
{
    atomicExch(p.err, 1);
    *reinterpret_cast<volatile int *>(abort_flag) = 1;
}

}  // namespace gemm_detail

template <int BN, int kBMode, int kEpi>
__global__ void __launch_bounds__(GemmCfg<BN, kBMode>::kThreads, 1)
    qgemm_kernel(const __grid_constant__ GemmParams p)
{
    using Cfg = GemmCfg<BN, kBMode>;
    using namespace sm100;
    using namespace gemm_detail;
    constexpr int S = Cfg::kStages;
    constexpr bool kFused = Cfg::kFused;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_a = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
    uint64_t *full_b = full_a + S;
    uint64_t *empty = full_b + S;
    uint64_t *acc_full = empty + S;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    float *lut = reinterpret_cast<float *>(tmem_slot + 4);

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
                mbar_wait_bounded(&full_a[j % S], (j / S) & 1, p.timeout_ns);
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
                const int m0 = mt * 128, n0 = nt * BN;
                if (ks < nmain) {
                    const int k0 = (kb0 + ks) * 64;
                    mbar_arrive_expect_tx(&full_a[s], Cfg::kABytes + (kFused ? Cfg::kPBytes : Cfg::kBBytes));
                    if (!p.a_mn) {
                        tma_load_2d(sA(s), &p.tm_a, &full_a[s], k0, m0);
                    } else {
                        tma_load_2d(sA(s), &p.tm_a, &full_a[s], m0, k0);
                        tma_load_2d(sA(s) + 8192, &p.tm_a, &full_a[s], m0 + 64, k0);
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
                    tma_load_2d(sA(s), &p.tm_a2, &full_a[s], r0, m0);
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
        const uint32_t idesc = idesc_bf16_f32(128, BN, p.a_mn, kBMn ? 1 : 0);
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
            const uint32_t d_tmem = tmem_base + buf * BN;
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
                    const uint64_t adesc = p.a_mn ? smem_desc_sw128(a_addr + 2048 * kk, 8192, 1024)
                                                  : smem_desc_sw128(a_addr + 32 * kk, 16, 1024);
                    const uint64_t bdesc = kBMn ? smem_desc_sw128(b_addr + 2048 * kk, 8192, 1024)
                                                : smem_desc_sw128(b_addr + 32 * kk, 16, 1024);
                    tc_mma_bf16(d_tmem, adesc, bdesc, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
            }
            if (!ok) break;
            tc_commit(&acc_full[buf]);
        }
        if (*vabort) {
            // after an abort: wait (bounded) until the MMAs already issued finish
            tc_commit(drain);
            mbar_wait_bounded(drain, 0, p.timeout_ns);
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
            const int row = mt * 128 + 32 * q + lane;
            const bool row_ok = row < p.m_total;
#pragma unroll 1
            for (int c = 0; c < BN / 32; c++) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + buf * BN + 32 * c, r);
                tmem_ld_wait();
                const int col0 = nt * BN + 32 * c;
                if (!row_ok) continue;
                if (kEpi == kEpiBf16) {
                    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + (int64_t)row * p.out_ld + col0;
#pragma unroll
                    for (int g = 0; g < 4; g++) {
                        if (col0 + 8 * g >= p.n_total) break;
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]));
                        v.y = pack_bf16x2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
                        v.z = pack_bf16x2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]));
                        v.w = pack_bf16x2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
                        *reinterpret_cast<uint4 *>(o + 8 * g) = v;
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
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    } else if (kFused && warp >= 8) {
      if constexpr (kFused) {
        // ---------------- dequantization producer ----------------
        // One quantization block (64 consecutive k of one row of W) per thread
        // per stage: forward stages hold BN rows x 64 columns of W, input-
        // gradient stages hold 64 rows x BN columns (BN / 64 blocks per row).
        // The block constant of the next stage is fetched one stage ahead.
        const int dt = (warp - 8) * 32 + lane;
        static_assert(32 * Cfg::kDeqWarps == BN, "one block per thread per stage");
        const float mu = *p.mean;
        uint32_t it = 0;
        for (int t = blockIdx.x; t < num_tiles && !*vabort; t += gridDim.x) {
            int mt, nt, sp, kb0, nmain;
            decode(t, mt, nt, sp);
            stages_of(sp, kb0, nmain);
            const int nst = nmain + (sp == 0 ? p.k_stages_lora : 0);
            // block (row, column block) of this thread at main stage ks
            auto block_of = [&](int ks, int64_t &n, int64_t &kb) {
                if (kBMode == kBNf4K) {
                    n = (int64_t)nt * BN + dt;
                    kb = kb0 + ks;
                } else {
                    n = (int64_t)(kb0 + ks) * 64 + (dt & 63);
                    kb = (int64_t)nt * (BN / 64) + (dt >> 6);
                }
            };
            int64_t n, kb;
            block_of(0, n, kb);
            float c1p = nmain > 0 ? block_scale(p, n, kb, mu) : 0.0f;
            bool ok = true;
            for (int ks = 0; ks < nst; ks++, it++) {
                const int s = it % S;
                const uint32_t use = it / S;
                // prefetch the next stage's block constant (raw bytes only)
                uint8_t e_next = 0;
                float c2_next = 0.0f;
                bool have_next = false;
                if (ks + 1 < nmain) {
                    int64_t n1, kb1;
                    block_of(ks + 1, n1, kb1);
                    if (n1 < p.wrows && kb1 < p.kblocks) {
                        const int64_t b = n1 * p.kblocks + kb1;
                        e_next = p.code2[b];
                        c2_next = p.c2[b >> 8];
                        have_next = true;
                    }
                }
                if (!mbar_wait_bounded(&full_a[s], use & 1, p.timeout_ns)) {
                    record_timeout(p, abort_flag);
                    ok = false;
                    break;
                }
                if (ks < nmain) {
                    const uint8_t *pb = sP(s);
                    uint8_t *bb = sB(s);
                    if (kBMode == kBNf4K) {
                        const int nl = dt;
                        const int sw = (nl >> 2) & 1;   // 32-byte swizzle of the packed tile
                        const uint4 lo = *reinterpret_cast<const uint4 *>(pb + nl * 32 + (sw << 4));
                        const uint4 hi = *reinterpret_cast<const uint4 *>(pb + nl * 32 + ((sw ^ 1) << 4));
                        const uint32_t words[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                        uint8_t *dst = bb + nl * 128;
#pragma unroll
                        for (int j = 0; j < 8; j++)
                            *reinterpret_cast<uint4 *>(dst + ((j ^ (nl & 7)) << 4)) = expand8(words[j], lut, c1p);
                    } else {
                        const int r = dt & 63, c = dt >> 6;
                        const uint4 lo = *reinterpret_cast<const uint4 *>(pb + r * 128 + (((2 * c) ^ (r & 7)) << 4));
                        const uint4 hi = *reinterpret_cast<const uint4 *>(pb + r * 128 + (((2 * c + 1) ^ (r & 7)) << 4));
                        const uint32_t words[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                        uint8_t *dst = bb + c * 8192 + r * 128;
#pragma unroll
                        for (int j = 0; j < 8; j++)
                            *reinterpret_cast<uint4 *>(dst + ((j ^ (r & 7)) << 4)) = expand8(words[j], lut, c1p);
                    }
                    fence_proxy_async_smem();
                    c1p = have_next ? __fmaf_rn(e4m3_to_float(e_next), c2_next, mu) : 0.0f;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_b[s]);
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
