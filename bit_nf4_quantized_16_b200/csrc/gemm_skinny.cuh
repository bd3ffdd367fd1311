// Skinny products of the QLoRA linear on sm_100a: the rank-r factors and the
// adapter gradients, each a tcgen05 GEMM whose contraction is split over the
// CTAs of a thread-block cluster and reduced through distributed shared
// memory, fused with the product's elementwise finish.
//
//   H  = s X A^T     [M, r]    contraction over K   -> hi/lo bf16 H2 (+ fp32 H)
//   G  = s dY B      [M, r]    contraction over N   -> hi/lo bf16 G2 (+ a saved
//                                                       fp32 H split into H2)
//   dA = X^T [G_hi | G_lo]     contraction over M   -> dA [r, K] (hi + lo)
//   dB = dY^T [H_hi | H_lo]    contraction over M   -> dB [N, r] (hi + lo)
// (mbrenndoerfer.com QLoRA essay, "Low-Rank Adaptation (LoRA)": the adapters
// A [r, d] and B [d, r]; "QLoRA: Efficient Finetuning of Quantized LLMs",
// abstract: gradients reach only the adapters.)
//
// One output tile of 128 rows x BN columns per cluster; the cluster's CTAs
// take consecutive ranges of the contraction.  Each CTA stages its fp32
// partial tile in its own shared memory (the operand ring, idle by then);
// after a cluster barrier, CTA q sums rows [q*128/C, (q+1)*128/C) of all C
// partials in rank order (deterministic), applies the finish and writes the
// result; a second barrier keeps every partial alive until it has been read.
// No partial sums go through global memory and no finalize kernel follows.
//
// Two independent jobs may share a launch (dA and dB): clusters
// [0, clusters0) take job 0, the rest job 1.
//
// Roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner, warps 4..7
// move the accumulator from TMEM to the staged partial; all 256 threads
// reduce.  Every mbarrier wait is bounded; a timeout is recorded in the
// device error word and the CTA winds down (the cluster barriers are still
// reached by every thread).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100.cuh"
#include "debug.cuh"

namespace qlora {

enum SkinnyFin : int {
    kFinLowRank = 0,   // v = scale * sum -> hi/lo bf16 columns (+ fp32 copy, + aux hi/lo split)
    kFinWgradT = 1,    // v = sum(hi half) + sum(lo half) -> out[j][row] (transposed)
    kFinWgrad = 2      // the same -> out[row][j]
};

struct SkinnyJob {
    CUtensorMap tm_a;          // A operand: [rows][contraction] K-major, or [contraction][rows] MN-major
    CUtensorMap tm_b;          // B operand: [BN cols][contraction] K-major, or [contraction][cols] MN-major
    int m_tiles;               // 128-row output tiles
    int k_total;               // 64-deep contraction steps
    int fin;                   // SkinnyFin
    int m_total;               // valid output rows
    float scale;               // kFinLowRank
    int r, r_pad;              // adapter rank and its 64-multiple
    __nv_bfloat16 *hl_out;     // kFinLowRank: [m_total][2 r_pad], hi of column c at 128(c/64) + c%64, lo 64 further
    float *f32_out;            // kFinLowRank: optional [m_total][r]; kFinWgrad(T): the gradient
    int64_t out_ld;            // kFinWgrad(T): leading dimension of f32_out
    const float *aux_in;       // kFinLowRank: optional [m_total][r] split into aux_out (same layout as hl_out)
    __nv_bfloat16 *aux_out;
};

struct SkinnyParams {
    SkinnyJob job[2];
    int clusters0;             // clusters (output tiles) of job 0
    int *err;                  // device error word
    uint64_t timeout_ns;       // limit of every pipeline wait
    uint64_t drain_ns;         // limit of the waits for work in flight after an abort
    int wait_at_end;           // 1: nothing this kernel reads was written by the kernel launched just
                               // before it, so the dependency wait moves to the end (the launch can
                               // fill SMs that kernel leaves idle in its last wave)
};

template <int BN, int A_MN, int B_MN>
struct SkinnyCfg {
    static constexpr int kThreads = 256;
    static constexpr uint32_t kABytes = 128 * 64 * 2;
    static constexpr uint32_t kBBytes = BN * 64 * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = 6;
    static constexpr uint32_t kRingBytes = kStages * kStageBytes;
    static constexpr uint32_t kPartLd = BN * 4 + 16;        // bytes per staged row (padding spreads banks)
    static constexpr uint32_t kPartBytes = 128 * kPartLd;
    static constexpr uint32_t kBarOff = kRingBytes;
    static constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
    static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
    static_assert(kPartBytes <= kRingBytes, "the staged partial reuses the operand ring");
    static_assert(kSmemBytes <= 232448, "shared memory per block");
    static_assert(BN == 64 || BN == 128, "tile width");
};

namespace skinny_detail {

// Bits of v rounded to the 16-bit compute type, and that value back in fp32.
template <bool F16>
__device__ __forceinline__ uint32_t bits16(float v)
{
    if constexpr (F16)
        return (uint32_t)__half_as_ushort(__float2half_rn(v));
    else
        return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}
template <bool F16>
__device__ __forceinline__ float from16(uint32_t b)
{
    if constexpr (F16)
        return __half2float(__ushort_as_half((unsigned short)b));
    else
        return __uint_as_float(b << 16);
}

// hi = t16(v), lo = t16(v - hi) (t16: the 16-bit compute type) of columns
// col..col+3 of row `row` into the chunked hi/lo layout [rows][2 r_pad].
template <bool F16>
__device__ __forceinline__ void store_hi_lo4(__nv_bfloat16 *dst, int64_t row, int r_pad, int col, float4 v)
{
    const float vv[4] = {v.x, v.y, v.z, v.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        hi[i] = bits16<F16>(vv[i]);
        lo[i] = bits16<F16>(__fsub_rn(vv[i], from16<F16>(hi[i])));
    }
    __nv_bfloat16 *d = dst + row * 2 * r_pad + 128 * (col >> 6) + (col & 63);
    *reinterpret_cast<uint2 *>(d) = make_uint2(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16));
    *reinterpret_cast<uint2 *>(d + 64) = make_uint2(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16));
}

__device__ __forceinline__ float4 add4(float4 a, float4 b)
{
    return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
}

}  // namespace skinny_detail

template <int BN, int A_MN, int B_MN, bool F16 = false>
__global__ void __launch_bounds__(256, 1) qgemm_skinny_kernel(const __grid_constant__ SkinnyParams p)
{
    using Cfg = SkinnyCfg<BN, A_MN, B_MN>;
    using namespace sm100;
    using namespace skinny_detail;
    constexpr int S = Cfg::kStages;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
    uint64_t *empty = full + S;
    uint64_t *acc_full = empty + S;
    uint64_t *drain = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t csize = cluster_nctarank(), rank = cluster_ctarank();
    const int cid = (int)(blockIdx.x / csize);
    const bool second = cid >= p.clusters0;
    const SkinnyJob &J = second ? p.job[1] : p.job[0];
    const int tile = second ? cid - p.clusters0 : cid;
    const int mt = tile % J.m_tiles, nt = tile / J.m_tiles;
    // this CTA's range of the contraction
    const int per = (J.k_total + (int)csize - 1) / (int)csize;
    const int k_begin = (int)rank * per;
    int n_k = J.k_total - k_begin;
    if (n_k > per) n_k = per;
    if (n_k < 0) n_k = 0;
    auto sA = [&](int s) { return smem + s * Cfg::kStageBytes; };
    auto sB = [&](int s) { return smem + s * Cfg::kStageBytes + Cfg::kABytes; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&J.tm_a);
        tma_prefetch_desc(&J.tm_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (!p.wait_at_end) pdl_wait();   // the inputs may come from the kernel before this one
    pdl_trigger();
    const uint32_t tmem_base = *tmem_slot;
    volatile int *vabort = abort_flag;
    auto record_timeout = [&]() {
        atomicExch(p.err, 1);
        *reinterpret_cast<volatile int *>(abort_flag) = 1;
    };

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        const int m0 = mt * 128, n0 = nt * BN;
        int ks = 0;
        for (; ks < n_k; ks++) {
            const int s = ks % S;
            const uint32_t use = (uint32_t)(ks / S);
            if (!mbar_wait_bounded(&empty[s], (use & 1) ^ 1, p.timeout_ns)) {
                record_timeout();
                break;
            }
            if (*vabort) break;
            const int k0 = (k_begin + ks) * 64;
            mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
            if (A_MN) {
#pragma unroll
                for (int j = 0; j < 2; j++) tma_load_2d(sA(s) + 8192 * j, &J.tm_a, &full[s], m0 + 64 * j, k0);
            } else {
                tma_load_2d(sA(s), &J.tm_a, &full[s], k0, m0);
            }
            if (B_MN) {
#pragma unroll
                for (int j = 0; j < BN / 64; j++) tma_load_2d(sB(s) + 8192 * j, &J.tm_b, &full[s], n0 + 64 * j, k0);
            } else {
                tma_load_2d(sB(s), &J.tm_b, &full[s], k0, n0);
            }
        }
        if (*vabort) {
            // wait (bounded) for the copies still in flight before the ring is reused
            for (int j = ks > S ? ks - S : 0; j < ks; j++) mbar_wait_bounded(&full[j % S], (j / S) & 1, p.drain_ns);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        const uint32_t idesc = idesc_bf16_f32(128, BN, A_MN, B_MN, F16);
        bool ok = true;
        for (int ks = 0; ks < n_k; ks++) {
            const int s = ks % S;
            const uint32_t use = (uint32_t)(ks / S);
            if (!mbar_wait_bounded(&full[s], use & 1, p.timeout_ns)) {
                record_timeout();
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA(s)), b_addr = smem_u32(sB(s));
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                const uint64_t adesc = A_MN ? smem_desc_sw128(a_addr + 2048 * kk, 8192, 1024)
                                            : smem_desc_sw128(a_addr + 32 * kk, 16, 1024);
                const uint64_t bdesc = B_MN ? smem_desc_sw128(b_addr + 2048 * kk, 8192, 1024)
                                            : smem_desc_sw128(b_addr + 32 * kk, 16, 1024);
                tc_mma_bf16(tmem_base, adesc, bdesc, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&empty[s]);
        }
        if (ok) tc_commit(acc_full);
        if (*vabort) {
            // wait (bounded) until the MMAs already issued have finished
            tc_commit(drain);
            mbar_wait_bounded(drain, 0, p.drain_ns);
        }
    } else if (warp >= 4) {
        // ---------------- accumulator -> staged fp32 partial ----------------
        const int q = warp - 4;
        bool got = mbar_wait_bounded(acc_full, 0, p.timeout_ns);
        if (!got) record_timeout();
        tc_fence_after();
        const bool zero = !got || n_k == 0;   // no contribution from this CTA
        uint8_t *prow = smem + (32 * q + lane) * Cfg::kPartLd;
#pragma unroll 1
        for (int c = 0; c < BN / 32; c++) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + 32 * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < 8; g++) {
                const uint4 v = zero ? make_uint4(0, 0, 0, 0)
                                     : make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
                *reinterpret_cast<uint4 *>(prow + 128 * c + 16 * g) = v;
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    cluster_sync();   // every CTA's partial is complete and visible to the cluster

    // ---------------- reduction over the cluster + finish ----------------
    {
        const int rows_per = 128 / (int)csize;
        const int row0 = (int)rank * rows_per;
        const bool wgrad = J.fin != kFinLowRank;
        const int ncol4 = wgrad ? BN / 8 : BN / 4;   // wgrad: hi half, the lo half is added in
        const uint32_t part0 = smem_u32(smem);
        for (int u = threadIdx.x; u < rows_per * ncol4; u += Cfg::kThreads) {
            const int lr = row0 + u % rows_per;
            const int c4 = u / rows_per;
            const uint32_t off = (uint32_t)lr * Cfg::kPartLd + 16u * (uint32_t)c4;
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (uint32_t qr = 0; qr < csize; qr++) acc = add4(acc, ld_dsmem_f4(mapa_shared(part0 + off, qr)));
            if (wgrad) {
                float4 lo = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                for (uint32_t qr = 0; qr < csize; qr++)
                    lo = add4(lo, ld_dsmem_f4(mapa_shared(part0 + off + 4u * (BN / 2), qr)));
                acc = add4(acc, lo);
            }
            const int64_t grow = (int64_t)mt * 128 + lr;
            if (grow >= J.m_total || !QLORA_IN(grow, J.m_total)) continue;
            if (!wgrad) {
                const int col = 4 * c4;
                const bool in = col < J.r;   // r % 8 == 0: four columns are all in or all out
                float4 v = make_float4(__fmul_rn(J.scale, acc.x), __fmul_rn(J.scale, acc.y),
                                       __fmul_rn(J.scale, acc.z), __fmul_rn(J.scale, acc.w));
                if (!in) v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (!QLORA_IN(col + 3, J.r_pad)) continue;
                if (J.f32_out && in) *reinterpret_cast<float4 *>(J.f32_out + grow * J.r + col) = v;
                store_hi_lo4<F16>(J.hl_out, grow, J.r_pad, col, v);
                if (J.aux_in) {
                    float4 h = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (in) h = *reinterpret_cast<const float4 *>(J.aux_in + grow * J.r + col);
                    store_hi_lo4<F16>(J.aux_out, grow, J.r_pad, col, h);
                }
            } else {
                const int j = 64 * nt + 4 * c4;
                if (j >= J.r) continue;
                if (!QLORA_IN((int64_t)(j + 3) * (J.fin == kFinWgradT ? J.out_ld : 1) +
                                  grow * (J.fin == kFinWgradT ? 1 : J.out_ld),
                              (int64_t)(J.fin == kFinWgradT ? J.r : J.m_total) * J.out_ld))
                    continue;
                if (J.fin == kFinWgradT) {
                    J.f32_out[(int64_t)(j + 0) * J.out_ld + grow] = acc.x;
                    J.f32_out[(int64_t)(j + 1) * J.out_ld + grow] = acc.y;
                    J.f32_out[(int64_t)(j + 2) * J.out_ld + grow] = acc.z;
                    J.f32_out[(int64_t)(j + 3) * J.out_ld + grow] = acc.w;
                } else {
                    *reinterpret_cast<float4 *>(J.f32_out + grow * J.out_ld + j) = acc;
                }
            }
        }
    }

    cluster_sync();   // every partial has been read
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
    // launched without an entry wait: complete only after the kernel before
    // this one, so that later kernels that wait on this one also wait on it
    if (p.wait_at_end) pdl_wait();
}

}  // namespace qlora
