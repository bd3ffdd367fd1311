// QLoRA linear layer on sm_100a: forward Y = X W'^T + s (X A^T) B^T and the
// backward pass dX, dA, dB (no dW: the quantized weight is frozen).
//
// Sources: mbrenndoerfer.com QLoRA essay, section "Low-Rank Adaptation
// (LoRA)" (x_out = (W_q + BA) x_in, A is r x d, B is d x r); "QLoRA: Efficient
// Finetuning of Quantized LLMs", section "Method" (dequantize to BFloat16 and
// multiply in 16-bit) and abstract (gradients flow through the frozen 4-bit
// weight into the adapters).
//
// Launch sequence (all on the caller's stream):
//   forward : H-partials (tcgen05, split-K) -> finalize H (x s, hi/lo bf16)
//             -> fused dequant-GEMM with the LoRA up-projection as extra K steps
//   backward: H (recomputed, or split from the saved fp32 H) -> G-partials ->
//             finalize G -> fused transposed dequant-GEMM for dX (+ G A)
//             -> dA partials (G^T X) -> dB partials (dY^T H) -> finalize both
// H and G are carried as hi + lo bf16 pairs (hi = bf16(v), lo = bf16(v - hi)):
// the weight gradients contract over all M tokens and need about 16 bits of
// each factor to stay at the level of fp32 accumulation; the fused GEMMs use
// only the hi half.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <algorithm>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "decode.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"

namespace qlora {
namespace {

constexpr uint64_t kTimeoutNs = 2000000000ull;   // bounded waits give up after 2 s

qlora_status map_bf16(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t ld,
                      uint32_t box_inner, uint32_t box_rows)
{
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, rows, ld * 2, box_inner, box_rows,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

// ---- launches ------------------------------------------------------------------------

// ---- GEMM launch ------------------------------------------------------------------

// Wait limits, and the failure-detection test hook when it is armed for `kind`.
void set_limits(GemmParams &p, int kind)
{
    p.timeout_ns = kTimeoutNs;
    p.drain_ns = kTimeoutNs;
    p.stall_inject = take_stall_injection(kind, &p.timeout_ns) ? 1 : 0;
}

template <int BN, int kBMode, int kEpi, int MT = 1>
qlora_status launch_gemm(GemmParams &p, const DeviceInfo &dev, cudaStream_t s, int kind)
{
    using Cfg = GemmCfg<BN, kBMode, MT>;
    static PerDeviceOnce attr;
    auto kern = qgemm_kernel<BN, kBMode, kEpi, MT>;
    QLORA_TRY(attr.run(dev.device, [&]() -> qlora_status {
        QLORA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
        return QLORA_OK;
    }));
    p.err = device_error_word();
    if (!p.err) return QLORA_ERR_CUDA;
    set_limits(p, kind);
    const int tiles = p.m_tiles * p.n_tiles * p.splits;
    const int grid = tiles < dev.sms ? tiles : dev.sms;
    {
        LaunchScope ls(kind, s);
        QLORA_CUDA_TRY(launch_pdl(kern, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmemBytes, s, p));
    }
    return launch_status();
}

// Fused dequant-GEMM on CTA pairs: p.m_tiles / p.n_tiles count pair tiles
// (2 * 128 * MT tokens x 256 features); one cluster of two CTAs per tile,
// persistent over tiles, at most as many clusters as can be resident at once.
template <int kBMode, int kEpi, int MT>
qlora_status launch_gemm_pair(GemmParams &p, const DeviceInfo &dev, cudaStream_t s, int kind)
{
    using Cfg = PairCfg<kBMode, MT>;
    static PerDeviceOnce setup;
    static int max_clusters[kMaxDevices] = {};
    auto kern = qgemm_pair_kernel<kBMode, kEpi, MT>;
    QLORA_TRY(setup.run(dev.device, [&]() -> qlora_status {
        QLORA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(2 * (dev.sms / 2));
        cfg.blockDim = dim3(Cfg::kThreads);
        cfg.dynamicSmemBytes = Cfg::kSmemBytes;
        int n = 0;
        QLORA_CUDA_TRY(cudaOccupancyMaxActiveClusters(&n, kern, &cfg));
        if (n < 1) return QLORA_ERR_CUDA;
        max_clusters[dev.device] = n;
        return QLORA_OK;
    }));
    p.err = device_error_word();
    if (!p.err) return QLORA_ERR_CUDA;
    set_limits(p, kind);
    p.splits = 1;
    const int tiles = p.m_tiles * p.n_tiles;
    const int clusters = tiles < max_clusters[dev.device] ? tiles : max_clusters[dev.device];
    {
        LaunchScope ls(kind, s);
        QLORA_CUDA_TRY(launch_pdl(kern, dim3(2 * clusters), dim3(Cfg::kThreads), Cfg::kSmemBytes, s, p));
    }
    return launch_status();
}

// number of splits of a contraction of `total` 64-deep steps over `tiles`
// output tiles: as many as fit in one wave of the GPU (tiles * splits <= sms),
// each with at least `min_per_split` steps; every split non-empty
void choose_splits(int tiles, int total, int sms, int min_per_split, int *splits, int *per)
{
    int sp = sms / (tiles > 0 ? tiles : 1);
    int cap = total / min_per_split;
    if (cap < 1) cap = 1;
    if (sp > cap) sp = cap;
    if (sp < 1) sp = 1;
    int pr = (total + sp - 1) / sp;
    *per = pr;
    *splits = (total + pr - 1) / pr;
}

int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }
int pad64(int v) { return (v + 63) / 64 * 64; }
int elementwise_grid(int64_t n) { return (int)((n + 255) / 256); }

// ---- finalize kernels (grid-wide, one thread per 4 outputs) ---------------------------

// Sum of the split partials at (row, col..col+3), splits added in order.
__device__ __forceinline__ float4 split_sum4(const float *part, int splits, int64_t split_stride, int64_t ld,
                                             int64_t row, int64_t col)
{
    const float *src = part + row * ld + col;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    // four splits' loads are issued before their in-order additions (issue is
    // in order, so an addition waiting on a load would hold back the next load)
    for (int sp0 = 0; sp0 < splits; sp0 += 4) {
        float4 v[4];
#pragma unroll
        for (int i = 0; i < 4; i++)
            v[i] = sp0 + i < splits ? __ldcg(reinterpret_cast<const float4 *>(src + (sp0 + i) * split_stride))
                                    : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            if (sp0 + i >= splits) break;
            acc.x = __fadd_rn(acc.x, v[i].x);
            acc.y = __fadd_rn(acc.y, v[i].y);
            acc.z = __fadd_rn(acc.z, v[i].z);
            acc.w = __fadd_rn(acc.w, v[i].w);
        }
    }
    return acc;
}

__device__ __forceinline__ uint32_t bf16_bits(float v) { return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// hi = bf16(v), lo = bf16(v - hi) of 4 consecutive columns col..col+3 into the
// chunked hi/lo layout: [M][2*r_pad], hi of column c at 128*(c/64) + c%64, lo 64 further.
__device__ __forceinline__ void store_hi_lo4(__nv_bfloat16 *dst, int64_t row, int r_pad, int col, float4 v)
{
    const float vv[4] = {v.x, v.y, v.z, v.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        hi[i] = bf16_bits(vv[i]);
        lo[i] = bf16_bits(__fsub_rn(vv[i], __uint_as_float(hi[i] << 16)));
    }
    __nv_bfloat16 *d = dst + row * 2 * r_pad + 128 * (col >> 6) + (col & 63);
    *reinterpret_cast<uint2 *>(d) = make_uint2(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16));
    *reinterpret_cast<uint2 *>(d + 64) = make_uint2(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16));
}

// v = scale * sum over splits of part[.][m][j]  ->  hi/lo chunked buffer (padding
// columns j >= r set to zero), optionally fp32 v [M][r]; optionally also the
// hi/lo split of aux_in [M][r] into aux_out.
__global__ void finalize_lowrank_kernel(const float *part, int splits, int64_t split_stride, int64_t M, int r,
                                        int r_pad, float scale, __nv_bfloat16 *out, float *out_f32,
                                        const float *aux_in, __nv_bfloat16 *aux_out)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int per_row = r_pad / 4;
    if (i >= M * per_row) return;
    const int64_t m = i / per_row;
    const int col = 4 * (int)(i % per_row);
    const bool in = col < r;   // r % 8 == 0: 4 columns are all in or all out
    float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (in) {
        v = split_sum4(part, splits, split_stride, r_pad, m, col);
        v = make_float4(__fmul_rn(scale, v.x), __fmul_rn(scale, v.y), __fmul_rn(scale, v.z), __fmul_rn(scale, v.w));
        if (out_f32) *reinterpret_cast<float4 *>(out_f32 + m * r + col) = v;
    }
    store_hi_lo4(out, m, r_pad, col, v);
    if (aux_in) {
        float4 h = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (in) h = *reinterpret_cast<const float4 *>(aux_in + m * r + col);
        store_hi_lo4(aux_out, m, r_pad, col, h);
    }
}

// Weight gradients from the partial products of the hi and lo halves, two jobs
// in one launch: job 0 = dA (rows k of X^T [G_hi|G_lo], stored transposed into
// dA[j][k]), job 1 = dB (rows n of dY^T [H_hi|H_lo], stored as dB[n][j]).
struct WgradJob {
    const float *part;
    int splits;
    int64_t split_stride;
    int64_t rows;
    float *out;
    int64_t out_ld;
    int transposed;
};

__global__ void finalize_wgrad_kernel(WgradJob j0, WgradJob j1, int64_t n0, int r, int r_pad)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int per_row = r / 4;
    const WgradJob &J = i < n0 ? j0 : j1;
    if (i >= n0) i -= n0;
    if (i >= J.rows * per_row) return;
    const int64_t row = i / per_row;
    const int j = 4 * (int)(i % per_row);
    const int64_t ld = 2 * r_pad;
    const int64_t chunk = 128 * (j >> 6) + (j & 63);
    const float4 hi = split_sum4(J.part, J.splits, J.split_stride, ld, row, chunk);
    const float4 lo = split_sum4(J.part, J.splits, J.split_stride, ld, row, chunk + 64);
    const float4 v = make_float4(__fadd_rn(hi.x, lo.x), __fadd_rn(hi.y, lo.y), __fadd_rn(hi.z, lo.z), __fadd_rn(hi.w, lo.w));
    if (J.transposed) {
        J.out[(int64_t)(j + 0) * J.out_ld + row] = v.x;
        J.out[(int64_t)(j + 1) * J.out_ld + row] = v.y;
        J.out[(int64_t)(j + 2) * J.out_ld + row] = v.z;
        J.out[(int64_t)(j + 3) * J.out_ld + row] = v.w;
    } else {
        *reinterpret_cast<float4 *>(J.out + row * J.out_ld + j) = v;
    }
}

// ---- problem plan -------------------------------------------------------------------

// H2 / G2 buffers: [M][2*r_pad] bf16, 64-column chunks alternating hi | lo
// (hi of columns 64c..64c+63 at 128c, their lo at 128c+64).
struct Plan {
    int64_t M, N, K;
    int r, r_pad;
    int h_splits, h_per;          // H = s X A^T : M tiles, split over K
    int g_splits, g_per;          // G = s dY B  : M tiles, split over N
    int da_splits, da_per;        // dA^T = X^T [G_hi|G_lo] : K tiles x chunks, split over M
    int db_splits, db_per;        // dB = dY^T [H_hi|H_lo]  : N tiles x chunks, split over M
    size_t off_h2, off_g2, off_part, off_part2, bytes;
};

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

Plan make_plan(int64_t M, int64_t N, int64_t K, int r, int sms)
{
    Plan pl{};
    pl.M = M;
    pl.N = N;
    pl.K = K;
    pl.r = r;
    pl.r_pad = pad64(r);
    const int chunks = pl.r_pad / 64;
    const int mt = ceil_div(M, 128), kt = ceil_div(K, 128), nt = ceil_div(N, 128);
    choose_splits(mt, ceil_div(K, 64), sms, 4, &pl.h_splits, &pl.h_per);
    choose_splits(mt, ceil_div(N, 64), sms, 4, &pl.g_splits, &pl.g_per);
    choose_splits(kt * chunks, ceil_div(M, 64), sms, 4, &pl.da_splits, &pl.da_per);
    choose_splits(nt * chunks, ceil_div(M, 64), sms, 4, &pl.db_splits, &pl.db_per);
    const size_t hl = align256((size_t)M * 2 * pl.r_pad * 2);
    size_t part = std::max((size_t)pl.h_splits, (size_t)pl.g_splits) * M * pl.r_pad * 4;
    part = std::max(part, (size_t)pl.da_splits * K * 2 * pl.r_pad * 4);
    const size_t part2 = (size_t)pl.db_splits * N * 2 * pl.r_pad * 4;
    pl.off_h2 = 0;
    pl.off_g2 = hl;
    pl.off_part = 2 * hl;
    pl.off_part2 = pl.off_part + align256(part);
    pl.bytes = pl.off_part2 + align256(part2);
    // the decode forward (M <= kDecodeMaxTokens) uses the start of the workspace for its partials
    if (M <= kDecodeMaxTokens) pl.bytes = std::max(pl.bytes, align256(decode_workspace_bytes(M, N, K, r, sms)));
    return pl;
}

qlora_status check_linear(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A, const void *B,
                          int32_t r, void *workspace)
{
    QLORA_TRY(check_weight(w));
    if (M < 0) return QLORA_ERR_INVALID_ARG;
    if (r < 8 || r > 128 || r % 8) return QLORA_ERR_SHAPE;
    if (w->rows % 8) return QLORA_ERR_SHAPE;
    if (w->rows > (int64_t)INT32_MAX || w->cols > (int64_t)INT32_MAX || M > (int64_t)INT32_MAX) return QLORA_ERR_SHAPE;
    if (!X || !A || !B || !workspace) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(workspace)) return QLORA_ERR_ALIGNMENT;
    return QLORA_OK;
}

void set_split(GemmParams &p, int splits, int per, int total_stages, int64_t plane)
{
    p.splits = splits;
    p.k_stages_total = total_stages;
    p.k_stages_split = per;
    p.split_stride = plane;
}

// H = s X A^T into the hi/lo buffer (and optionally fp32 H_out)
qlora_status run_h(const Plan &pl, const DeviceInfo &dev, const void *X, const void *A, float scale, float *H_out,
                   char *ws, cudaStream_t s)
{
    GemmParams p{};
    QLORA_TRY(map_bf16(&p.tm_a, X, pl.K, pl.M, pl.K, 64, 128));
    QLORA_TRY(map_bf16(&p.tm_b, A, pl.K, pl.r, pl.K, 64, pl.r_pad));
    p.m_tiles = ceil_div(pl.M, 128);
    p.n_tiles = 1;
    set_split(p, pl.h_splits, pl.h_per, ceil_div(pl.K, 64), pl.M * pl.r_pad);
    p.out = ws + pl.off_part;
    p.out_ld = pl.r_pad;
    p.m_total = (int)pl.M;
    p.n_total = pl.r_pad;
    if (pl.r_pad == 64)
        QLORA_TRY((launch_gemm<64, kBTmaK, kEpiF32>(p, dev, s, QLORA_KERNEL_LOWRANK)));
    else
        QLORA_TRY((launch_gemm<128, kBTmaK, kEpiF32>(p, dev, s, QLORA_KERNEL_LOWRANK)));
    {
        LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
        QLORA_CUDA_TRY(launch_pdl(finalize_lowrank_kernel, dim3(elementwise_grid(pl.M * pl.r_pad / 4)), dim3(256), 0,
                                  s, reinterpret_cast<const float *>(ws + pl.off_part), pl.h_splits,
                                  (int64_t)(pl.M * pl.r_pad), pl.M, pl.r, pl.r_pad, scale,
                                  reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_h2), H_out, (const float *)nullptr,
                                  (__nv_bfloat16 *)nullptr));
    }
    return launch_status();
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" size_t qlora_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r)
{
    if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return 256;
    DeviceInfo dev;
    int sms = device_info(&dev) == QLORA_OK ? dev.sms : 148;
    return make_plan(M, N, K, r, sms).bytes;
}

extern "C" qlora_status qlora_linear_fwd(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A,
                                         const void *B, int32_t r, float scale, void *Y, qlora_dtype y_dtype,
                                         float *H_save, void *workspace, size_t workspace_bytes, void *stream)
{
    QLORA_TRY(check_linear(w, X, M, A, B, r, workspace));
    if (!Y) return QLORA_ERR_INVALID_ARG;
    if (y_dtype != QLORA_BF16 && y_dtype != QLORA_FP32) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(Y) || (H_save && !aligned16(H_save))) return QLORA_ERR_ALIGNMENT;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    if (M == 0) return QLORA_OK;
    const Plan pl = make_plan(M, w->rows, w->cols, r, dev.sms);
    if (workspace_bytes < pl.bytes) return QLORA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);

    // a handful of tokens: stream the packed weight once (bound by HBM, not the tensor cores)
    if (M <= kDecodeMaxTokens)
        return run_decode_fwd(w, X, M, A, B, r, scale, Y, y_dtype, H_save, ws, workspace_bytes, dev, s);

    QLORA_TRY(run_h(pl, dev, X, A, scale, H_save, ws, s));

    // fused forward: 256 tokens (two 128-row accumulators) x 128 output features per tile
    constexpr int kFBN = 128, kFMT = 2;
    GemmParams p{};
    QLORA_TRY(map_bf16(&p.tm_a, X, pl.K, M, pl.K, 64, 128 * kFMT));
    QLORA_TRY(make_map(&p.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, pl.K / 2, pl.N, pl.K / 2, 32, kFBN,
                       CU_TENSOR_MAP_SWIZZLE_32B));
    QLORA_TRY(map_bf16(&p.tm_a2, ws + pl.off_h2, 2 * pl.r_pad, M, 2 * pl.r_pad, 64, 128 * kFMT));   // hi chunks of H
    QLORA_TRY(map_bf16(&p.tm_b2, B, r, pl.N, r, 64, kFBN));
    p.a2_x_step = 128;
    p.code2 = w->code2;
    p.c2 = w->c2;
    p.mean = w->mean;
    p.kblocks = pl.K / 64;
    p.wrows = pl.N;
    for (int i = 0; i < 16; i++) p.q[i] = w->codebook[i];
    p.m_tiles = ceil_div(M, 128 * kFMT);
    p.n_tiles = ceil_div(pl.N, kFBN);
    p.splits = 1;
    p.k_stages_total = (int)(pl.K / 64);
    p.k_stages_split = p.k_stages_total;
    p.k_stages_lora = pl.r_pad / 64;
    p.out = Y;
    p.out_ld = pl.N;
    p.m_total = (int)M;
    p.n_total = (int)pl.N;
    if (M > 128 * kFMT) {
        // more than one tile of tokens: CTA pairs, 512 tokens x 256 features per pair
        if (y_dtype == QLORA_BF16)
            QLORA_TRY(make_map(&p.tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, pl.N, M, pl.N * 2, 32, 32,
                               CU_TENSOR_MAP_SWIZZLE_64B));
        p.m_tiles = ceil_div(M, 2 * 128 * kFMT);
        p.n_tiles = ceil_div(pl.N, 2 * kFBN);
        if (y_dtype == QLORA_BF16) return launch_gemm_pair<kBNf4K, kEpiBf16, kFMT>(p, dev, s, QLORA_KERNEL_FWD_FUSED);
        return launch_gemm_pair<kBNf4K, kEpiF32, kFMT>(p, dev, s, QLORA_KERNEL_FWD_FUSED);
    }
    if (y_dtype == QLORA_BF16) return launch_gemm<kFBN, kBNf4K, kEpiBf16, kFMT>(p, dev, s, QLORA_KERNEL_FWD_FUSED);
    return launch_gemm<kFBN, kBNf4K, kEpiF32, kFMT>(p, dev, s, QLORA_KERNEL_FWD_FUSED);
}

extern "C" qlora_status qlora_linear_bwd(const qlora_nf4_weight *w, const void *X, const void *dY, int64_t M,
                                         const void *A, const void *B, int32_t r, float scale,
                                         const float *H_saved, void *dX, qlora_dtype dx_dtype, float *dA, float *dB,
                                         void *workspace, size_t workspace_bytes, void *stream)
{
    QLORA_TRY(check_linear(w, X, M, A, B, r, workspace));
    if (!dY || !dA || !dB) return QLORA_ERR_INVALID_ARG;
    if (dx_dtype != QLORA_BF16 && dx_dtype != QLORA_FP32) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(dY) || !aligned16(dA) || !aligned16(dB) || (dX && !aligned16(dX)) ||
        (H_saved && !aligned16(H_saved)))
        return QLORA_ERR_ALIGNMENT;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    const int64_t N = w->rows, K = w->cols;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) {
        // no tokens: the adapter gradients are zero
        QLORA_CUDA_TRY(cudaMemsetAsync(dA, 0, (size_t)r * K * 4, s));
        QLORA_CUDA_TRY(cudaMemsetAsync(dB, 0, (size_t)N * r * 4, s));
        return QLORA_OK;
    }
    const Plan pl = make_plan(M, N, K, r, dev.sms);
    if (workspace_bytes < pl.bytes) return QLORA_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    __nv_bfloat16 *H2 = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_h2);
    __nv_bfloat16 *G2 = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_g2);
    const int hl_cols = 2 * pl.r_pad;

    // H (hi/lo) recomputed when no saved H is given
    if (!H_saved) QLORA_TRY(run_h(pl, dev, X, A, scale, nullptr, ws, s));

    // G = s dY B (contraction over N); its finalize also splits a saved H into hi/lo
    {
        GemmParams p{};
        QLORA_TRY(map_bf16(&p.tm_a, dY, N, M, N, 64, 128));
        QLORA_TRY(map_bf16(&p.tm_b, B, r, N, r, 64, 64));      // B[n][j]: MN-major operand
        p.m_tiles = ceil_div(M, 128);
        p.n_tiles = 1;
        set_split(p, pl.g_splits, pl.g_per, ceil_div(N, 64), M * pl.r_pad);
        p.out = ws + pl.off_part;
        p.out_ld = pl.r_pad;
        p.m_total = (int)M;
        p.n_total = pl.r_pad;
        if (pl.r_pad == 64)
            QLORA_TRY((launch_gemm<64, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_LOWRANK)));
        else
            QLORA_TRY((launch_gemm<128, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_LOWRANK)));
        {
            LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
            QLORA_CUDA_TRY(launch_pdl(finalize_lowrank_kernel, dim3(elementwise_grid(M * pl.r_pad / 4)), dim3(256), 0,
                                      s, reinterpret_cast<const float *>(ws + pl.off_part), pl.g_splits,
                                      (int64_t)(M * pl.r_pad), M, r, pl.r_pad, scale, G2, (float *)nullptr, H_saved,
                                      H_saved ? H2 : (__nv_bfloat16 *)nullptr));
        }
        QLORA_TRY(launch_status());
    }

    // dX = dY W' + bf16(G) A  (fused transposed dequant-GEMM)
    if (dX) {
        // fused input gradient: 256 tokens x 128 input features per tile
        constexpr int kBBN = 128, kBMT = 2;
        GemmParams p{};
        QLORA_TRY(map_bf16(&p.tm_a, dY, N, M, N, 64, 128 * kBMT));
        QLORA_TRY(make_map(&p.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, K / 2, N, K / 2, kBBN / 2, 64,
                           kBBN == 256 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B));
        QLORA_TRY(map_bf16(&p.tm_a2, G2, hl_cols, M, hl_cols, 64, 128 * kBMT));   // hi chunks of G
        QLORA_TRY(map_bf16(&p.tm_b2, A, K, r, K, 64, 64));                        // A[j][k]: MN-major operand
        p.a2_x_step = 128;
        p.code2 = w->code2;
        p.c2 = w->c2;
        p.mean = w->mean;
        p.kblocks = K / 64;
        p.wrows = N;
        for (int i = 0; i < 16; i++) p.q[i] = w->codebook[i];
        p.m_tiles = ceil_div(M, 128 * kBMT);
        p.n_tiles = ceil_div(K, kBBN);
        p.splits = 1;
        p.k_stages_total = ceil_div(N, 64);
        p.k_stages_split = p.k_stages_total;
        p.k_stages_lora = pl.r_pad / 64;
        p.out = dX;
        p.out_ld = K;
        p.m_total = (int)M;
        p.n_total = (int)K;
        if (M > 128 * kBMT) {
            // CTA pairs: 512 tokens x 256 input features per pair
            if (dx_dtype == QLORA_BF16)
                QLORA_TRY(make_map(&p.tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dX, K, M, K * 2, 32, 32,
                                   CU_TENSOR_MAP_SWIZZLE_64B));
            p.m_tiles = ceil_div(M, 2 * 128 * kBMT);
            p.n_tiles = ceil_div(K, 2 * kBBN);
            if (dx_dtype == QLORA_BF16)
                QLORA_TRY((launch_gemm_pair<kBNf4MN, kEpiBf16, kBMT>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
            else
                QLORA_TRY((launch_gemm_pair<kBNf4MN, kEpiF32, kBMT>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
        } else if (dx_dtype == QLORA_BF16)
            QLORA_TRY((launch_gemm<kBBN, kBNf4MN, kEpiBf16, kBMT>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
        else
            QLORA_TRY((launch_gemm<kBBN, kBNf4MN, kEpiF32, kBMT>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
    }

    // dA^T = X^T [G_hi | G_lo]  and  dB = dY^T [H_hi | H_lo]: rows k (resp. n), chunked
    // hi | lo columns, contraction over tokens; one finalize adds the halves
    float *part_a = reinterpret_cast<float *>(ws + pl.off_part);
    float *part_b = reinterpret_cast<float *>(ws + pl.off_part2);
    {
        GemmParams p{};
        QLORA_TRY(map_bf16(&p.tm_a, X, K, M, K, 64, 64));              // MN-major A
        QLORA_TRY(map_bf16(&p.tm_b, G2, hl_cols, M, hl_cols, 64, 64));  // MN-major B
        p.a_mn = 1;
        p.m_tiles = ceil_div(K, 128);
        p.n_tiles = pl.r_pad / 64;
        set_split(p, pl.da_splits, pl.da_per, ceil_div(M, 64), K * hl_cols);
        p.out = part_a;
        p.out_ld = hl_cols;
        p.m_total = (int)K;
        p.n_total = hl_cols;
        QLORA_TRY((launch_gemm<128, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_WGRAD)));
    }
    {
        GemmParams p{};
        QLORA_TRY(map_bf16(&p.tm_a, dY, N, M, N, 64, 64));              // MN-major A
        QLORA_TRY(map_bf16(&p.tm_b, H2, hl_cols, M, hl_cols, 64, 64));  // MN-major B
        p.a_mn = 1;
        p.m_tiles = ceil_div(N, 128);
        p.n_tiles = pl.r_pad / 64;
        set_split(p, pl.db_splits, pl.db_per, ceil_div(M, 64), N * hl_cols);
        p.out = part_b;
        p.out_ld = hl_cols;
        p.m_total = (int)N;
        p.n_total = hl_cols;
        QLORA_TRY((launch_gemm<128, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_WGRAD)));
    }
    {
        WgradJob ja{part_a, pl.da_splits, K * hl_cols, K, dA, K, 1};
        WgradJob jb{part_b, pl.db_splits, N * hl_cols, N, dB, r, 0};
        const int64_t n0 = K * (r / 4), n1 = N * (r / 4);
        LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
        QLORA_CUDA_TRY(launch_pdl(finalize_wgrad_kernel, dim3(elementwise_grid(n0 + n1)), dim3(256), 0, s, ja, jb,
                                  (int64_t)n0, r, pl.r_pad));
    }
    return launch_status();
}
