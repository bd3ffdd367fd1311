// QLoRA linear layer on sm_100a: forward Y = X W'^T + s (X A^T) B^T and the
// backward pass dX, dA, dB (no dW: the quantized weight is frozen).
//
// Sources: mbrenndoerfer.com QLoRA essay, section "Low-Rank Adaptation
// (LoRA)" (x_out = (W_q + BA) x_in, A is r x d, B is d x r); "QLoRA: Efficient
// Finetuning of Quantized LLMs", section "Method" (dequantize to BFloat16 and
// multiply in 16-bit) and abstract (gradients flow through the frozen 4-bit
// weight into the adapters).
//
// Launch sequence (all on the caller's stream, chained by programmatic
// dependent launch):
//   forward : H = s X A^T (cluster split-K, hi/lo bf16 + optional fp32 H)
//             -> fused dequant-GEMM with the LoRA up-projection as extra K steps
//   backward: [H recomputed when no saved H is given]
//             -> G = s dY B (cluster split-K, hi/lo bf16; a saved H is split
//                into hi/lo in the same kernel)
//             -> fused transposed dequant-GEMM for dX (+ G A)
//             -> dA = G^T X and dB = dY^T H in one launch (cluster split over
//                the tokens); its inputs were all written at least two
//                launches earlier, so it starts without waiting for the dX
//                GEMM and fills the SMs that GEMM's last wave leaves idle
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
#include "debug.cuh"
#include "decode.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_skinny.cuh"

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

template <int BN, int kBMode, int kEpi, int MT = 1, bool F16 = false>
qlora_status launch_gemm(GemmParams &p, const DeviceInfo &dev, cudaStream_t s, int kind)
{
    using Cfg = GemmCfg<BN, kBMode, MT>;
    static PerDeviceOnce attr;
    auto kern = qgemm_kernel<BN, kBMode, kEpi, MT, F16>;
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
template <int kBMode, int kEpi, int MT, bool F16 = false>
qlora_status launch_gemm_pair(GemmParams &p, const DeviceInfo &dev, cudaStream_t s, int kind)
{
    using Cfg = PairCfg<kBMode, MT>;
    static PerDeviceOnce setup;
    static int max_clusters[kMaxDevices] = {};
    auto kern = qgemm_pair_kernel<kBMode, kEpi, MT, F16>;
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

int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }
int pad64(int v) { return (v + 63) / 64 * 64; }

// ---- skinny products (gemm_skinny.cuh) ------------------------------------------

// Launches one skinny-product grid: `clusters` output tiles, `csize` CTAs per
// cluster (the contraction split).
template <int BN, int A_MN, int B_MN, bool F16 = false>
qlora_status launch_skinny(SkinnyParams &p, int clusters, int csize, const DeviceInfo &dev, cudaStream_t s, int kind)
{
    using Cfg = SkinnyCfg<BN, A_MN, B_MN>;
    auto kern = qgemm_skinny_kernel<BN, A_MN, B_MN, F16>;
    p.err = device_error_word();
    if (!p.err) return QLORA_ERR_CUDA;
    p.timeout_ns = kTimeoutNs;
    p.drain_ns = kTimeoutNs;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(clusters * csize));
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    {
        LaunchScope ls(kind, s);
        QLORA_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, p));
    }
    return launch_status();
}

// Kernel attributes and the number of co-resident clusters for each cluster
// size 1, 2, 4, 8 (once per device and instantiation).
template <int BN, int A_MN, int B_MN, bool F16 = false>
qlora_status skinny_setup(const DeviceInfo &dev, const int **max_clusters)
{
    using Cfg = SkinnyCfg<BN, A_MN, B_MN>;
    static PerDeviceOnce once;
    static int maxc[kMaxDevices][4] = {};
    auto kern = qgemm_skinny_kernel<BN, A_MN, B_MN, F16>;
    QLORA_TRY(once.run(dev.device, [&]() -> qlora_status {
        QLORA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
        for (int i = 0; i < 4; i++) {
            const int c = 1 << i;
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3((unsigned)(c * (dev.sms / c)));
            cfg.blockDim = dim3(Cfg::kThreads);
            cfg.dynamicSmemBytes = Cfg::kSmemBytes;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)c;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            QLORA_CUDA_TRY(cudaOccupancyMaxActiveClusters(&n, kern, &cfg));
            maxc[dev.device][i] = n;
        }
        return QLORA_OK;
    }));
    *max_clusters = maxc[dev.device];
    return QLORA_OK;
}

// Contraction split (cluster size): the largest of 8, 4, 2 for which all
// tiles' clusters are co-resident in one wave and every CTA keeps at least
// four 64-deep steps; else 1.
int choose_csize(int tiles, int k_total, const int *max_clusters)
{
    for (int i = 3; i >= 1; i--) {
        const int c = 1 << i;
        if (tiles <= max_clusters[i] && k_total >= 4 * c) return c;
    }
    return 1;
}

qlora_status map_k_major(CUtensorMap *m, const void *base, int64_t inner, int64_t rows, uint32_t box_rows)
{
    return map_bf16(m, base, (uint64_t)inner, (uint64_t)rows, (uint64_t)inner, 64, box_rows);
}

// ---- problem plan -------------------------------------------------------------------

// H2 / G2 buffers: [M][2*r_pad] bf16, 64-column chunks alternating hi | lo
// (hi of columns 64c..64c+63 at 128c, their lo at 128c+64).
struct Plan {
    int64_t M, N, K;
    int r, r_pad;
    size_t off_h2, off_g2, bytes;
    // 17..256 tokens (single-CTA engine): contraction splits of the fused
    // forward and input gradient when their output tiles would leave SMs idle,
    // and the fp32 partial planes they write
    int split_fwd, split_dx;
    size_t off_split;
    // LoRA dropout: the dropped-out input X_d (bf16 [M][K]) and the frozen
    // path's fp32 input gradient [M][K]
    size_t off_xd, off_dxs;
};

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Contraction splits for a single-CTA fused GEMM with `tiles` output tiles and
// `k_steps` 64-deep steps: enough CTAs to cover the SMs, at most 8 splits and
// at least 8 steps per split.
int choose_splits(int tiles, int k_steps, int sms)
{
    int sp = tiles > 0 ? sms / tiles : 1;
    sp = std::max(1, std::min(sp, 8));
    while (sp > 1 && k_steps / sp < 8) sp--;
    return sp;
}

Plan make_plan(int64_t M, int64_t N, int64_t K, int r, int sms, bool dropout = false)
{
    Plan pl{};
    pl.M = M;
    pl.N = N;
    pl.K = K;
    pl.r = r;
    pl.r_pad = pad64(r);
    const size_t hl = align256((size_t)M * 2 * pl.r_pad * 2);
    pl.off_h2 = 0;
    pl.off_g2 = hl;
    pl.bytes = 2 * hl;
    // the decode forward (M <= kDecodeMaxTokens) uses the start of the workspace for its partials
    if (M <= kDecodeMaxTokens) pl.bytes = std::max(pl.bytes, align256(decode_workspace_bytes(M, N, K, r, sms)));
    if (dropout) {
        pl.off_xd = pl.bytes;
        pl.off_dxs = pl.off_xd + align256((size_t)M * K * 2);
        pl.bytes = pl.off_dxs + align256((size_t)M * K * 4);
    }
    pl.split_fwd = pl.split_dx = 1;
    if (M > kDecodeMaxTokens && M <= 256) {
        pl.split_fwd = choose_splits(ceil_div(N, 128), (int)(K / 64), sms);
        pl.split_dx = dropout ? 1 : choose_splits(ceil_div(K, 128), ceil_div(N, 64), sms);
        const size_t planes = std::max((size_t)pl.split_fwd * M * N, (size_t)pl.split_dx * M * K);
        if (pl.split_fwd > 1 || pl.split_dx > 1) {
            pl.off_split = pl.bytes;
            pl.bytes = pl.off_split + align256(planes * 4);
        }
    }
    return pl;
}

// ---- split contraction of the single-CTA fused GEMMs ------------------------------------

// out[m][c] = sum over s = 0 .. splits-1 (in that order) of planes[s][m][c],
// stored as bf16 / fp16 / fp32; four columns per thread (cols % 4 == 0).
__global__ void __launch_bounds__(256) split_sum_kernel(const float *planes, int splits, int64_t rows, int64_t cols,
                                                        void *out, int out_type)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int64_t n4 = rows * cols / 4, plane = rows * cols;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        float4 a = __ldcg(reinterpret_cast<const float4 *>(planes) + i);
        for (int sp = 1; sp < splits; sp++) {
            if (!QLORA_IN(sp * plane + 4 * i + 3, splits * plane)) break;
            const float4 b = __ldcg(reinterpret_cast<const float4 *>(planes + sp * plane) + i);
            a = make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
        }
        if (out_type == QLORA_FP32) {
            reinterpret_cast<float4 *>(out)[i] = a;
        } else if (out_type == QLORA_FP16) {
            const __half2 lo = __floats2half2_rn(a.x, a.y), hi = __floats2half2_rn(a.z, a.w);
            reinterpret_cast<uint2 *>(out)[i] =
                make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
        } else {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
            reinterpret_cast<uint2 *>(out)[i] =
                make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
        }
    }
}

qlora_status run_split_sum(const float *planes, int splits, int64_t rows, int64_t cols, void *out, qlora_dtype out_type,
                           const DeviceInfo &dev, cudaStream_t s, int kind)
{
    const int64_t n4 = rows * cols / 4;
    const int grid = (int)std::min<int64_t>((n4 + 255) / 256, 4 * dev.sms);
    LaunchScope ls(kind, s);
    QLORA_CUDA_TRY(launch_pdl(split_sum_kernel, dim3(grid), dim3(256), 0, s, planes, splits, rows, cols, out,
                              (int)out_type));
    return launch_status();
}

// ---- LoRA dropout ---------------------------------------------------------------------
//
// The blog's LoraConfig snippet ("Efficient Language Model Fine-Tuning with
// QLoRA on Resource-Constrained Hardware", marciocunha.net) sets lora_dropout:
// the adapter branch sees X_d = X * mask / (1 - p), the frozen path X.  Kept
// elements are RN_bf16(RN32(x * RN32(1 / (1 - p)))), dropped ones 0; the
// mask holds bit k % 8 of byte (m K + k) / 8 for element (m, k), 1 = kept.

bool dropout_on(const qlora_linear_opts *o) { return o && o->dropout_mask; }

// Which part of a linear call runs: all of it, only the adapter's low-rank
// products (the split-off first step), or all but them (adapter_ready).
enum Phase { kPhaseAll, kPhaseAdapter, kPhaseMain };
Phase phase_of(const qlora_linear_opts *o) { return o && o->adapter_ready ? kPhaseMain : kPhaseAll; }

float dropout_scale(const qlora_linear_opts *o) { return 1.0f / (1.0f - o->dropout_p); }

// X_d from X and the mask, eight elements (one mask byte) per thread (F16:
// fp16 X and X_d).
template <bool F16>
__global__ void __launch_bounds__(256) dropout_input_kernel(const __nv_bfloat16 *X, const uint8_t *mask, float scale,
                                                            __nv_bfloat16 *Xd, int64_t n8)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 xv = *reinterpret_cast<const uint4 *>(X + 8 * i);
        const uint32_t bits = mask[i];
        const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            float xa, xb;
            if constexpr (F16) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[j]));
                xa = f.x;
                xb = f.y;
            } else {
                xa = __uint_as_float(w[j] << 16);
                xb = __uint_as_float(w[j] & 0xFFFF0000u);
            }
            const uint32_t packed = nf4::pack16x2<F16>(__fmul_rn(xa, scale), __fmul_rn(xb, scale));
            const uint32_t keep = ((bits >> (2 * j)) & 1u ? 0x0000FFFFu : 0u) | ((bits >> (2 * j + 1)) & 1u ? 0xFFFF0000u : 0u);
            o[j] = packed & keep;
        }
        *reinterpret_cast<uint4 *>(Xd + 8 * i) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

template <bool F16>
qlora_status run_dropout_input(const Plan &pl, const DeviceInfo &dev, const void *X, const qlora_linear_opts *o,
                               char *ws, cudaStream_t s)
{
    const int64_t n8 = pl.M * pl.K / 8;
    const int grid = (int)std::min<int64_t>((n8 + 255) / 256, (int64_t)dev.sms * 16);
    LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
    QLORA_CUDA_TRY(launch_pdl(dropout_input_kernel<F16>, dim3(grid), dim3(256), 0, s, static_cast<const __nv_bfloat16 *>(X),
                              o->dropout_mask, dropout_scale(o), reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_xd),
                              n8));
    return launch_status();
}

qlora_status check_opts(const qlora_linear_opts *o)
{
    if (!o) return QLORA_OK;
    if (o->compute_dtype != QLORA_BF16 && o->compute_dtype != QLORA_FP16) return QLORA_ERR_INVALID_ARG;
    if (o->adapter_ready != 0 && o->adapter_ready != 1) return QLORA_ERR_INVALID_ARG;
    if (!o->dropout_mask) return QLORA_OK;
    if (!(o->dropout_p >= 0.0f && o->dropout_p < 1.0f)) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(o->dropout_mask)) return QLORA_ERR_ALIGNMENT;
    return QLORA_OK;
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

// Low-rank factor v = scale * P Q^T (P [M][Kc] bf16, Q given as the B operand)
// into the hi/lo buffer `hl`, with an optional fp32 copy and an optional
// hi/lo split of aux_in into aux_out.
template <int BN, int B_MN, bool F16 = false>
qlora_status run_lowrank(const Plan &pl, const DeviceInfo &dev, const void *P, int64_t Kc, const void *Q,
                         float scale, __nv_bfloat16 *hl, float *f32_out, const float *aux_in, __nv_bfloat16 *aux_out,
                         cudaStream_t s)
{
    const int *maxc = nullptr;
    QLORA_TRY((skinny_setup<BN, 0, B_MN, F16>(dev, &maxc)));
    SkinnyParams p{};
    SkinnyJob &J = p.job[0];
    QLORA_TRY(map_k_major(&J.tm_a, P, Kc, pl.M, 128));
    if (B_MN)
        QLORA_TRY(map_k_major(&J.tm_b, Q, pl.r, Kc, 64));       // B [Kc][r]: 64-column chunks
    else
        QLORA_TRY(map_k_major(&J.tm_b, Q, Kc, pl.r, pl.r_pad));  // A [r][Kc]
    J.m_tiles = ceil_div(pl.M, 128);
    J.k_total = ceil_div(Kc, 64);
    J.fin = kFinLowRank;
    J.m_total = (int)pl.M;
    J.scale = scale;
    J.r = pl.r;
    J.r_pad = pl.r_pad;
    J.hl_out = hl;
    J.f32_out = f32_out;
    J.aux_in = aux_in;
    J.aux_out = aux_out;
    p.clusters0 = J.m_tiles;
    p.wait_at_end = 0;
    const int cs = choose_csize(J.m_tiles, J.k_total, maxc);
    return launch_skinny<BN, 0, B_MN, F16>(p, J.m_tiles, cs, dev, s, QLORA_KERNEL_LOWRANK);
}

// H = s X A^T into the hi/lo buffer (and optionally fp32 H_out)
template <bool F16>
qlora_status run_h(const Plan &pl, const DeviceInfo &dev, const void *X, const void *A, float scale, float *H_out,
                   char *ws, cudaStream_t s)
{
    __nv_bfloat16 *H2 = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_h2);
    if (pl.r_pad == 64)
        return run_lowrank<64, 0, F16>(pl, dev, X, pl.K, A, scale, H2, H_out, nullptr, nullptr, s);
    return run_lowrank<128, 0, F16>(pl, dev, X, pl.K, A, scale, H2, H_out, nullptr, nullptr, s);
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" size_t qlora_linear_workspace_bytes_ex(int64_t M, int64_t N, int64_t K, int32_t r,
                                                  const qlora_linear_opts *opts)
{
    if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return 256;
    DeviceInfo dev;
    int sms = device_info(&dev) == QLORA_OK ? dev.sms : 148;
    return make_plan(M, N, K, r, sms, dropout_on(opts)).bytes;
}

extern "C" size_t qlora_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r)
{
    return qlora_linear_workspace_bytes_ex(M, N, K, r, nullptr);
}

template <bool F16>
static qlora_status linear_fwd(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A, const void *B,
                               int32_t r, float scale, void *Y, qlora_dtype y_dtype, float *H_save, void *workspace,
                               size_t workspace_bytes, void *stream, const qlora_linear_opts *opts, Phase phase)
{
    const bool drop = dropout_on(opts);
    if (phase != kPhaseAdapter) {
        if (!Y) return QLORA_ERR_INVALID_ARG;
        if (y_dtype != (F16 ? QLORA_FP16 : QLORA_BF16) && y_dtype != QLORA_FP32) return QLORA_ERR_INVALID_ARG;
        if (!aligned16(Y)) return QLORA_ERR_ALIGNMENT;
    }
    if (H_save && !aligned16(H_save)) return QLORA_ERR_ALIGNMENT;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    if (M == 0) return QLORA_OK;
    const Plan pl = make_plan(M, w->rows, w->cols, r, dev.sms, drop);
    if (workspace_bytes < pl.bytes) return QLORA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    // the adapter branch's input: X, or X_d under LoRA dropout
    const void *Xa = X;
    if (drop) {
        if (phase != kPhaseMain) QLORA_TRY(run_dropout_input<F16>(pl, dev, X, opts, ws, s));
        Xa = ws + pl.off_xd;
    }

    // a handful of tokens: stream the packed weight once (bound by HBM, not
    // the tensor cores); H is formed inside that path
    if (M <= kDecodeMaxTokens) {
        if (phase == kPhaseAdapter) return launch_status();
        return run_decode_fwd(w, X, Xa, M, A, B, r, scale, Y, y_dtype, H_save, ws, workspace_bytes, dev, s, F16);
    }

    if (phase != kPhaseMain) QLORA_TRY(run_h<F16>(pl, dev, Xa, A, scale, H_save, ws, s));
    if (phase == kPhaseAdapter) return launch_status();

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
        if (y_dtype != QLORA_FP32)
            QLORA_TRY(make_map(&p.tm_out, F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y,
                               pl.N, M, pl.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
        p.m_tiles = ceil_div(M, 2 * 128 * kFMT);
        p.n_tiles = ceil_div(pl.N, 2 * kFBN);
        if (y_dtype != QLORA_FP32) return launch_gemm_pair<kBNf4K, kEpiBf16, kFMT, F16>(p, dev, s, QLORA_KERNEL_FWD_FUSED);
        return launch_gemm_pair<kBNf4K, kEpiF32, kFMT, F16>(p, dev, s, QLORA_KERNEL_FWD_FUSED);
    }
    if (pl.split_fwd > 1) {
        // few output tiles: split the contraction, then sum the planes in order
        float *planes = reinterpret_cast<float *>(ws + pl.off_split);
        p.splits = pl.split_fwd;
        p.k_stages_split = ceil_div(p.k_stages_total, p.splits);
        p.out = planes;
        p.split_stride = M * pl.N;
        QLORA_TRY((launch_gemm<kFBN, kBNf4K, kEpiF32, kFMT, F16>(p, dev, s, QLORA_KERNEL_FWD_FUSED)));
        return run_split_sum(planes, p.splits, M, pl.N, Y, y_dtype, dev, s, QLORA_KERNEL_ELEMENTWISE);
    }
    if (y_dtype != QLORA_FP32) return launch_gemm<kFBN, kBNf4K, kEpiBf16, kFMT, F16>(p, dev, s, QLORA_KERNEL_FWD_FUSED);
    return launch_gemm<kFBN, kBNf4K, kEpiF32, kFMT, F16>(p, dev, s, QLORA_KERNEL_FWD_FUSED);
}

extern "C" qlora_status qlora_linear_fwd_ex(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A,
                                            const void *B, int32_t r, float scale, void *Y, qlora_dtype y_dtype,
                                            float *H_save, void *workspace, size_t workspace_bytes, void *stream,
                                            const qlora_linear_opts *opts)
{
    QLORA_TRY(check_linear(w, X, M, A, B, r, workspace));
    QLORA_TRY(check_opts(opts));
    if (opts && opts->compute_dtype == QLORA_FP16)
        return linear_fwd<true>(w, X, M, A, B, r, scale, Y, y_dtype, H_save, workspace, workspace_bytes, stream, opts,
                                phase_of(opts));
    return linear_fwd<false>(w, X, M, A, B, r, scale, Y, y_dtype, H_save, workspace, workspace_bytes, stream, opts,
                             phase_of(opts));
}

extern "C" qlora_status qlora_linear_adapter_fwd(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A,
                                                 const void *B, int32_t r, float scale, float *H_save,
                                                 void *workspace, size_t workspace_bytes, void *stream,
                                                 const qlora_linear_opts *opts)
{
    QLORA_TRY(check_linear(w, X, M, A, B, r, workspace));
    QLORA_TRY(check_opts(opts));
    const qlora_dtype none = QLORA_FP32;
    if (opts && opts->compute_dtype == QLORA_FP16)
        return linear_fwd<true>(w, X, M, A, B, r, scale, nullptr, none, H_save, workspace, workspace_bytes, stream,
                                opts, kPhaseAdapter);
    return linear_fwd<false>(w, X, M, A, B, r, scale, nullptr, none, H_save, workspace, workspace_bytes, stream, opts,
                             kPhaseAdapter);
}

extern "C" qlora_status qlora_linear_fwd(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A,
                                         const void *B, int32_t r, float scale, void *Y, qlora_dtype y_dtype,
                                         float *H_save, void *workspace, size_t workspace_bytes, void *stream)
{
    return qlora_linear_fwd_ex(w, X, M, A, B, r, scale, Y, y_dtype, H_save, workspace, workspace_bytes, stream,
                               nullptr);
}

template <bool F16>
static qlora_status linear_bwd(const qlora_nf4_weight *w, const void *X, const void *dY, int64_t M, const void *A,
                               const void *B, int32_t r, float scale, const float *H_saved, void *dX,
                               qlora_dtype dx_dtype, float *dA, float *dB, void *workspace, size_t workspace_bytes,
                               void *stream, const qlora_linear_opts *opts, Phase phase)
{
    const bool drop = dropout_on(opts);
    if (!dY) return QLORA_ERR_INVALID_ARG;
    // the weight gradients are formed unless both dA and dB are NULL, which
    // only the rest of a split call allows (it then forms dX alone)
    const bool wgrad = dA || dB;
    if (phase != kPhaseAdapter) {
        if (wgrad && (!dA || !dB)) return QLORA_ERR_INVALID_ARG;
        if (!wgrad && (phase != kPhaseMain || !dX)) return QLORA_ERR_INVALID_ARG;
        if (dx_dtype != (F16 ? QLORA_FP16 : QLORA_BF16) && dx_dtype != QLORA_FP32) return QLORA_ERR_INVALID_ARG;
        if ((wgrad && (!aligned16(dA) || !aligned16(dB))) || (dX && !aligned16(dX))) return QLORA_ERR_ALIGNMENT;
    }
    if (!aligned16(dY) || (H_saved && !aligned16(H_saved))) return QLORA_ERR_ALIGNMENT;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    const int64_t N = w->rows, K = w->cols;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) {
        if (phase == kPhaseAdapter || !wgrad) return QLORA_OK;
        // no tokens: the adapter gradients are zero
        QLORA_CUDA_TRY(cudaMemsetAsync(dA, 0, (size_t)r * K * 4, s));
        QLORA_CUDA_TRY(cudaMemsetAsync(dB, 0, (size_t)N * r * 4, s));
        return QLORA_OK;
    }
    const Plan pl = make_plan(M, N, K, r, dev.sms, drop);
    if (workspace_bytes < pl.bytes) return QLORA_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    __nv_bfloat16 *H2 = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_h2);
    __nv_bfloat16 *G2 = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_g2);
    const int hl_cols = 2 * pl.r_pad;
    // the adapter branch's input: X, or X_d under LoRA dropout
    const void *Xa = X;
    if (drop) {
        if (phase != kPhaseMain) QLORA_TRY(run_dropout_input<F16>(pl, dev, X, opts, ws, s));
        Xa = ws + pl.off_xd;
    }

    if (phase != kPhaseMain) {
        // H (hi/lo) recomputed when no saved H is given
        if (!H_saved) QLORA_TRY(run_h<F16>(pl, dev, Xa, A, scale, nullptr, ws, s));
        // G = s dY B (contraction over N); the same kernel splits a saved H into hi/lo
        if (pl.r_pad == 64)
            QLORA_TRY((run_lowrank<64, 1, F16>(pl, dev, dY, N, B, scale, G2, nullptr, H_saved, H_saved ? H2 : nullptr,
                                               s)));
        else
            QLORA_TRY((run_lowrank<128, 1, F16>(pl, dev, dY, N, B, scale, G2, nullptr, H_saved, H_saved ? H2 : nullptr,
                                                s)));
        if (phase == kPhaseAdapter) return launch_status();
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
        // under dropout the adapter term is masked elementwise: the fused GEMM
        // forms the frozen path dY W' alone, in fp32, and a second product adds
        // the masked adapter term (below)
        const bool f32_out = drop || dx_dtype == QLORA_FP32;
        if (drop) {
            p.k_stages_lora = 0;
            p.out = ws + pl.off_dxs;
        }
        if (M > 128 * kBMT) {
            // CTA pairs: 512 tokens x 256 input features per pair
            if (!f32_out)
                QLORA_TRY(make_map(&p.tm_out,
                                   F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dX, K,
                                   M, K * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
            p.m_tiles = ceil_div(M, 2 * 128 * kBMT);
            p.n_tiles = ceil_div(K, 2 * kBBN);
            if (!f32_out)
                QLORA_TRY((launch_gemm_pair<kBNf4MN, kEpiBf16, kBMT, F16>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
            else
                QLORA_TRY((launch_gemm_pair<kBNf4MN, kEpiF32, kBMT, F16>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
        } else if (pl.split_dx > 1) {
            // few output tiles: split the contraction, then sum the planes in order
            float *planes = reinterpret_cast<float *>(ws + pl.off_split);
            p.splits = pl.split_dx;
            p.k_stages_split = ceil_div(p.k_stages_total, p.splits);
            p.out = planes;
            p.split_stride = M * K;
            QLORA_TRY((launch_gemm<kBBN, kBNf4MN, kEpiF32, kBMT, F16>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
            QLORA_TRY(run_split_sum(planes, p.splits, M, K, dX, dx_dtype, dev, s, QLORA_KERNEL_ELEMENTWISE));
        } else if (!f32_out)
            QLORA_TRY((launch_gemm<kBBN, kBNf4MN, kEpiBf16, kBMT, F16>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
        else
            QLORA_TRY((launch_gemm<kBBN, kBNf4MN, kEpiF32, kBMT, F16>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
        if (drop) {
            // dX = frozen path + (bf16(G) A) * mask / (1 - p): the adapter product
            // alone (LoRA steps only), its epilogue adding the masked term
            GemmParams q{};
            QLORA_TRY(map_bf16(&q.tm_a2, G2, hl_cols, M, hl_cols, 64, 128 * kBMT));   // hi chunks of G
            QLORA_TRY(map_bf16(&q.tm_b2, A, K, r, K, 64, 64));                        // A[j][k]: MN-major operand
            q.tm_a = q.tm_a2;   // main operands unused (no main steps)
            q.tm_b = q.tm_b2;
            q.a2_x_step = 128;
            q.m_tiles = ceil_div(M, 128 * kBMT);
            q.n_tiles = ceil_div(K, kBBN);
            q.splits = 1;
            q.k_stages_total = 0;
            q.k_stages_split = 0;
            q.k_stages_lora = pl.r_pad / 64;
            q.out = dX;
            q.out_ld = K;
            q.m_total = (int)M;
            q.n_total = (int)K;
            q.drop_mask = opts->dropout_mask;
            q.drop_base = reinterpret_cast<const float *>(ws + pl.off_dxs);
            q.drop_scale = dropout_scale(opts);
            if (dx_dtype != QLORA_FP32)
                QLORA_TRY((launch_gemm<kBBN, kBTmaMN, kEpiDropBf16, kBMT, F16>(q, dev, s, QLORA_KERNEL_BWD_FUSED)));
            else
                QLORA_TRY((launch_gemm<kBBN, kBTmaMN, kEpiDropF32, kBMT, F16>(q, dev, s, QLORA_KERNEL_BWD_FUSED)));
        }
    }

    // dA = (X^T [G_hi | G_lo])^T and dB = dY^T [H_hi | H_lo] in one launch: output rows k
    // (resp. n), 128-column tiles = the hi and lo halves of one 64-column chunk,
    // contraction over the tokens; the reduction adds the halves
    if (wgrad) {
        const int *maxc = nullptr;
        QLORA_TRY((skinny_setup<128, 1, 1, F16>(dev, &maxc)));
        SkinnyParams p{};
        SkinnyJob &Ja = p.job[0], &Jb = p.job[1];
        QLORA_TRY(map_bf16(&Ja.tm_a, Xa, K, M, K, 64, 64));              // MN-major: rows k, contraction m
        QLORA_TRY(map_bf16(&Ja.tm_b, G2, hl_cols, M, hl_cols, 64, 64));
        QLORA_TRY(map_bf16(&Jb.tm_a, dY, N, M, N, 64, 64));
        QLORA_TRY(map_bf16(&Jb.tm_b, H2, hl_cols, M, hl_cols, 64, 64));
        const int chunks = pl.r_pad / 64;
        Ja.m_tiles = ceil_div(K, 128);
        Jb.m_tiles = ceil_div(N, 128);
        Ja.k_total = Jb.k_total = ceil_div(M, 64);
        Ja.fin = kFinWgradT;
        Jb.fin = kFinWgrad;
        Ja.m_total = (int)K;
        Jb.m_total = (int)N;
        Ja.r = Jb.r = r;
        Ja.r_pad = Jb.r_pad = pl.r_pad;
        Ja.f32_out = dA;
        Ja.out_ld = K;
        Jb.f32_out = dB;
        Jb.out_ld = r;
        const int tiles_a = Ja.m_tiles * chunks, tiles_b = Jb.m_tiles * chunks;
        p.clusters0 = tiles_a;
        // after the dX GEMM nothing read here comes from the kernel just before
        p.wait_at_end = dX ? 1 : 0;
        const int cs = choose_csize(tiles_a + tiles_b, Ja.k_total, maxc);
        QLORA_TRY((launch_skinny<128, 1, 1, F16>(p, tiles_a + tiles_b, cs, dev, s, QLORA_KERNEL_WGRAD)));
    }
    return launch_status();
}

extern "C" qlora_status qlora_linear_bwd_ex(const qlora_nf4_weight *w, const void *X, const void *dY, int64_t M,
                                            const void *A, const void *B, int32_t r, float scale,
                                            const float *H_saved, void *dX, qlora_dtype dx_dtype, float *dA,
                                            float *dB, void *workspace, size_t workspace_bytes, void *stream,
                                            const qlora_linear_opts *opts)
{
    QLORA_TRY(check_linear(w, X, M, A, B, r, workspace));
    QLORA_TRY(check_opts(opts));
    if (opts && opts->compute_dtype == QLORA_FP16)
        return linear_bwd<true>(w, X, dY, M, A, B, r, scale, H_saved, dX, dx_dtype, dA, dB, workspace, workspace_bytes,
                                stream, opts, phase_of(opts));
    return linear_bwd<false>(w, X, dY, M, A, B, r, scale, H_saved, dX, dx_dtype, dA, dB, workspace, workspace_bytes,
                             stream, opts, phase_of(opts));
}

extern "C" qlora_status qlora_linear_adapter_bwd(const qlora_nf4_weight *w, const void *X, const void *dY, int64_t M,
                                                 const void *A, const void *B, int32_t r, float scale,
                                                 const float *H_saved, void *workspace, size_t workspace_bytes,
                                                 void *stream, const qlora_linear_opts *opts)
{
    QLORA_TRY(check_linear(w, X, M, A, B, r, workspace));
    QLORA_TRY(check_opts(opts));
    const qlora_dtype none = QLORA_FP32;
    if (opts && opts->compute_dtype == QLORA_FP16)
        return linear_bwd<true>(w, X, dY, M, A, B, r, scale, H_saved, nullptr, none, nullptr, nullptr, workspace,
                                workspace_bytes, stream, opts, kPhaseAdapter);
    return linear_bwd<false>(w, X, dY, M, A, B, r, scale, H_saved, nullptr, none, nullptr, nullptr, workspace,
                             workspace_bytes, stream, opts, kPhaseAdapter);
}

extern "C" qlora_status qlora_linear_bwd(const qlora_nf4_weight *w, const void *X, const void *dY, int64_t M,
                                         const void *A, const void *B, int32_t r, float scale,
                                         const float *H_saved, void *dX, qlora_dtype dx_dtype, float *dA, float *dB,
                                         void *workspace, size_t workspace_bytes, void *stream)
{
    return qlora_linear_bwd_ex(w, X, dY, M, A, B, r, scale, H_saved, dX, dx_dtype, dA, dB, workspace, workspace_bytes,
                               stream, nullptr);
}
