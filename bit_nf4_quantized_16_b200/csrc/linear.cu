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

#include "common.cuh"
#include "gemm.cuh"

namespace qlora {
namespace {

constexpr uint64_t kTimeoutNs = 2000000000ull;   // bounded waits give up after 2 s

// ---- tensor maps -----------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D row-major tensor: `inner` elements per row (contiguous), `rows` rows,
// `pitch_bytes` between rows; box = box_inner x box_rows elements.
qlora_status make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw)
{
    auto fn = encode_fn();
    if (!fn) return QLORA_ERR_CUDA;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status map_bf16(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t ld,
                      uint32_t box_inner, uint32_t box_rows)
{
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, rows, ld * 2, box_inner, box_rows,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

// ---- GEMM launch ------------------------------------------------------------------

template <int BN, int kBMode, int kEpi, int MT = 1>
qlora_status launch_gemm(GemmParams &p, const DeviceInfo &dev, cudaStream_t s, int kind)
{
    using Cfg = GemmCfg<BN, kBMode, MT>;
    static bool attr_done[64] = {};
    auto kern = qgemm_kernel<BN, kBMode, kEpi, MT>;
    if (!attr_done[dev.device]) {
        QLORA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
        attr_done[dev.device] = true;
    }
    p.err = device_error_word();
    if (!p.err) return QLORA_ERR_CUDA;
    p.timeout_ns = kTimeoutNs;
    const int tiles = p.m_tiles * p.n_tiles * p.splits;
    const int grid = tiles < dev.sms ? tiles : dev.sms;
    {
        LaunchScope ls(kind, s);
        kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, s>>>(p);
    }
    return launch_status();
}

// number of splits of a contraction of `total` 64-deep steps over `tiles`
// output tiles, aiming at about one wave of the GPU; every split non-empty
void choose_splits(int tiles, int total, int sms, int min_per_split, int *splits, int *per)
{
    int sp = (sms + tiles - 1) / tiles;
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

// ---- small elementwise kernels ----------------------------------------------------

__device__ __forceinline__ void store_hi_lo(__nv_bfloat16 *h2, int64_t m, int r, int j, float v)
{
    __nv_bfloat16 hi = __float2bfloat16_rn(v);
    __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
    h2[m * 2 * r + j] = hi;
    h2[m * 2 * r + r + j] = lo;
}

// v[m][j] = scale * sum_s part[s][m][j] (splits in order); writes the hi/lo
// pair and optionally the fp32 value.
__global__ void finalize_lowrank_kernel(const float *part, int splits, int64_t split_stride, int ld, int64_t M,
                                        int r, float scale, float *out_f32, __nv_bfloat16 *out_hi_lo)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= M * r) return;
    int64_t m = i / r;
    int j = (int)(i % r);
    float acc = 0.0f;
    for (int s = 0; s < splits; s++) acc = __fadd_rn(acc, part[s * split_stride + m * ld + j]);
    float v = __fmul_rn(scale, acc);
    if (out_f32) out_f32[m * r + j] = v;
    store_hi_lo(out_hi_lo, m, r, j, v);
}

__global__ void split_hi_lo_kernel(const float *h, int64_t M, int r, __nv_bfloat16 *out_hi_lo)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= M * r) return;
    store_hi_lo(out_hi_lo, i / r, r, (int)(i % r), h[i]);
}

// out[a][b] = sum_s part[s][a][b] + sum_s part[s][a + da][b + db]: the hi and
// lo halves of a weight-gradient product, added in a fixed order.
__global__ void finalize_wgrad_kernel(const float *part, int splits, int64_t split_stride, int64_t ld, int64_t rows,
                                      int64_t cols, int64_t da, int64_t db, float *out)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * cols) return;
    int64_t a = i / cols, b = i % cols;
    float hi = 0.0f, lo = 0.0f;
    for (int s = 0; s < splits; s++) {
        hi = __fadd_rn(hi, part[s * split_stride + a * ld + b]);
        lo = __fadd_rn(lo, part[s * split_stride + (a + da) * ld + b + db]);
    }
    out[i] = __fadd_rn(hi, lo);
}

int elementwise_grid(int64_t n) { return (int)((n + 255) / 256); }

// ---- problem plan -------------------------------------------------------------------

struct Plan {
    int64_t M, N, K;
    int r, r_pad;
    // H = X A^T : tiles over M, split over K
    int h_splits, h_per;
    // G = dY B  : tiles over M, split over N
    int g_splits, g_per;
    // dA = G2^T X : tiles (2r rows) x (K / 128), split over M
    int da_splits, da_per, da_mtiles;
    // dB = dY^T H2 : tiles (N / 128) x 1, split over M
    int db_splits, db_per, db_bn;
    // workspace offsets
    size_t off_h2, off_g2, off_part, bytes;
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
    const int mt = ceil_div(M, 128);
    choose_splits(mt, ceil_div(K, 64), sms, 4, &pl.h_splits, &pl.h_per);
    choose_splits(mt, ceil_div(N, 64), sms, 4, &pl.g_splits, &pl.g_per);
    pl.da_mtiles = ceil_div(2 * r, 128);
    choose_splits(pl.da_mtiles * ceil_div(K, 128), ceil_div(M, 64), sms, 4, &pl.da_splits, &pl.da_per);
    pl.db_bn = 2 * r <= 64 ? 64 : (2 * r <= 128 ? 128 : 256);
    choose_splits(ceil_div(N, 128), ceil_div(M, 64), sms, 4, &pl.db_splits, &pl.db_per);
    size_t hl = align256((size_t)M * 2 * r * 2);
    size_t part = 0;
    part = std::max(part, (size_t)pl.h_splits * M * pl.r_pad * 4);
    part = std::max(part, (size_t)pl.g_splits * M * pl.r_pad * 4);
    part = std::max(part, (size_t)pl.da_splits * 2 * r * K * 4);
    part = std::max(part, (size_t)pl.db_splits * N * 2 * r * 4);
    pl.off_h2 = 0;
    pl.off_g2 = hl;
    pl.off_part = 2 * hl;
    pl.bytes = 2 * hl + align256(part);
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

// H = s X A^T into the hi/lo workspace buffer (and optionally fp32 H_out)
qlora_status run_h(const Plan &pl, const DeviceInfo &dev, const void *X, const void *A, float scale, float *H_out,
                   char *ws, cudaStream_t s)
{
    GemmParams p{};
    QLORA_TRY(map_bf16(&p.tm_a, X, pl.K, pl.M, pl.K, 64, 128));
    QLORA_TRY(map_bf16(&p.tm_b, A, pl.K, pl.r, pl.K, 64, pl.r_pad));
    p.m_tiles = ceil_div(pl.M, 128);
    p.n_tiles = 1;
    p.splits = pl.h_splits;
    p.k_stages_total = ceil_div(pl.K, 64);
    p.k_stages_split = pl.h_per;
    p.out = ws + pl.off_part;
    p.out_ld = pl.r_pad;
    p.split_stride = pl.M * pl.r_pad;
    p.m_total = (int)pl.M;
    p.n_total = pl.r_pad;
    if (pl.r_pad == 64)
        QLORA_TRY((launch_gemm<64, kBTmaK, kEpiF32>(p, dev, s, QLORA_KERNEL_LOWRANK)));
    else
        QLORA_TRY((launch_gemm<128, kBTmaK, kEpiF32>(p, dev, s, QLORA_KERNEL_LOWRANK)));
    {
        LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
        finalize_lowrank_kernel<<<elementwise_grid(pl.M * pl.r), 256, 0, s>>>(
            reinterpret_cast<const float *>(ws + pl.off_part), pl.h_splits, pl.M * pl.r_pad, pl.r_pad, pl.M, pl.r,
            scale, H_out, reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_h2));
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

    QLORA_TRY(run_h(pl, dev, X, A, scale, H_save, ws, s));

    // fused forward: 256 tokens (two 128-row accumulators) x 128 output features per tile
    constexpr int kFBN = 128, kFMT = 2;
    GemmParams p{};
    QLORA_TRY(map_bf16(&p.tm_a, X, pl.K, M, pl.K, 64, 128 * kFMT));
    QLORA_TRY(make_map(&p.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, pl.K / 2, pl.N, pl.K / 2, 32, kFBN,
                       CU_TENSOR_MAP_SWIZZLE_32B));
    QLORA_TRY(map_bf16(&p.tm_a2, ws + pl.off_h2, r, M, 2 * r, 64, 128 * kFMT));   // hi half of H
    QLORA_TRY(map_bf16(&p.tm_b2, B, r, pl.N, r, 64, kFBN));
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
    p.k_stages_lora = ceil_div(r, 64);
    p.out = Y;
    p.out_ld = pl.N;
    p.m_total = (int)M;
    p.n_total = (int)pl.N;
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
    float *part = reinterpret_cast<float *>(ws + pl.off_part);

    // H (hi/lo) from the saved fp32 H, or recomputed
    if (H_saved) {
        {
            LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
            split_hi_lo_kernel<<<elementwise_grid(M * r), 256, 0, s>>>(H_saved, M, r, H2);
        }
        QLORA_TRY(launch_status());
    } else {
        QLORA_TRY(run_h(pl, dev, X, A, scale, nullptr, ws, s));
    }

    // G = s dY B  (contraction over N)
    {
        GemmParams p{};
        QLORA_TRY(map_bf16(&p.tm_a, dY, N, M, N, 64, 128));
        QLORA_TRY(map_bf16(&p.tm_b, B, r, N, r, 64, 64));      // B[n][j]: MN-major operand
        p.m_tiles = ceil_div(M, 128);
        p.n_tiles = 1;
        p.splits = pl.g_splits;
        p.k_stages_total = ceil_div(N, 64);
        p.k_stages_split = pl.g_per;
        p.out = part;
        p.out_ld = pl.r_pad;
        p.split_stride = M * pl.r_pad;
        p.m_total = (int)M;
        p.n_total = pl.r_pad;
        if (pl.r_pad == 64)
            QLORA_TRY((launch_gemm<64, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_LOWRANK)));
        else
            QLORA_TRY((launch_gemm<128, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_LOWRANK)));
        {
            LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
            finalize_lowrank_kernel<<<elementwise_grid(M * r), 256, 0, s>>>(part, pl.g_splits, M * pl.r_pad, pl.r_pad,
                                                                             M, r, scale, nullptr, G2);
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
        QLORA_TRY(map_bf16(&p.tm_a2, G2, r, M, 2 * r, 64, 128 * kBMT));   // hi half of G
        QLORA_TRY(map_bf16(&p.tm_b2, A, K, r, K, 64, 64));                // A[j][k]: MN-major operand
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
        p.k_stages_lora = ceil_div(r, 64);
        p.out = dX;
        p.out_ld = K;
        p.m_total = (int)M;
        p.n_total = (int)K;
        if (dx_dtype == QLORA_BF16)
            QLORA_TRY((launch_gemm<kBBN, kBNf4MN, kEpiBf16, kBMT>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
        else
            QLORA_TRY((launch_gemm<kBBN, kBNf4MN, kEpiF32, kBMT>(p, dev, s, QLORA_KERNEL_BWD_FUSED)));
    }

    // dA = G^T X  (rows j of [G_hi | G_lo], contraction over tokens)
    {
        GemmParams p{};
        QLORA_TRY(map_bf16(&p.tm_a, G2, 2 * r, M, 2 * r, 64, 64));   // MN-major A
        QLORA_TRY(map_bf16(&p.tm_b, X, K, M, K, 64, 64));            // MN-major B
        p.a_mn = 1;
        p.m_tiles = pl.da_mtiles;
        p.n_tiles = ceil_div(K, 128);
        p.splits = pl.da_splits;
        p.k_stages_total = ceil_div(M, 64);
        p.k_stages_split = pl.da_per;
        p.out = part;
        p.out_ld = K;
        p.split_stride = 2 * r * K;
        p.m_total = 2 * r;
        p.n_total = (int)K;
        QLORA_TRY((launch_gemm<128, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_WGRAD)));
        {
            LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
            finalize_wgrad_kernel<<<elementwise_grid((int64_t)r * K), 256, 0, s>>>(part, pl.da_splits, 2 * r * K, K, r,
                                                                                   K, r, 0, dA);
        }
        QLORA_TRY(launch_status());
    }

    // dB = dY^T H  (rows n, columns [H_hi | H_lo], contraction over tokens)
    {
        GemmParams p{};
        QLORA_TRY(map_bf16(&p.tm_a, dY, N, M, N, 64, 64));           // MN-major A
        QLORA_TRY(map_bf16(&p.tm_b, H2, 2 * r, M, 2 * r, 64, 64));   // MN-major B
        p.a_mn = 1;
        p.m_tiles = ceil_div(N, 128);
        p.n_tiles = 1;
        p.splits = pl.db_splits;
        p.k_stages_total = ceil_div(M, 64);
        p.k_stages_split = pl.db_per;
        p.out = part;
        p.out_ld = 2 * r;
        p.split_stride = N * 2 * r;
        p.m_total = (int)N;
        p.n_total = 2 * r;
        if (pl.db_bn == 64)
            QLORA_TRY((launch_gemm<64, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_WGRAD)));
        else if (pl.db_bn == 128)
            QLORA_TRY((launch_gemm<128, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_WGRAD)));
        else
            QLORA_TRY((launch_gemm<256, kBTmaMN, kEpiF32>(p, dev, s, QLORA_KERNEL_WGRAD)));
        {
            LaunchScope ls(QLORA_KERNEL_ELEMENTWISE, s);
            finalize_wgrad_kernel<<<elementwise_grid(N * r), 256, 0, s>>>(part, pl.db_splits, N * 2 * r, 2 * r, N, r,
                                                                           0, r, dB);
        }
        return launch_status();
    }
}
