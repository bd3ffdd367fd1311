// One QLoRA transformer block on sm_100a, forward and backward, with
// gradient checkpointing.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs", Introduction: LoRA
// adapters at every network layer; gradient checkpointing (activations are
// recomputed instead of stored, and the paged optimizer absorbs the memory
// spikes).  The pages give the seven linear shapes of the LLaMA models they
// finetune but not the rest of the block; it follows the LLaMA decoder layer:
//     u1 = RMSNorm(x; g1); q, k, v = Lq(u1), Lk(u1), Lv(u1); RoPE(q), RoPE(k)
//     a = causal softmax(q k^T / sqrt(D)) v;   h = x + Lo(a)
//     u2 = RMSNorm(h; g2); y = h + Ldown(silu(Lgate(u2)) * Lup(u2))
// Every L is the library's QLoRA linear (frozen NF4 + DQ weight, trainable
// adapters); the norm weights are frozen.
//
// Checkpointing: qlora_block_fwd keeps nothing but its output; the backward
// pass recomputes the forward from the block input (saving H of each linear
// and the attention probabilities on the way), then runs the chain rule.
// Attention is computed with batched tensor-core products over (sequence,
// head) pairs with the probabilities materialized in bf16, skipping the
// products above the causal diagonal.
#include <cuda_bf16.h>
#include <math.h>

#include "block_kernels.cuh"
#include "common.cuh"

namespace qlora {
namespace {

constexpr int kL = 7;   // q, k, v, o, gate, up, down
enum { Lq = 0, Lk, Lv, Lo, Lgate, Lup, Ldown };

size_t al(size_t v) { return (v + 255) / 256 * 256; }

struct BlockLayout {
    int64_t T, d, I, Z, S;
    size_t u1, q, k, v, a, ao, h, u2, gt, up, m, rstd1, rstd2, hs[kL], sc, P, rope;
    size_t dm, dgt, dup, dxg, dxu, dh, da, dq, dk, dv, dxq, dxk, dxv, lin, lin_bytes, bytes;
};

int64_t in_features(const qlora_block *b, int l) { return b->w[l].cols; }
int64_t out_features(const qlora_block *b, int l) { return b->w[l].rows; }

BlockLayout layout(const qlora_block *b)
{
    BlockLayout L{};
    L.T = (int64_t)b->batch * b->seq;
    L.d = b->hidden;
    L.I = b->inter;
    L.S = b->seq;
    L.Z = (int64_t)b->batch * b->heads;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += al(bytes);
        return o;
    };
    const size_t td = (size_t)L.T * L.d * 2, ti = (size_t)L.T * L.I * 2;
    L.u1 = take(td);
    L.q = take(td);
    L.k = take(td);
    L.v = take(td);
    L.a = take(td);
    L.ao = take(td);
    L.h = take(td);
    L.u2 = take(td);
    L.gt = take(ti);
    L.up = take(ti);
    L.m = take(ti);
    L.rstd1 = take((size_t)L.T * 4);
    L.rstd2 = take((size_t)L.T * 4);
    for (int l = 0; l < kL; l++) L.hs[l] = take((size_t)L.T * b->r * 4);
    L.sc = take((size_t)L.Z * L.S * L.S * 4);
    L.P = take((size_t)L.Z * L.S * L.S * 2);
    L.rope = take((size_t)L.S * (b->head_dim / 2) * 8);
    L.dm = take(ti);
    L.dgt = take(ti);
    L.dup = take(ti);
    L.dxg = take(td);
    L.dxu = take(td);
    L.dh = take(td);
    L.da = take(td);
    L.dq = take(td);
    L.dk = take(td);
    L.dv = take(td);
    L.dxq = take(td);
    L.dxk = take(td);
    L.dxv = take(td);
    size_t lin = 0;
    for (int l = 0; l < kL; l++) {
        const size_t n = qlora_linear_workspace_bytes(L.T, out_features(b, l), in_features(b, l), b->r);
        lin = n > lin ? n : lin;
    }
    L.lin_bytes = lin;
    L.lin = take(lin);
    L.bytes = off;
    return L;
}

qlora_status check_block(const qlora_block *b)
{
    if (!b) return QLORA_ERR_INVALID_ARG;
    if (b->batch < 1 || b->seq < 1 || b->heads < 1 || b->head_dim < 8 || b->hidden < 8 || b->inter < 8)
        return QLORA_ERR_SHAPE;
    if (b->head_dim % 16 || b->hidden % 64 || b->inter % 64 || b->seq % 8) return QLORA_ERR_SHAPE;
    if ((int64_t)b->heads * b->head_dim != b->hidden) return QLORA_ERR_SHAPE;
    const int64_t want[kL][2] = {{b->hidden, b->hidden}, {b->hidden, b->hidden}, {b->hidden, b->hidden},
                                 {b->hidden, b->hidden}, {b->inter, b->hidden}, {b->inter, b->hidden},
                                 {b->hidden, b->inter}};
    for (int l = 0; l < kL; l++) {
        if (b->w[l].rows != want[l][0] || b->w[l].cols != want[l][1]) return QLORA_ERR_SHAPE;
        if (!b->A[l] || !b->B[l]) return QLORA_ERR_INVALID_ARG;
    }
    if (!b->norm1 || !b->norm2) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(b->norm1) || !aligned16(b->norm2)) return QLORA_ERR_ALIGNMENT;
    if (!(b->rms_eps >= 0.0f) || !(b->rope_base > 1.0f)) return QLORA_ERR_INVALID_ARG;
    return QLORA_OK;
}

using bf16 = __nv_bfloat16;

struct Ctx {
    const qlora_block *b;
    BlockLayout L;
    char *ws;
    cudaStream_t s;
    int sms;
    template <typename T = bf16>
    T *at(size_t off) const { return reinterpret_cast<T *>(ws + off); }
};

int grid_for(int64_t n, int sms) { return (int)std::min<int64_t>((n + 255) / 256, (int64_t)sms * 16); }

qlora_status lin_fwd(const Ctx &c, int l, const void *X, void *Y, float *H)
{
    return qlora_linear_fwd(&c.b->w[l], X, c.L.T, c.b->A[l], c.b->B[l], c.b->r, c.b->lora_scale, Y, QLORA_BF16, H,
                            c.ws + c.L.lin, c.L.lin_bytes, c.s);
}

qlora_status lin_bwd(const Ctx &c, int l, const void *X, const void *dY, const float *H, void *dX, float *dA,
                     float *dB)
{
    return qlora_linear_bwd(&c.b->w[l], X, dY, c.L.T, c.b->A[l], c.b->B[l], c.b->r, c.b->lora_scale, H, dX, QLORA_BF16,
                            dA, dB, c.ws + c.L.lin, c.L.lin_bytes, c.s);
}

template <bool AT, bool BT, bool F32>
qlora_status bmm(const Ctx &c, blk::BmmArgs a, int kind)
{
    dim3 grid((unsigned)((a.N + blk::kBN - 1) / blk::kBN), (unsigned)((a.M + blk::kBM - 1) / blk::kBM),
              (unsigned)c.L.Z);
    LaunchScope ls(kind, c.s);
    QLORA_CUDA_TRY(launch_pdl(blk::bmm_kernel<AT, BT, F32>, grid, dim3(256), 0, c.s, a));
    return QLORA_OK;
}

// elements of a [T][hidden] activation and of the [Z][S][S] score buffers
// (the extents the bounds-checked build checks attention operands against)
int64_t act_elems(const Ctx &c) { return c.L.T * c.L.d; }
int64_t score_elems(const Ctx &c) { return c.L.Z * c.L.S * c.L.S; }

// batch strides of a [T][hidden] activation viewed as (sequence, head) tiles
void act_view(const Ctx &c, int64_t &ld, int64_t &s0, int64_t &s1)
{
    ld = c.L.d;
    s0 = c.L.S * c.L.d;
    s1 = c.b->head_dim;
}

// attention scores / probabilities [Z][S][S]: (sequence, head) = (z0, z1)
void score_view(const Ctx &c, int64_t &ld, int64_t &s0, int64_t &s1)
{
    ld = c.L.S;
    s1 = c.L.S * c.L.S;
    s0 = (int64_t)c.b->heads * s1;
}

// The forward pass; with `save`, what the backward pass reads is kept in the
// workspace (H of every linear but the last, the attention probabilities) and
// the last linear is skipped.
qlora_status forward(const Ctx &c, const bf16 *x, bf16 *y, bool save)
{
    const qlora_block *b = c.b;
    const BlockLayout &L = c.L;
    float *hs[kL];
    for (int l = 0; l < kL; l++) hs[l] = save ? c.at<float>(L.hs[l]) : nullptr;
    {
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        QLORA_CUDA_TRY(launch_pdl(blk::rmsnorm_fwd_kernel, dim3((unsigned)L.T), dim3(256), 0, c.s, x, (const bf16 *)nullptr,
                                  (bf16 *)nullptr, (const bf16 *)b->norm1, (int)L.d, b->rms_eps, c.at(L.u1),
                                  c.at<float>(L.rstd1)));
    }
    QLORA_TRY(lin_fwd(c, Lq, c.at(L.u1), c.at(L.q), hs[Lq]));
    QLORA_TRY(lin_fwd(c, Lk, c.at(L.u1), c.at(L.k), hs[Lk]));
    QLORA_TRY(lin_fwd(c, Lv, c.at(L.u1), c.at(L.v), hs[Lv]));
    const float log2b = log2f(b->rope_base);
    const int64_t groups = L.T * b->heads * (b->head_dim / 16);
    const float2 *cs = c.at<float2>(L.rope);
    {
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        const int entries = (int)(L.S * (b->head_dim / 2));
        QLORA_CUDA_TRY(launch_pdl(blk::rope_table_kernel, dim3((entries + 255) / 256), dim3(256), 0, c.s,
                                  c.at<float2>(L.rope), (int)L.S, b->head_dim, log2b));
        QLORA_CUDA_TRY(launch_pdl(blk::rope_kernel, dim3(grid_for(groups, c.sms)), dim3(256), 0, c.s, c.at(L.q), cs,
                                  L.T, b->seq, b->heads, b->head_dim, 1.0f));
        QLORA_CUDA_TRY(launch_pdl(blk::rope_kernel, dim3(grid_for(groups, c.sms)), dim3(256), 0, c.s, c.at(L.k), cs,
                                  L.T, b->seq, b->heads, b->head_dim, 1.0f));
    }
    int64_t ald, as0, as1, sld, ss0, ss1;
    act_view(c, ald, as0, as1);
    score_view(c, sld, ss0, ss1);
    {
        // scores = q k^T / sqrt(D), causal
        blk::BmmArgs a{};
        a.A = c.at(L.q);
        a.a_n = act_elems(c);
        a.B = c.at(L.k);
        a.b_n = act_elems(c);
        a.C = c.at<float>(L.sc);
        a.c_n = score_elems(c);
        a.M = (int)L.S; a.N = (int)L.S; a.K = b->head_dim;
        a.lda = ald; a.sa0 = as0; a.sa1 = as1;
        a.ldb = ald; a.sb0 = as0; a.sb1 = as1;
        a.ldc = sld; a.sc0 = ss0; a.sc1 = ss1;
        a.nz1 = b->heads;
        a.alpha = 1.0f / sqrtf((float)b->head_dim);
        a.causal = 1;
        QLORA_TRY((bmm<false, true, true>(c, a, QLORA_KERNEL_ATTENTION)));
    }
    {
        LaunchScope ls(QLORA_KERNEL_ATTENTION, c.s);
        const int64_t rows = L.Z * L.S;
        QLORA_CUDA_TRY(launch_pdl(blk::softmax_rows_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, c.s,
                                  (const float *)c.at<float>(L.sc), c.at(L.P), rows, (int)L.S));
    }
    {
        // a = P v (P is zero above the diagonal)
        blk::BmmArgs a{};
        a.A = c.at(L.P);
        a.a_n = score_elems(c);
        a.B = c.at(L.v);
        a.b_n = act_elems(c);
        a.C = c.at(L.a);
        a.c_n = act_elems(c);
        a.M = (int)L.S; a.N = b->head_dim; a.K = (int)L.S;
        a.lda = sld; a.sa0 = ss0; a.sa1 = ss1;
        a.ldb = ald; a.sb0 = as0; a.sb1 = as1;
        a.ldc = ald; a.sc0 = as0; a.sc1 = as1;
        a.nz1 = b->heads;
        a.alpha = 1.0f;
        a.tri = 1;
        QLORA_TRY((bmm<false, false, false>(c, a, QLORA_KERNEL_ATTENTION)));
    }
    QLORA_TRY(lin_fwd(c, Lo, c.at(L.a), c.at(L.ao), hs[Lo]));
    {
        // h = x + o(a); u2 = RMSNorm(h)
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        QLORA_CUDA_TRY(launch_pdl(blk::rmsnorm_fwd_kernel, dim3((unsigned)L.T), dim3(256), 0, c.s, x,
                                  (const bf16 *)c.at(L.ao), c.at(L.h), (const bf16 *)b->norm2, (int)L.d, b->rms_eps,
                                  c.at(L.u2), c.at<float>(L.rstd2)));
    }
    QLORA_TRY(lin_fwd(c, Lgate, c.at(L.u2), c.at(L.gt), hs[Lgate]));
    QLORA_TRY(lin_fwd(c, Lup, c.at(L.u2), c.at(L.up), hs[Lup]));
    {
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        QLORA_CUDA_TRY(launch_pdl(blk::swiglu_fwd_kernel, dim3(grid_for(L.T * L.I / 8, c.sms)), dim3(256), 0, c.s,
                                  (const bf16 *)c.at(L.gt), (const bf16 *)c.at(L.up), c.at(L.m), L.T * L.I));
    }
    if (save) return launch_status();
    // y = h + down(m): the residual add rides on an RMSNorm launch whose
    // normalized output is discarded into the (free) u1 buffer
    QLORA_TRY(lin_fwd(c, Ldown, c.at(L.m), c.at(L.ao), nullptr));
    {
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        QLORA_CUDA_TRY(launch_pdl(blk::rmsnorm_fwd_kernel, dim3((unsigned)L.T), dim3(256), 0, c.s,
                                  (const bf16 *)c.at(L.h), (const bf16 *)c.at(L.ao), y, (const bf16 *)b->norm2,
                                  (int)L.d, b->rms_eps, c.at(L.u1), (float *)nullptr));
    }
    return launch_status();
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" size_t qlora_block_workspace_bytes(const qlora_block *b)
{
    if (check_block(b) != QLORA_OK) return 0;
    return layout(b).bytes;
}

extern "C" qlora_status qlora_block_fwd(const qlora_block *b, const void *x, void *y, void *workspace,
                                        size_t workspace_bytes, void *stream)
{
    QLORA_TRY(check_block(b));
    if (!x || !y || !workspace) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(workspace)) return QLORA_ERR_ALIGNMENT;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    Ctx c{b, layout(b), static_cast<char *>(workspace), static_cast<cudaStream_t>(stream), dev.sms};
    if (workspace_bytes < c.L.bytes) return QLORA_ERR_WORKSPACE;
    return forward(c, static_cast<const bf16 *>(x), static_cast<bf16 *>(y), false);
}

extern "C" qlora_status qlora_block_bwd(const qlora_block *b, const void *x, const void *dy, void *dx,
                                        float *const dA[7], float *const dB[7], void *workspace,
                                        size_t workspace_bytes, void *stream)
{
    QLORA_TRY(check_block(b));
    if (!x || !dy || !dx || !dA || !dB || !workspace) return QLORA_ERR_INVALID_ARG;
    for (int l = 0; l < kL; l++)
        if (!dA[l] || !dB[l]) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || !aligned16(workspace)) return QLORA_ERR_ALIGNMENT;
    DeviceInfo dev;
    QLORA_TRY(device_info(&dev));
    Ctx c{b, layout(b), static_cast<char *>(workspace), static_cast<cudaStream_t>(stream), dev.sms};
    if (workspace_bytes < c.L.bytes) return QLORA_ERR_WORKSPACE;
    const BlockLayout &L = c.L;
    const bf16 *xb = static_cast<const bf16 *>(x);
    const bf16 *dyb = static_cast<const bf16 *>(dy);

    // 1. recompute the forward pass (checkpointing)
    QLORA_TRY(forward(c, xb, nullptr, true));

    // 2. MLP: down, SwiGLU, gate/up, second norm (+ residual)
    QLORA_TRY(lin_bwd(c, Ldown, c.at(L.m), dyb, nullptr, c.at(L.dm), dA[Ldown], dB[Ldown]));
    {
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        QLORA_CUDA_TRY(launch_pdl(blk::swiglu_bwd_kernel, dim3(grid_for(L.T * L.I / 8, c.sms)), dim3(256), 0, c.s,
                                  (const bf16 *)c.at(L.dm), (const bf16 *)c.at(L.gt), (const bf16 *)c.at(L.up),
                                  c.at(L.dgt), c.at(L.dup), L.T * L.I));
    }
    QLORA_TRY(lin_bwd(c, Lgate, c.at(L.u2), c.at(L.dgt), c.at<float>(L.hs[Lgate]), c.at(L.dxg), dA[Lgate], dB[Lgate]));
    QLORA_TRY(lin_bwd(c, Lup, c.at(L.u2), c.at(L.dup), c.at<float>(L.hs[Lup]), c.at(L.dxu), dA[Lup], dB[Lup]));
    {
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        QLORA_CUDA_TRY(launch_pdl(blk::rmsnorm_bwd_kernel, dim3((unsigned)L.T), dim3(256), 0, c.s,
                                  (const bf16 *)c.at(L.h), (const bf16 *)b->norm2, (const float *)c.at<float>(L.rstd2),
                                  (const bf16 *)c.at(L.dxg), (const bf16 *)c.at(L.dxu), (const bf16 *)nullptr, dyb,
                                  (int)L.d, c.at(L.dh)));
    }

    // 3. attention: o, then the softmax products, then RoPE^-1
    QLORA_TRY(lin_bwd(c, Lo, c.at(L.a), c.at(L.dh), c.at<float>(L.hs[Lo]), c.at(L.da), dA[Lo], dB[Lo]));
    int64_t ald, as0, as1, sld, ss0, ss1;
    act_view(c, ald, as0, as1);
    score_view(c, sld, ss0, ss1);
    {
        // dv = P^T da (row i of P^T, key i, is non-zero only for queries i and later)
        blk::BmmArgs a{};
        a.A = c.at(L.P);
        a.a_n = score_elems(c);
        a.B = c.at(L.da);
        a.b_n = act_elems(c);
        a.C = c.at(L.dv);
        a.c_n = act_elems(c);
        a.M = (int)L.S; a.N = b->head_dim; a.K = (int)L.S;
        a.lda = sld; a.sa0 = ss0; a.sa1 = ss1;
        a.ldb = ald; a.sb0 = as0; a.sb1 = as1;
        a.ldc = ald; a.sc0 = as0; a.sc1 = as1;
        a.nz1 = b->heads;
        a.alpha = 1.0f;
        a.tri = 2;
        QLORA_TRY((bmm<true, false, false>(c, a, QLORA_KERNEL_ATTENTION)));
    }
    {
        // dP = da v^T (the scores buffer)
        blk::BmmArgs a{};
        a.A = c.at(L.da);
        a.a_n = act_elems(c);
        a.B = c.at(L.v);
        a.b_n = act_elems(c);
        a.C = c.at<float>(L.sc);
        a.c_n = score_elems(c);
        a.M = (int)L.S; a.N = (int)L.S; a.K = b->head_dim;
        a.lda = ald; a.sa0 = as0; a.sa1 = as1;
        a.ldb = ald; a.sb0 = as0; a.sb1 = as1;
        a.ldc = sld; a.sc0 = ss0; a.sc1 = ss1;
        a.nz1 = b->heads;
        a.alpha = 1.0f;
        QLORA_TRY((bmm<false, true, true>(c, a, QLORA_KERNEL_ATTENTION)));
    }
    {
        // dS = P (dP - rowsum(P dP)) / sqrt(D), written over P
        LaunchScope ls(QLORA_KERNEL_ATTENTION, c.s);
        const int64_t rows = L.Z * L.S;
        QLORA_CUDA_TRY(launch_pdl(blk::dsoftmax_rows_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, c.s,
                                  (const bf16 *)c.at(L.P), (const float *)c.at<float>(L.sc), c.at(L.P), rows, (int)L.S,
                                  1.0f / sqrtf((float)b->head_dim)));
    }
    {
        // dq = dS k
        blk::BmmArgs a{};
        a.A = c.at(L.P);
        a.a_n = score_elems(c);
        a.B = c.at(L.k);
        a.b_n = act_elems(c);
        a.C = c.at(L.dq);
        a.c_n = act_elems(c);
        a.M = (int)L.S; a.N = b->head_dim; a.K = (int)L.S;
        a.lda = sld; a.sa0 = ss0; a.sa1 = ss1;
        a.ldb = ald; a.sb0 = as0; a.sb1 = as1;
        a.ldc = ald; a.sc0 = as0; a.sc1 = as1;
        a.nz1 = b->heads;
        a.alpha = 1.0f;
        a.tri = 1;
        QLORA_TRY((bmm<false, false, false>(c, a, QLORA_KERNEL_ATTENTION)));
        // dk = dS^T q
        a.B = c.at(L.q);
        a.b_n = act_elems(c);
        a.C = c.at(L.dk);
        a.c_n = act_elems(c);
        a.tri = 2;
        QLORA_TRY((bmm<true, false, false>(c, a, QLORA_KERNEL_ATTENTION)));
    }
    const int64_t groups = L.T * b->heads * (b->head_dim / 16);
    const float2 *cs = c.at<float2>(L.rope);   // written by the recomputed forward pass
    {
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        QLORA_CUDA_TRY(launch_pdl(blk::rope_kernel, dim3(grid_for(groups, c.sms)), dim3(256), 0, c.s, c.at(L.dq), cs,
                                  L.T, b->seq, b->heads, b->head_dim, -1.0f));
        QLORA_CUDA_TRY(launch_pdl(blk::rope_kernel, dim3(grid_for(groups, c.sms)), dim3(256), 0, c.s, c.at(L.dk), cs,
                                  L.T, b->seq, b->heads, b->head_dim, -1.0f));
    }

    // 4. q, k, v, first norm (+ residual)
    QLORA_TRY(lin_bwd(c, Lq, c.at(L.u1), c.at(L.dq), c.at<float>(L.hs[Lq]), c.at(L.dxq), dA[Lq], dB[Lq]));
    QLORA_TRY(lin_bwd(c, Lk, c.at(L.u1), c.at(L.dk), c.at<float>(L.hs[Lk]), c.at(L.dxk), dA[Lk], dB[Lk]));
    QLORA_TRY(lin_bwd(c, Lv, c.at(L.u1), c.at(L.dv), c.at<float>(L.hs[Lv]), c.at(L.dxv), dA[Lv], dB[Lv]));
    {
        LaunchScope ls(QLORA_KERNEL_BLOCK, c.s);
        QLORA_CUDA_TRY(launch_pdl(blk::rmsnorm_bwd_kernel, dim3((unsigned)L.T), dim3(256), 0, c.s, xb,
                                  (const bf16 *)b->norm1, (const float *)c.at<float>(L.rstd1),
                                  (const bf16 *)c.at(L.dxq), (const bf16 *)c.at(L.dxk), (const bf16 *)c.at(L.dxv),
                                  (const bf16 *)c.at(L.dh), (int)L.d, static_cast<bf16 *>(dx)));
    }
    return launch_status();
}
