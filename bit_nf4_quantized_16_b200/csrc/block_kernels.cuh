// Kernels of the transformer block around the seven QLoRA linears (sm_100a):
// RMSNorm forward/backward, rotary position embedding, SwiGLU, and causal
// attention built from batched bf16 tensor-core products plus row-wise
// softmax kernels.  See block.cu for the layer they belong to.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100.cuh"
#include "debug.cuh"

namespace qlora {
namespace blk {

__device__ __forceinline__ float bf(const __nv_bfloat16 v) { return __bfloat162float(v); }

// ---- RMSNorm ------------------------------------------------------------------
// u = bf16(x * rstd * g), rstd = 1 / sqrt(mean(x^2) + eps); with `res`, x is
// first formed as bf16(xin + res) and written to x_out (the residual add).
// One CTA of 256 threads per row; d % 8 == 0.
__global__ void __launch_bounds__(256) rmsnorm_fwd_kernel(const __nv_bfloat16 *xin, const __nv_bfloat16 *res,
                                                          __nv_bfloat16 *x_out, const __nv_bfloat16 *g, int d,
                                                          float eps, __nv_bfloat16 *u, float *rstd_out)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int64_t row = blockIdx.x;
    const __nv_bfloat16 *xr = xin + row * d;
    __shared__ float red[8];
    float ss = 0.0f;
    for (int c = threadIdx.x * 8; c < d; c += 256 * 8) {
        if (!QLORA_IN(c + 7, d)) break;
        uint4 xv = *reinterpret_cast<const uint4 *>(xr + c);
        if (res) {
            const uint4 rv = *reinterpret_cast<const uint4 *>(res + row * d + c);
            const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(&xv);
            const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&rv);
            uint4 sv;
            __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(&sv);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float2 fa = __bfloat1622float2(a[i]), fb = __bfloat1622float2(b[i]);
                o[i] = __floats2bfloat162_rn(__fadd_rn(fa.x, fb.x), __fadd_rn(fa.y, fb.y));
            }
            *reinterpret_cast<uint4 *>(x_out + row * d + c) = sv;
            xv = sv;
        }
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&xv);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 f = __bfloat1622float2(h[i]);
            ss = __fmaf_rn(f.x, f.x, ss);
            ss = __fmaf_rn(f.y, f.y, ss);
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; w++) tot += red[w];
    const float rstd = rsqrtf(tot / (float)d + eps);
    if (threadIdx.x == 0 && rstd_out) rstd_out[row] = rstd;
    const __nv_bfloat16 *xs = res ? x_out + row * d : xr;
    for (int c = threadIdx.x * 8; c < d; c += 256 * 8) {
        if (!QLORA_IN(c + 7, d)) break;
        const uint4 xv = *reinterpret_cast<const uint4 *>(xs + c);
        const uint4 gv = *reinterpret_cast<const uint4 *>(g + c);
        const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(&xv);
        const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&gv);
        uint4 ov;
        __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(&ov);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 fa = __bfloat1622float2(a[i]), fg = __bfloat1622float2(b[i]);
            o[i] = __floats2bfloat162_rn(fa.x * rstd * fg.x, fa.y * rstd * fg.y);
        }
        *reinterpret_cast<uint4 *>(u + row * d + c) = ov;
    }
}

// dx = dres + rstd * (g*du - xhat * mean(xhat * g * du)), xhat = x * rstd,
// du = du0 + du1 (+ du2) summed in fp32.  One CTA of 256 threads per row.
__global__ void __launch_bounds__(256) rmsnorm_bwd_kernel(const __nv_bfloat16 *x, const __nv_bfloat16 *g,
                                                          const float *rstd_in, const __nv_bfloat16 *du0,
                                                          const __nv_bfloat16 *du1, const __nv_bfloat16 *du2,
                                                          const __nv_bfloat16 *dres, int d, __nv_bfloat16 *dx)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int64_t row = blockIdx.x;
    const float rstd = rstd_in[row];
    __shared__ float red[8];
    auto du_at = [&](int c, float (&out)[8]) {
        const __nv_bfloat16 *src[3] = {du0, du1, du2};
#pragma unroll
        for (int i = 0; i < 8; i++) out[i] = 0.0f;
#pragma unroll
        for (int s = 0; s < 3; s++) {
            if (!src[s]) continue;
            const uint4 v = *reinterpret_cast<const uint4 *>(src[s] + row * d + c);
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float2 f = __bfloat1622float2(h[i]);
                out[2 * i] += f.x;
                out[2 * i + 1] += f.y;
            }
        }
    };
    auto load8 = [&](const __nv_bfloat16 *p, float (&out)[8]) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 f = __bfloat1622float2(h[i]);
            out[2 * i] = f.x;
            out[2 * i + 1] = f.y;
        }
    };
    float dot = 0.0f;
    for (int c = threadIdx.x * 8; c < d; c += 256 * 8) {
        if (!QLORA_IN(c + 7, d)) break;
        float du[8], xv[8], gv[8];
        du_at(c, du);
        load8(x + row * d + c, xv);
        load8(g + c, gv);
#pragma unroll
        for (int i = 0; i < 8; i++) dot = __fmaf_rn(xv[i] * rstd, gv[i] * du[i], dot);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dot;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; w++) tot += red[w];
    const float mean = tot / (float)d;
    for (int c = threadIdx.x * 8; c < d; c += 256 * 8) {
        if (!QLORA_IN(c + 7, d)) break;
        float du[8], xv[8], gv[8], rv[8];
        du_at(c, du);
        load8(x + row * d + c, xv);
        load8(g + c, gv);
        if (dres)
            load8(dres + row * d + c, rv);
        else
            for (int i = 0; i < 8; i++) rv[i] = 0.0f;
        uint4 ov;
        __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(&ov);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            float v0 = rv[2 * i] + rstd * (gv[2 * i] * du[2 * i] - xv[2 * i] * rstd * mean);
            float v1 = rv[2 * i + 1] + rstd * (gv[2 * i + 1] * du[2 * i + 1] - xv[2 * i + 1] * rstd * mean);
            o[i] = __floats2bfloat162_rn(v0, v1);
        }
        *reinterpret_cast<uint4 *>(dx + row * d + c) = ov;
    }
}

// ---- rotary position embedding --------------------------------------------------
// Angle table: cs[p][i] = (cos, sin) of p * base^(-2i/hd) for positions p <
// seq and pairs i < hd/2, computed once per block call.
__global__ void __launch_bounds__(256) rope_table_kernel(float2 *cs, int seq, int hd, float log2_base)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int half = hd / 2;
    const int id = blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= seq * half || !QLORA_IN(id, seq * half)) return;
    const int p = id / half, i = id % half;
    const float inv = exp2f(-2.0f * (float)i / (float)hd * log2_base);
    float s, c;
    sincosf((float)p * inv, &s, &c);
    cs[id] = make_float2(c, s);
}

// t [rows][heads * hd], row = b * seq + p: the pairs (i, i + hd/2) of each
// head rotate by the table's angle for (p, i) (sign < 0: the inverse rotation,
// which is the backward pass).  One thread per 8 consecutive pairs (16-byte
// accesses); hd % 16 == 0.
__global__ void __launch_bounds__(256) rope_kernel(__nv_bfloat16 *t, const float2 *cs, int64_t rows, int seq,
                                                   int heads, int hd, float sign)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int half = hd / 2, groups = half / 8;
    const int64_t n = rows * heads * groups;
    for (int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; id < n; id += (int64_t)gridDim.x * blockDim.x) {
        const int i0 = (int)(id % groups) * 8;
        const int64_t rh = id / groups;
        const int h = (int)(rh % heads);
        const int64_t row = rh / heads;
        const int p = (int)(row % seq);
        __nv_bfloat16 *base = t + row * (int64_t)heads * hd + (int64_t)h * hd;
        if (!QLORA_IN(row * (int64_t)heads * hd + (int64_t)h * hd + i0 + half + 7, rows * heads * hd) ||
            !QLORA_IN((int64_t)p * half + i0 + 7, (int64_t)seq * half))
            continue;
        uint4 av = *reinterpret_cast<const uint4 *>(base + i0);
        uint4 bv = *reinterpret_cast<const uint4 *>(base + i0 + half);
        __nv_bfloat162 *a2 = reinterpret_cast<__nv_bfloat162 *>(&av);
        __nv_bfloat162 *b2 = reinterpret_cast<__nv_bfloat162 *>(&bv);
        const float2 *tab = cs + (int64_t)p * half + i0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float2 fa = __bfloat1622float2(a2[j]), fb = __bfloat1622float2(b2[j]);
            const float2 c0 = tab[2 * j], c1 = tab[2 * j + 1];
            const float s0 = sign * c0.y, s1 = sign * c1.y;
            a2[j] = __floats2bfloat162_rn(fa.x * c0.x - fb.x * s0, fa.y * c1.x - fb.y * s1);
            b2[j] = __floats2bfloat162_rn(fa.x * s0 + fb.x * c0.x, fa.y * s1 + fb.y * c1.x);
        }
        *reinterpret_cast<uint4 *>(base + i0) = av;
        *reinterpret_cast<uint4 *>(base + i0 + half) = bv;
    }
}

// ---- SwiGLU -----------------------------------------------------------------------
__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + __expf(-z)); }

__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8])
{
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8])
{
    uint4 v;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; i++) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return v;
}

// m = bf16(silu(gate) * up), 8 elements per thread (n % 8 == 0)
__global__ void __launch_bounds__(256) swiglu_fwd_kernel(const __nv_bfloat16 *gate, const __nv_bfloat16 *up,
                                                         __nv_bfloat16 *m, int64_t n)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; 8 * i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float g[8], u[8], o[8];
        if (!QLORA_IN(8 * i + 7, n)) break;
        unpack8(*reinterpret_cast<const uint4 *>(gate + 8 * i), g);
        unpack8(*reinterpret_cast<const uint4 *>(up + 8 * i), u);
#pragma unroll
        for (int j = 0; j < 8; j++) o[j] = g[j] * sigmoidf_(g[j]) * u[j];
        *reinterpret_cast<uint4 *>(m + 8 * i) = pack8(o);
    }
}

// dgate = dm * up * silu'(gate), dup = dm * silu(gate), 8 elements per thread
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const __nv_bfloat16 *dm, const __nv_bfloat16 *gate,
                                                         const __nv_bfloat16 *up, __nv_bfloat16 *dgate,
                                                         __nv_bfloat16 *dup, int64_t n)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; 8 * i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float d[8], g[8], u[8], og[8], ou[8];
        if (!QLORA_IN(8 * i + 7, n)) break;
        unpack8(*reinterpret_cast<const uint4 *>(dm + 8 * i), d);
        unpack8(*reinterpret_cast<const uint4 *>(gate + 8 * i), g);
        unpack8(*reinterpret_cast<const uint4 *>(up + 8 * i), u);
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const float sg = sigmoidf_(g[j]);
            og[j] = d[j] * u[j] * (sg + g[j] * sg * (1.0f - sg));
            ou[j] = d[j] * g[j] * sg;
        }
        *reinterpret_cast<uint4 *>(dgate + 8 * i) = pack8(og);
        *reinterpret_cast<uint4 *>(dup + 8 * i) = pack8(ou);
    }
}

// ---- batched bf16 products for attention --------------------------------------------
// C[z] = alpha * A[z] B[z] with A [M x K], B [K x N] (fp32 accumulation on the
// tensor cores, mma m16n8k16).  A is stored [M][K] (AT = false) or [K][M]
// (AT = true); B is stored [K][N] (BT = false) or [N][K] (BT = true); leading
// dimensions and two-level batch strides (z = z0 * nz1 + z1) in elements.
// tri: 0 full contraction; 1 A is lower-triangular (zero for k > i): the
// contraction stops after the tile's last row; 2 A is upper-triangular (zero
// for k < i): it starts at the tile's first row.  causal (fp32 output): C[i][j]
// for j > i is written as -inf and tiles wholly above the diagonal skip the
// products.  M, N, K and every leading dimension are multiples of 8, base
// addresses 16-byte aligned.
struct BmmArgs {
    const __nv_bfloat16 *A, *B;
    void *C;
    int M, N, K;
    int64_t lda, ldb, ldc;
    int64_t sa0, sa1, sb0, sb1, sc0, sc1;
    int nz1;
    float alpha;
    int tri;
    int causal;
    int64_t a_n, b_n, c_n;   // elements of the buffers behind A, B and C (bounds-checked build)
};

constexpr int kBM = 128, kBN = 128, kBK = 32;
constexpr int kPadK = kBK + 8;     // row stride of [rows][k] tiles (bank spread)
constexpr int kPadMN = kBM + 8;    // row stride of [k][cols] tiles

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid)
{
    const int bytes = valid ? 16 : 0;   // zero-fill when out of range
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sm100::smem_u32(smem)), "l"(gmem), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <bool AT, bool BT, bool OUT_F32>
__global__ void __launch_bounds__(256) bmm_kernel(const BmmArgs p)
{
    constexpr int A_ELEMS = AT ? kBK * kPadMN : kBM * kPadK;
    constexpr int B_ELEMS = BT ? kBN * kPadK : kBK * kPadMN;
    __shared__ __align__(16) __nv_bfloat16 sA[2][A_ELEMS];
    __shared__ __align__(16) __nv_bfloat16 sB[2][B_ELEMS];
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int z = blockIdx.z;
    const int z0 = z / p.nz1, z1 = z % p.nz1;
    const __nv_bfloat16 *A = p.A + z0 * p.sa0 + z1 * p.sa1;
    const __nv_bfloat16 *B = p.B + z0 * p.sb0 + z1 * p.sb1;
    const int i0 = blockIdx.y * kBM, j0 = blockIdx.x * kBN;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = warp >> 2, wn = warp & 3;   // 2 x 4 warps, 64 x 32 each

    if (OUT_F32 && p.causal && j0 > i0 + kBM - 1) {
        // wholly above the diagonal
        float *C = static_cast<float *>(p.C) + z0 * p.sc0 + z1 * p.sc1;
        for (int e = tid; e < kBM * kBN; e += 256) {
            const int i = i0 + e / kBN, j = j0 + e % kBN;
            if (i < p.M && j < p.N && QLORA_IN(z0 * p.sc0 + z1 * p.sc1 + (int64_t)i * p.ldc + j, p.c_n))
                C[(int64_t)i * p.ldc + j] = -INFINITY;
        }
        return;
    }
    int kbeg = 0, kend = p.K;
    if (p.tri == 1) kend = min(p.K, i0 + kBM);
    if (p.tri == 2) kbeg = (i0 / kBK) * kBK;
    const int nk = (kend - kbeg + kBK - 1) / kBK;

    auto load = [&](int st, int k0) {
        // A tile: 512 16-byte chunks, two per thread
#pragma unroll
        for (int rep = 0; rep < 2; rep++) {
            const int ch = tid + rep * 256;
            if (!AT) {
                const int r = ch >> 2, c = (ch & 3) * 8;            // [128 rows][32 k]
                const int gi = i0 + r, gk = k0 + c;
                const bool ok = gi < p.M && gk < kend &&
                                QLORA_IN(z0 * p.sa0 + z1 * p.sa1 + (int64_t)gi * p.lda + gk + 7, p.a_n);
                cp_async16(&sA[st][r * kPadK + c], A + (ok ? (int64_t)gi * p.lda + gk : 0), ok);
            } else {
                const int r = ch >> 4, c = (ch & 15) * 8;           // [32 k][128 rows]
                const int gk = k0 + r, gi = i0 + c;
                const bool ok = gk < kend && gi < p.M &&
                                QLORA_IN(z0 * p.sa0 + z1 * p.sa1 + (int64_t)gk * p.lda + gi + 7, p.a_n);
                cp_async16(&sA[st][r * kPadMN + c], A + (ok ? (int64_t)gk * p.lda + gi : 0), ok);
            }
        }
#pragma unroll
        for (int rep = 0; rep < 2; rep++) {
            const int ch = tid + rep * 256;
            if (BT) {
                const int r = ch >> 2, c = (ch & 3) * 8;            // [128 cols][32 k]
                const int gj = j0 + r, gk = k0 + c;
                const bool ok = gj < p.N && gk < kend &&
                                QLORA_IN(z0 * p.sb0 + z1 * p.sb1 + (int64_t)gj * p.ldb + gk + 7, p.b_n);
                cp_async16(&sB[st][r * kPadK + c], B + (ok ? (int64_t)gj * p.ldb + gk : 0), ok);
            } else {
                const int r = ch >> 4, c = (ch & 15) * 8;           // [32 k][128 cols]
                const int gk = k0 + r, gj = j0 + c;
                const bool ok = gk < kend && gj < p.N &&
                                QLORA_IN(z0 * p.sb0 + z1 * p.sb1 + (int64_t)gk * p.ldb + gj + 7, p.b_n);
                cp_async16(&sB[st][r * kPadMN + c], B + (ok ? (int64_t)gk * p.ldb + gj : 0), ok);
            }
        }
        cp_async_commit();
    };

    float acc[4][4][4];
#pragma unroll
    for (int a = 0; a < 4; a++)
#pragma unroll
        for (int b = 0; b < 4; b++)
#pragma unroll
            for (int c = 0; c < 4; c++) acc[a][b][c] = 0.0f;

    if (nk > 0) load(0, kbeg);
    for (int kt = 0; kt < nk; kt++) {
        const int st = kt & 1;
        if (kt + 1 < nk) {
            load(st ^ 1, kbeg + (kt + 1) * kBK);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kBK; kk += 16) {
            uint32_t af[4][4];
#pragma unroll
            for (int mi = 0; mi < 4; mi++) {
                const int r0 = wm * 64 + mi * 16;
                if (!AT) {
                    const int row = r0 + (lane & 15), col = kk + (lane >> 4) * 8;
                    ldsm_x4(sm100::smem_u32(&sA[st][row * kPadK + col]), af[mi][0], af[mi][1], af[mi][2], af[mi][3]);
                } else {
                    // matrices: (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
                    const int mtx = lane >> 3;
                    const int kr = kk + (mtx >> 1) * 8 + (lane & 7), ic = r0 + (mtx & 1) * 8;
                    ldsm_x4_t(sm100::smem_u32(&sA[st][kr * kPadMN + ic]), af[mi][0], af[mi][1], af[mi][2], af[mi][3]);
                }
            }
#pragma unroll
            for (int nj = 0; nj < 4; nj += 2) {
                // two n8 tiles: b0/b1 of tile nj, b0/b1 of tile nj + 1
                uint32_t b[4];
                const int c0 = wn * 32 + nj * 8;
                if (BT) {
                    // matrices: (n 0-7, k 0-7), (n 0-7, k 8-15), (n 8-15, k 0-7), (n 8-15, k 8-15)
                    const int mtx = lane >> 3;
                    const int nr = c0 + (mtx >> 1) * 8 + (lane & 7), kc = kk + (mtx & 1) * 8;
                    ldsm_x4(sm100::smem_u32(&sB[st][nr * kPadK + kc]), b[0], b[1], b[2], b[3]);
                } else {
                    // matrices: (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
                    const int mtx = lane >> 3;
                    const int kr = kk + (mtx & 1) * 8 + (lane & 7), nc = c0 + (mtx >> 1) * 8;
                    ldsm_x4_t(sm100::smem_u32(&sB[st][kr * kPadMN + nc]), b[0], b[1], b[2], b[3]);
                }
#pragma unroll
                for (int mi = 0; mi < 4; mi++) {
                    mma16816(acc[mi][nj], af[mi], b[0], b[1]);
                    mma16816(acc[mi][nj + 1], af[mi], b[2], b[3]);
                }
            }
        }
        __syncthreads();
    }

    // epilogue: lane (g, c) holds rows g and g + 8, columns 2c and 2c + 1
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int mi = 0; mi < 4; mi++) {
#pragma unroll
        for (int nj = 0; nj < 4; nj++) {
#pragma unroll
            for (int half = 0; half < 2; half++) {
                const int i = i0 + wm * 64 + mi * 16 + g + 8 * half;
                const int j = j0 + wn * 32 + nj * 8 + 2 * c;
                if (i >= p.M || j >= p.N) continue;
                if (!QLORA_IN(z0 * p.sc0 + z1 * p.sc1 + (int64_t)i * p.ldc + j + 1, p.c_n)) continue;
                float v0 = p.alpha * acc[mi][nj][2 * half], v1 = p.alpha * acc[mi][nj][2 * half + 1];
                if (OUT_F32) {
                    if (p.causal) {
                        if (j > i) v0 = -INFINITY;
                        if (j + 1 > i) v1 = -INFINITY;
                    }
                    float *C = static_cast<float *>(p.C) + z0 * p.sc0 + z1 * p.sc1;
                    *reinterpret_cast<float2 *>(C + (int64_t)i * p.ldc + j) = make_float2(v0, v1);
                } else {
                    __nv_bfloat16 *C = static_cast<__nv_bfloat16 *>(p.C) + z0 * p.sc0 + z1 * p.sc1;
                    *reinterpret_cast<__nv_bfloat162 *>(C + (int64_t)i * p.ldc + j) = __floats2bfloat162_rn(v0, v1);
                }
            }
        }
    }
}

// ---- softmax rows -----------------------------------------------------------------------
// P[r][:] = bf16(exp(S[r][:] - max) / sum) for rows of length n (S holds -inf
// where masked).  One warp per row.
__global__ void __launch_bounds__(256) softmax_rows_kernel(const float *S, __nv_bfloat16 *P, int64_t rows, int n)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const float *s = S + r * n;
    float mx = -INFINITY;
    for (int j = lane; j < n; j += 32) mx = fmaxf(mx, s[j]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.0f;
    for (int j = lane; j < n; j += 32) sum += __expf(s[j] - mx);
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.0f / sum;
    __nv_bfloat16 *pr = P + r * n;
    for (int j = lane; j < n; j += 32) pr[j] = __float2bfloat16_rn(__expf(s[j] - mx) * inv);
}

// dS[r][:] = bf16(scale * P (dP - sum_j P dP)) row by row (softmax backward;
// scale = 1/sqrt(head_dim) folds the score scaling into dS).  dS may alias P.
__global__ void __launch_bounds__(256) dsoftmax_rows_kernel(const __nv_bfloat16 *P, const float *dP,
                                                            __nv_bfloat16 *dS, int64_t rows, int n, float scale)
{
    sm100::pdl_wait();
    sm100::pdl_trigger();
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const __nv_bfloat16 *pr = P + r * n;
    const float *dpr = dP + r * n;
    float dot = 0.0f;
    for (int j = lane; j < n; j += 32) dot = __fmaf_rn(bf(pr[j]), dpr[j], dot);
#pragma unroll
    for (int o = 16; o; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    __nv_bfloat16 *out = dS + r * n;
    for (int j = lane; j < n; j += 32) {
        const float pv = bf(pr[j]);
        out[j] = __float2bfloat16_rn(scale * pv * (dpr[j] - dot));
    }
}

}  // namespace blk
}  // namespace qlora
