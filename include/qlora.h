/*
 * qlora.h -- C ABI of the B200 (sm_100a) QLoRA hot path.
 *
 * What is computed (all citations are to "QLoRA: Efficient Finetuning of
 * Quantized LLMs", inquiringlines.com/papers/2305.14314, unless noted):
 *   - a frozen weight W [N, K] is stored as 4-bit NormalFloat codes with one
 *     absmax constant per block of 64 ("Method", paragraphs "4-bit NormalFloat
 *     Quantization" and "Double Quantization"), and the block constants are
 *     quantized a second time (double quantization) to 8-bit floats in groups
 *     of 256 blocks after subtracting their mean;
 *   - whenever the weight is used it is dequantized to BFloat16 and multiplied
 *     in 16-bit arithmetic ("Method", storage vs. computation data type);
 *   - the QLoRA linear layer x_out = (W_q + B A) x_in (mbrenndoerfer.com QLoRA
 *     essay, "Low-Rank Adaptation (LoRA)"), in row-vector form
 *         Y = X W'^T + s (X A^T) B^T,      W' = dequant(W_q),
 *     with its backward pass dX, dA, dB; the quantized weight is frozen, so
 *     there is no dW (abstract: the gradients pass through the frozen 4-bit
 *     base model and update only the low-rank adapters).
 *
 * Conventions common to every entry point
 *   - Pointers named "device" must point to memory of the current CUDA device;
 *     the caller allocates and frees every buffer.  The library never
 *     allocates device memory and never frees what it is given, except
 *     through the paged-memory helpers qlora_paged_alloc / qlora_paged_free,
 *     which exist to hand out unified memory for optimizer states.
 *   - Every device pointer must be 16-byte aligned (tensor-memory-access
 *     copies require it); QLORA_ERR_ALIGNMENT otherwise.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and is asynchronous.  Argument validation is synchronous
 *     and happens before anything is enqueued: a non-OK status means nothing
 *     was launched.  No entry point synchronizes the stream.
 *   - Inputs must be finite numbers; results for NaN or infinite inputs are
 *     unspecified.
 *   - Outputs must not alias inputs or each other.
 *   - Matrices are row-major and dense (leading dimension = column count).
 *   - Kernel-side failures (a bounded wait that timed out) are recorded in a
 *     device error word, read back by qlora_check_device_error().
 *   - The library requires a compute capability 10.0 device (B200);
 *     QLORA_ERR_UNSUPPORTED otherwise.  There is no CPU fallback.
 *   - Per-device state is set up on first use and kept for the life of the
 *     process: device properties, kernel attributes, and the device addresses
 *     of the library's own __device__ variables (the error word, the fixed
 *     scratch of qlora_quantize_nf4_dq_noalloc).  cudaDeviceReset() destroys
 *     what that state refers to: do not use the library on a device again
 *     after resetting it in the same process.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Blocksize of the first quantization level: 64 consecutive elements of one
 * row ("Method", paragraph "Double Quantization": W uses blocks of 64). */
#define QLORA_BLOCK 64
/* Number of first-level constants per second-level (double-quantization)
 * group: 256 consecutive blocks in row-major block order. */
#define QLORA_GROUP 256

typedef enum {
    QLORA_OK = 0,
    QLORA_ERR_INVALID_ARG = 1, /* null pointer, unknown enum, negative size   */
    QLORA_ERR_SHAPE = 2,       /* a size violates the documented constraints  */
    QLORA_ERR_ALIGNMENT = 3,   /* a device pointer is not 16-byte aligned     */
    QLORA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required  */
    QLORA_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed           */
    QLORA_ERR_UNSUPPORTED = 6, /* not a compute capability 10.x device        */
    QLORA_ERR_TIMEOUT = 7      /* a kernel's bounded wait gave up (device)    */
} qlora_status;

typedef enum { QLORA_BF16 = 0, QLORA_FP32 = 1, QLORA_FP16 = 2 } qlora_dtype;

/*
 * A quantized weight W [rows, cols] (rows = N = out_features, cols = K =
 * in_features).  Plain data: the struct holds caller-owned device pointers
 * and a host copy of the 16-entry codebook.
 *   packed  device, rows*cols/2 bytes.  Element (n, k) has flat index
 *           i = n*cols + k; its 4-bit code sits in byte i/2, in bits 0-3 when
 *           i is even and bits 4-7 when i is odd.
 *   code2   device, nblocks = rows*cols/64 bytes: E4M3 (OCP "e4m3fn") code of
 *           block b's constant after subtracting the mean and dividing by
 *           the group scale.  Block b covers flat indices [64b, 64b+64).
 *   c2      device, ngroups = ceil(nblocks/256) floats: group scale of blocks
 *           [256g, 256g+256).
 *   mean    device, 1 float: mean of all first-level constants of W.
 *   codebook  host values q[0..15], strictly ascending, containing exactly
 *           one 0; the NF4 table from qlora_build_nf4_codebook(), the Int4
 *           table from qlora_build_int4_codebook(), the FP4 table from
 *           qlora_build_fp4_codebook(), or any other 16-value table with the
 *           same properties that the quantizer accepts.
 */
typedef struct {
    int64_t rows;
    int64_t cols;
    uint8_t *packed;
    uint8_t *code2;
    float *c2;
    float *mean;
    float codebook[16];
} qlora_nf4_weight;

/*
 * qlora_build_nf4_codebook -- the NF4 data type ("Method", "4-bit NormalFloat
 * Quantization", steps (1)-(2) and the asymmetric construction: 2^(k-1)
 * quantiles of N(0,1) for the negative part and 2^(k-1)+1 for the positive
 * part, unified with one of the two zeros removed, normalized into [-1, 1]).
 * The page omits the probabilities; each side uses equally spaced
 * probabilities from 1 - delta down to 1/2, delta being the tail probability
 * of the outermost value.  Host-only, no CUDA call.
 *   delta          tail probability in (0, 0.5); delta <= 0 selects the
 *                  default (1/32 + 1/30)/2.
 *   codebook_out   host, 16 floats, written ascending: -1 first, +1 last,
 *                  exactly one 0 at index 7.
 * Errors: QLORA_ERR_INVALID_ARG for a null pointer or delta >= 0.5.
 */
QLORA_API qlora_status qlora_build_nf4_codebook(double delta, float codebook_out[16]);

/*
 * qlora_build_nfk_codebook -- k-bit NormalFloat (k = 2, 3, 4) from the same
 * construction, held in the 16-entry table of the 4-bit codec: the 2^k NF-k
 * values (ascending, -1 .. 1, one zero), then 16 - 2^k padding values beyond
 * +-1 (half at -1 - i/4 below -1, half at 1 + i/4 above 1, i = 1, 2, ...),
 * which are never the nearest value to a scaled element; k = 4 is NF4 itself.
 *   delta  tail probability in (0, 0.5); <= 0 selects
 *          1/2 (1/(2 * 2^k) + 1/(2 (2^k - 1))).
 * Host-only, no CUDA call.  Errors: QLORA_ERR_INVALID_ARG (null pointer, k
 * outside 2..4, delta >= 0.5).
 */
QLORA_API qlora_status qlora_build_nfk_codebook(int k, double delta, float codebook_out[16]);

/*
 * qlora_build_int4_codebook -- a 4-bit integer table for the same codec and
 * GEMMs ("Introduction", item (1), names 4-bit integers as the baseline NF4
 * is compared with, without defining them).  Reading: the two's-complement
 * integers -8 .. 7 divided by 7, q_j = RN32((j - 8) / 7), so that +-7 carry
 * the block's absmax; -8/7 is never the nearest value to a scaled element.
 * Strictly ascending with its one zero at index 8.  Host-only, no CUDA call.
 *   codebook_out   host, 16 floats.
 * Errors: QLORA_ERR_INVALID_ARG for a null pointer.
 */
QLORA_API qlora_status qlora_build_int4_codebook(float codebook_out[16]);

/*
 * qlora_build_fp4_codebook -- a 4-bit float table for the same codec and
 * GEMMs ("Introduction", item (1), names 4-bit floats as the other data type
 * NF4 is compared with, without defining them).  Reading: the E2M1 element
 * type (1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit; magnitudes
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6) divided by 6, each value RN32(v / 6).  E2M1's
 * +0 and -0 are one table value, so index 0 holds -8/6, which lies below -1
 * and is never the nearest value; -1 .. 1 follow at indices 1 .. 15 with the
 * zero at index 8.  Host-only, no CUDA call.
 *   codebook_out   host, 16 floats.
 * Errors: QLORA_ERR_INVALID_ARG for a null pointer.
 */
QLORA_API qlora_status qlora_build_fp4_codebook(float codebook_out[16]);

/*
 * Workspace in bytes that qlora_quantize_nf4_dq needs for a rows x cols
 * weight (first-level constants plus a few reduction slots).
 */
QLORA_API size_t qlora_quantize_workspace_bytes(int64_t rows, int64_t cols);

/*
 * qlora_quantize_nf4_dq -- NF4 quantization with double quantization.
 * ("Method": "4-bit NormalFloat Quantization" step (3) and "Double
 * Quantization".)  Per block of 64: c1 = max|x|; if c1 < 2^-126 every code is
 * the codebook's zero, else n = RN32(x * RN32(1/c1)) and the code is the
 * index of the codebook value nearest to n (ties: lower index).  Then
 * mean = binary32 nearest to the exact mean of all c1 (ties to even); per
 * group: d = RN32(c1 - mean), c2 = RN32(max|d| / 448), code2 = E4M3 with
 * round-to-nearest-even and saturation of RN32(d / c2) (all zero if c2 = 0).
 *   W          device, rows*cols elements of w_dtype (QLORA_BF16, QLORA_FP16
 *              or QLORA_FP32), row-major.
 *   out        host struct: rows, cols, the four device buffers (written) and
 *              the codebook (read).  rows >= 1, cols % 64 == 0.
 *   workspace  device, at least qlora_quantize_workspace_bytes(rows, cols)
 *              bytes; contents on entry do not matter; clobbered.
 * Errors: INVALID_ARG (null pointer, unknown dtype, a codebook that is not
 * strictly increasing or does not hold exactly one zero), SHAPE, ALIGNMENT,
 * WORKSPACE, CUDA, UNSUPPORTED (not a B200, or a codebook the code lookup
 * cannot serve: two midpoints between neighbouring values that share the top
 * 12 bits of their order-preserving binary32 keys, or a pair of neighbours
 * whose sum is not exact in binary64; neither happens for the NF4 and Int4
 * tables of the builders above).
 * Deterministic: the same input gives the same bytes on every call.
 */
QLORA_API qlora_status qlora_quantize_nf4_dq(const void *W, qlora_dtype w_dtype, const qlora_nf4_weight *out,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Largest number of 64-weight blocks qlora_quantize_nf4_dq_noalloc accepts
 * (rows * cols / 64): 2^20 blocks, i.e. 67,108,864 weights, such as 8192 x
 * 8192.  Its fixed scratch array takes about 4 MiB of device memory per
 * device, reserved when the library's device code is loaded.
 */
#define QLORA_NOALLOC_MAX_BLOCKS (1 << 20)

/*
 * qlora_quantize_nf4_dq_noalloc -- qlora_quantize_nf4_dq without a workspace.
 * The papers describe no such variant; it is a library convenience.  It
 * writes the same bytes as qlora_quantize_nf4_dq, but its scratch memory
 * (reduction slots and the first-level constants) is a fixed array inside
 * the library, so the call allocates nothing and needs no buffer from the
 * caller: for callers that have no device memory to spare at quantization
 * time (memory already reserved for a pool or a cache) or that must not
 * call cudaMalloc / cudaFree, which synchronize the whole device, while
 * other streams are running.
 *   W, w_dtype, out  as for qlora_quantize_nf4_dq.
 *   stream           cudaStream_t the kernels run on (NULL: legacy default).
 * Limits and caveats:
 *   - rows * cols / 64 must not exceed QLORA_NOALLOC_MAX_BLOCKS; larger
 *     weights are rejected with QLORA_ERR_SHAPE before any CUDA call.
 *   - The scratch array is one per device and shared by all calls: two calls
 *     whose kernels may run at the same time (different streams or host
 *     threads without ordering between them) race and corrupt each other's
 *     results.  Order them, e.g. on one stream.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture begins.  Each call then clears the reduction
 *     slots with cudaMemsetAsync on `stream` and launches two kernels.
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, CUDA, UNSUPPORTED.
 */
QLORA_API qlora_status qlora_quantize_nf4_dq_noalloc(const void *W, qlora_dtype w_dtype,
                                                     const qlora_nf4_weight *out, void *stream);

/*
 * qlora_dequantize_nf4_dq -- expand a quantized weight to BFloat16 ("Method":
 * the tensor is dequantized to BFloat16 whenever it is used).  Per block:
 * c1' = fmaf(E4M3value(code2), c2, mean) (one rounding); per element
 * w = bf16_RNE(RN32(q[code] * c1')).
 *   w        host struct describing the quantized weight (read only).
 *   out_bf16 device, rows*cols bf16, row-major.
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, CUDA, UNSUPPORTED.
 */
QLORA_API qlora_status qlora_dequantize_nf4_dq(const qlora_nf4_weight *w, void *out_bf16, void *stream);

/*
 * qlora_dequantize_nf4_dq_ex -- the same with the output type out_dtype:
 * QLORA_BF16 (as above) or QLORA_FP16 (w = fp16_RNE(RN32(q[code] * c1')),
 * the fp16 compute dtype).  Errors as above, INVALID_ARG for another dtype.
 */
QLORA_API qlora_status qlora_dequantize_nf4_dq_ex(const qlora_nf4_weight *w, void *out, qlora_dtype out_dtype,
                                                  void *stream);

/*
 * Workspace in bytes for qlora_linear_fwd / qlora_linear_bwd at these sizes
 * (M tokens, weight N x K, rank r).  One workspace sized by this function
 * serves both directions.
 */
QLORA_API size_t qlora_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r);

/*
 * qlora_linear_fwd -- Y = X W'^T + H_b B^T with H = s X A^T (float32 sums),
 * H_b = bf16(H); W' is the dequantized weight of `w`, expanded tile by tile
 * on chip and never written to memory.
 *   w       quantized weight, N = w->rows, K = w->cols; N % 8 == 0.
 *   X       device bf16 [M, K].  M >= 0 (M == 0: nothing is done).
 *   A       device bf16 [r, K];  B  device bf16 [N, r].
 *   r       adapter rank, 8 <= r <= 128, r % 8 == 0.
 *   scale   s (usually lora_alpha / r), any finite value.
 *   Y       device [M, N] of y_dtype (QLORA_BF16 or QLORA_FP32).
 *   H_save  device float [M, r] or NULL: receives H = s X A^T for the
 *           backward pass.
 *   workspace  device, >= qlora_linear_workspace_bytes(M, N, K, r) bytes.
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, WORKSPACE, CUDA, UNSUPPORTED.
 */
QLORA_API qlora_status qlora_linear_fwd(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A,
                              const void *B, int32_t r, float scale, void *Y, qlora_dtype y_dtype,
                              float *H_save, void *workspace, size_t workspace_bytes, void *stream);

/*
 * qlora_linear_bwd -- gradients of the layer above for dY = dL/dY:
 *     G  = s dY B                      (float32 sums)
 *     dX = dY W' + bf16(G) A           (W' expanded on chip, transposed use)
 *     dA = G^T X                       (= s (dY B)^T X)
 *     dB = dY^T H                      (= s dY^T (X A^T))
 * dA and dB are computed from G and H carried at about 16 significant bits
 * (each split into two bf16 terms), so their error stays at the level of
 * float32 accumulation.  No gradient is formed for the frozen weight.
 *   w, X, A, B, r, scale, M   as for qlora_linear_fwd.
 *   dY       device bf16 [M, N].
 *   H_saved  device float [M, r] from qlora_linear_fwd, or NULL to recompute.
 *   dX       device [M, K] of dx_dtype, or NULL to skip the input gradient.
 *   dA       device float [r, K], overwritten.
 *   dB       device float [N, r], overwritten.
 *   workspace  device, >= qlora_linear_workspace_bytes(M, N, K, r) bytes.
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, WORKSPACE, CUDA, UNSUPPORTED.
 */
QLORA_API qlora_status qlora_linear_bwd(const qlora_nf4_weight *w, const void *X, const void *dY, int64_t M,
                              const void *A, const void *B, int32_t r, float scale,
                              const float *H_saved, void *dX, qlora_dtype dx_dtype, float *dA,
                              float *dB, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Paged optimizer ("QLoRA: Efficient Finetuning of Quantized LLMs",
 * Introduction item (3) and "Method", opening paragraph; mbrenndoerfer.com
 * essay, "Paged Optimizers"): the optimizer states are allocated in NVIDIA
 * unified memory, so the driver evicts them to CPU RAM when the GPU runs out
 * of memory and pages them back in when the update step touches them.
 *
 * qlora_paged_alloc -- `bytes` of unified (managed) memory, zero-filled on the
 * host (the pages start in CPU memory).  The one place where the library
 * allocates: paging is the point of these buffers.  The caller owns the
 * allocation and releases it with qlora_paged_free (a synchronizing call).
 * Errors: INVALID_ARG (null ptr, bytes == 0), CUDA, UNSUPPORTED.
 */
QLORA_API qlora_status qlora_paged_alloc(size_t bytes, void **ptr);
QLORA_API qlora_status qlora_paged_free(void *ptr);

/*
 * qlora_paged_prefetch -- migrate [ptr, ptr + bytes) of a paged allocation to
 * the current device (to_device = 1) or to host memory (to_device = 0),
 * asynchronously on `stream`.  Without it, pages move on demand when a kernel
 * or the host touches them.
 * Errors: INVALID_ARG, CUDA, UNSUPPORTED.
 */
QLORA_API qlora_status qlora_paged_prefetch(const void *ptr, size_t bytes, int to_device, void *stream);

/* Hyperparameters of one AdamW step; `step` counts from 1. */
typedef struct {
    float lr;
    float beta1;
    float beta2;
    float eps;
    float weight_decay;
    int64_t step;
} qlora_adamw_hparams;

/*
 * qlora_adamw_step -- one AdamW update (Adam with decoupled weight decay) of
 * n parameters, element by element, in float32:
 *     p <- p * (1 - lr * wd)
 *     m <- beta1 m + (1 - beta1) g
 *     v <- beta2 v + (1 - beta2) g^2
 *     p <- p - (lr / (1 - beta1^t)) * m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
 * The pages name paged optimizers and optimizer states but no optimizer; AdamW
 * is the reading used here.
 *   param       device float [n], updated in place (the master copy).
 *   param_bf16  device bf16 [n] or NULL: receives bf16(p) after the update,
 *               e.g. a flat buffer holding the adapters A and B that the
 *               linear layer reads; 8-byte aligned.
 *   grad        device float [n] (dA and dB of qlora_linear_bwd, flattened).
 *   exp_avg, exp_avg_sq  float [n], the moments m and v: device memory or a
 *               qlora_paged_alloc buffer (zero before the first step).
 *   h           host struct, lr >= 0, 0 <= beta < 1, eps > 0, wd >= 0, step >= 1.
 * Errors: INVALID_ARG, ALIGNMENT (param, grad, m, v not 16-byte aligned), CUDA,
 * UNSUPPORTED.
 */
QLORA_API qlora_status qlora_adamw_step(float *param, void *param_bf16, const float *grad, float *exp_avg,
                                        float *exp_avg_sq, int64_t n, const qlora_adamw_hparams *h, void *stream);

/*
 * One QLoRA transformer block ("QLoRA: Efficient Finetuning of Quantized
 * LLMs", Introduction: LoRA adapters at every network layer, trained with
 * gradient checkpointing).  The pages fix the seven linear shapes of the
 * LLaMA models but not the rest of the block; it is the LLaMA decoder layer:
 *     u1 = RMSNorm(x; norm1); q, k, v = Lq(u1), Lk(u1), Lv(u1)
 *     q, k rotated (RoPE: pairs (i, i + D/2) of each head by p * base^(-2i/D)
 *     at sequence position p)
 *     a = causal softmax(q k^T / sqrt(D)) v per sequence and head
 *     h = x + Lo(a);  u2 = RMSNorm(h; norm2)
 *     y = h + Ldown(silu(Lgate(u2)) * Lup(u2))
 * with RMSNorm(x; g) = x / sqrt(mean(x^2) + eps) * g.  Every L is the QLoRA
 * linear of qlora_linear_fwd (frozen NF4 + DQ weight, adapters A, B, scale
 * lora_scale).  Activations are bf16 [batch * seq, hidden], row = b * seq + p.
 *   w[7], A[7], B[7]  in the order q, k, v, o, gate, up, down; w[l] as for
 *                     qlora_linear_fwd, A[l] device bf16 [r][in], B[l] device
 *                     bf16 [out][r].
 *   norm1, norm2      device bf16 [hidden] (frozen).
 * Constraints: heads * head_dim == hidden, head_dim % 16 == 0, hidden % 64 ==
 * 0, inter % 64 == 0, seq % 8 == 0, r as for the linear layer.
 */
typedef struct {
    int32_t batch, seq, hidden, heads, head_dim, inter, r;
    float lora_scale;
    float rms_eps;
    float rope_base;
    qlora_nf4_weight w[7];
    const void *A[7];
    const void *B[7];
    const void *norm1;
    const void *norm2;
} qlora_block;

/* Workspace bytes of qlora_block_fwd / qlora_block_bwd (0 for an invalid
 * description). */
QLORA_API size_t qlora_block_workspace_bytes(const qlora_block *blk);

/*
 * qlora_block_fwd -- y = block(x).  Keeps nothing else (gradient
 * checkpointing: the backward pass recomputes what it needs from x).
 *   x, y       device bf16 [batch * seq, hidden].
 *   workspace  device, >= qlora_block_workspace_bytes(blk).
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, WORKSPACE, CUDA, UNSUPPORTED.
 */
QLORA_API qlora_status qlora_block_fwd(const qlora_block *blk, const void *x, void *y, void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * qlora_block_bwd -- gradients of the block for dy = dL/dy: recomputes the
 * forward pass from x, then returns dx and the adapter gradients of all seven
 * linears (the quantized weights and the norm weights are frozen).
 *   dy, dx     device bf16 [batch * seq, hidden].
 *   dA[l], dB[l]  device float [r][in] and [out][r], overwritten.
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, WORKSPACE, CUDA, UNSUPPORTED.
 */
QLORA_API qlora_status qlora_block_bwd(const qlora_block *blk, const void *x, const void *dy, void *dx,
                                       float *const dA[7], float *const dB[7], void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * Options of the QLoRA linear layer (the _ex entry points below; the plain
 * entry points are the _ex ones with opts = NULL).
 *   dropout_mask  device or NULL.  LoRA dropout on the adapter input (the
 *                 blog "Efficient Language Model Fine-Tuning with QLoRA on
 *                 Resource-Constrained Hardware", LoraConfig snippet,
 *                 lora_dropout): the adapter branch sees X_d = X * mask /
 *                 (1 - p) while the frozen weight sees X.  Bit (k % 8) of
 *                 byte (m * K + k) / 8 is element (m, k)'s mask bit (1 =
 *                 kept); M * K / 8 bytes, 16-byte aligned.  Kept elements
 *                 are bf16(RN32(x * RN32(1 / RN32(1 - p)))), dropped ones 0.
 *                 The same mask must be passed to the forward and the
 *                 backward call of one step.  With dropout:
 *                     H  = s X_d A^T
 *                     dX = dY W' + (bf16(G) A) * mask / (1 - p)
 *                     dA = G^T X_d,  dB = dY^T H
 *   dropout_p     probability the mask was drawn with, 0 <= p < 1.
 *   compute_dtype QLORA_BF16 (0, the default) or QLORA_FP16: the 16-bit type
 *                 of X, A, B, dY, of the expanded weight (w = fp16_RNE(RN32(
 *                 q[code] * c1')) for fp16) and of 16-bit outputs; y_dtype and
 *                 dx_dtype are then that type or QLORA_FP32 (the blog's
 *                 BitsAndBytesConfig snippet, bnb_4bit_compute_dtype).  H and
 *                 G are carried as hi + lo pairs of the same type.
 *   adapter_ready 0 (default) or 1: the adapter's low-rank products of this
 *                 call are already in the workspace, written by
 *                 qlora_linear_adapter_fwd / qlora_linear_adapter_bwd with the
 *                 same arguments and options; the call runs the rest only.
 */
typedef struct {
    const uint8_t *dropout_mask;
    float dropout_p;
    qlora_dtype compute_dtype;
    int32_t adapter_ready;
} qlora_linear_opts;

/* Workspace bytes for the _ex entry points with these options (dropout needs
 * 6 M K bytes more than qlora_linear_workspace_bytes). */
QLORA_API size_t qlora_linear_workspace_bytes_ex(int64_t M, int64_t N, int64_t K, int32_t r,
                                                 const qlora_linear_opts *opts);

/* qlora_linear_fwd / qlora_linear_bwd with options (NULL: none).  Errors as
 * for the plain calls, plus INVALID_ARG for p outside [0, 1), an unknown
 * compute dtype or an output dtype that does not match it, and ALIGNMENT for
 * a misaligned mask. */
QLORA_API qlora_status qlora_linear_fwd_ex(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A,
                                           const void *B, int32_t r, float scale, void *Y, qlora_dtype y_dtype,
                                           float *H_save, void *workspace, size_t workspace_bytes, void *stream,
                                           const qlora_linear_opts *opts);
QLORA_API qlora_status qlora_linear_bwd_ex(const qlora_nf4_weight *w, const void *X, const void *dY, int64_t M,
                                           const void *A, const void *B, int32_t r, float scale,
                                           const float *H_saved, void *dX, qlora_dtype dx_dtype, float *dA,
                                           float *dB, void *workspace, size_t workspace_bytes, void *stream,
                                           const qlora_linear_opts *opts);

/*
 * The first step of a linear call on its own: the adapter's low-rank products
 * (and, under LoRA dropout, the dropped-out input), written into the
 * workspace.  A later qlora_linear_fwd_ex / qlora_linear_bwd_ex on the same
 * workspace, with the same arguments and opts->adapter_ready = 1, runs the
 * rest and produces the same bits as the undivided call.  Splitting lets a
 * caller run these small, bandwidth-bound products of independent linears on
 * a second stream, beside another linear's fused GEMM (the two halves must
 * then be ordered by an event; nothing else may use the workspace between
 * them).
 *   qlora_linear_adapter_fwd: H = s X A^T (X_d under dropout), into the
 *       workspace and into H_save if given.  At 16 tokens or fewer H is formed
 *       inside the decode forward instead; this call then only prepares X_d
 *       (if dropout is on), and the forward writes H_save.
 *   qlora_linear_adapter_bwd: H recomputed if H_saved is NULL (else split
 *       into its hi + lo halves) and G = s dY B.
 * Arguments as for qlora_linear_fwd_ex / qlora_linear_bwd_ex (Y, dX, dA, dB
 * omitted).  Errors as there.
 * The rest of a split backward (adapter_ready = 1) may also be divided: with
 * dA = dB = NULL it forms dX alone, with dX = NULL dA and dB alone (the weight
 * gradients need G, not dX, so they may run on another stream than dX).  The
 * undivided backward requires dA and dB (INVALID_ARG otherwise).
 */
QLORA_API qlora_status qlora_linear_adapter_fwd(const qlora_nf4_weight *w, const void *X, int64_t M, const void *A,
                                                const void *B, int32_t r, float scale, float *H_save, void *workspace,
                                                size_t workspace_bytes, void *stream, const qlora_linear_opts *opts);
QLORA_API qlora_status qlora_linear_adapter_bwd(const qlora_nf4_weight *w, const void *X, const void *dY, int64_t M,
                                                const void *A, const void *B, int32_t r, float scale,
                                                const float *H_saved, void *workspace, size_t workspace_bytes,
                                                void *stream, const qlora_linear_opts *opts);

/* Human-readable name of a status code (static string, never NULL). */
QLORA_API const char *qlora_status_string(qlora_status status);

/*
 * Synchronizes `stream`, then reads and clears the device error word of the
 * current device.  Returns QLORA_OK if no kernel recorded a failure since
 * the last call, QLORA_ERR_TIMEOUT if a bounded wait gave up, QLORA_ERR_CUDA
 * if the synchronization itself failed.
 */
QLORA_API qlora_status qlora_check_device_error(void *stream);

/*
 * Kernel timing for benchmarks.  While enabled, every kernel this library
 * launches is bracketed by two CUDA events recorded on the kernel's own
 * stream; qlora_timing_read() waits for the recorded events and returns the
 * summed device time and launch count per kernel kind since the last reset.
 * Disabled by default; enabling it adds two event records per launch.
 *   kinds: QLORA_KERNEL_* below; ms and launches have QLORA_NUM_KERNELS
 *   entries (host arrays, written).
 * qlora_launch_count() counts every kernel launch of the library since the
 * process started, whether timing is enabled or not.
 */
enum {
    QLORA_KERNEL_QUANTIZE = 0,    /* first-level quantization pass       */
    QLORA_KERNEL_DQ_ENCODE = 1,   /* double quantization of constants    */
    QLORA_KERNEL_DEQUANTIZE = 2,  /* stand-alone dequantizer             */
    QLORA_KERNEL_FWD_FUSED = 3,   /* fused dequant-GEMM, forward         */
    QLORA_KERNEL_BWD_FUSED = 4,   /* fused dequant-GEMM, input gradient  */
    QLORA_KERNEL_LOWRANK = 5,     /* H = X A^T and G = dY B products     */
    QLORA_KERNEL_WGRAD = 6,       /* dA and dB products                  */
    QLORA_KERNEL_ELEMENTWISE = 7, /* split-sum, finalize, slot resets    */
    QLORA_KERNEL_OPTIMIZER = 8,   /* AdamW update of the adapters        */
    QLORA_KERNEL_BLOCK = 9,       /* block norms, RoPE, SwiGLU           */
    QLORA_KERNEL_ATTENTION = 10,  /* block attention products, softmax   */
    QLORA_NUM_KERNELS = 11
};
QLORA_API qlora_status qlora_timing_enable(int enable);
QLORA_API qlora_status qlora_timing_reset(void);
QLORA_API qlora_status qlora_timing_read(double ms[QLORA_NUM_KERNELS], int64_t launches[QLORA_NUM_KERNELS]);
QLORA_API int64_t qlora_launch_count(void);

/*
 * qlora_debug_bounds -- the bounds-checked build (library compiled with
 * QLORA_DEBUG, libqlora_b200_debug.so).  Its kernels check every computed
 * index of a raw pointer access against the extent of the buffer the
 * arguments describe; a failed check records its source line and skips the
 * access instead of faulting.  Synchronizes the current device, then returns
 * the first recorded line (0 if no check failed since the last call) and
 * clears it; `unit` (nullable, `unit_len` bytes) receives the source file's
 * name.  Returns -1 in the ordinary build, which has no checks.
 */
QLORA_API int qlora_debug_bounds(char *unit, size_t unit_len);

/*
 * qlora_debug_bounds_selftest -- launches (on the current device, default
 * stream) one thread that evaluates a single bounds check whose index equals
 * its extent and touches no memory, so that qlora_debug_bounds() then reports
 * that check's line in api.cu.  QLORA_ERR_UNSUPPORTED in the ordinary build.
 */
QLORA_API qlora_status qlora_debug_bounds_selftest(void);

/*
 * qlora_debug_inject_stall -- failure-detection test hook (the pages describe
 * no such facility; it exists so that tests can drive the bounded-wait path
 * without faulting the GPU).  Arms a one-shot fault in the next launch of
 * one kernel family in this process:
 *   kind  QLORA_KERNEL_QUANTIZE (quantizer, bf16 input: the first warp of the
 *         first CTA does not issue its first tensor copy),
 *         QLORA_KERNEL_FWD_FUSED or QLORA_KERNEL_BWD_FUSED (the tcgen05 fused
 *         dequant-GEMMs, which run from 17 tokens on: the first
 *         dequantization warp of the first CTA skips its first arrival on the
 *         stage barrier the MMA issuer waits on),
 *         or -1 to disarm.
 *   timeout_ns  wait limit of that one launch, 1e3 .. 2e9 (the normal limit
 *         is 2 s).
 * In the armed launch the consumer's wait runs out after timeout_ns; the
 * kernel records QLORA_ERR_TIMEOUT in the device error word, tells its other
 * roles to stop, waits (bounded by the normal 2 s) for the copies and MMAs it
 * already issued, frees its tensor memory and returns.  The outputs of that
 * one call are unspecified; qlora_check_device_error() reports the timeout;
 * later calls are unaffected.  Host-only, no CUDA call.
 * Errors: QLORA_ERR_INVALID_ARG (unknown kind, limit out of range).
 */
QLORA_API qlora_status qlora_debug_inject_stall(int kind, uint64_t timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
