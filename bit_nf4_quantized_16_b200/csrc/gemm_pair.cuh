// Fused dequant-GEMM on a tcgen05 CTA pair (cta_group::2) for sm_100a.
//
// Two CTAs of a cluster form one MMA unit: the leader issues
// tcgen05.mma.cta_group::2 with M = 256, taking 128 rows of A from each CTA's
// shared memory and splitting the N = 256 columns of B between them, and D
// lands in both CTAs' tensor memory.  Each CTA therefore stages only half of
// the dequantized weight tile and reads half of the B operand per MMA, which
// halves the shared-memory traffic of both the expansion and the MMA compared
// with a single CTA computing the same 256 x 256 block.
//
// Tile of one pair: (2 * MT * 128) tokens x 256 features of W (forward) or
// of W's columns (input gradient); MT accumulators of 128 rows per CTA.
// The weight is expanded exactly as in the stand-alone dequantizer
// ("QLoRA: Efficient Finetuning of Quantized LLMs", section "Method": the
// stored weight is dequantized to BFloat16 and multiplied in 16-bit); the
// bf16 tile never reaches HBM.
//
// Synchronization (every wait bounded, as in gemm.cuh):
//   full_a[s]   leader; TMA bytes of A (and LoRA B) of both CTAs
//   pk_full[s]  per CTA; this CTA's packed codes landed
//   full_b[s]   leader; expansion finished in both CTAs (16 warp arrivals)
//   empty[s]    per CTA; the pair's MMAs that read stage s completed (multicast commit)
//   acc_full    per CTA; accumulators ready (multicast commit)
//   acc_empty   leader; both CTAs' epilogues drained the accumulators (16 warp arrivals)
// Roles per CTA: warp 0 TMA, warp 1 MMA (leader only) and TMEM allocation,
// warps 8..15 dequantization, warps 4..7 and 16..19 epilogue (two warps per
// TMEM lane quadrant, each half of the columns; bf16 results leave through a
// shared-memory box and a TMA store).
// No load uses cluster multicast.
#pragma once
#include "gemm.cuh"

namespace qlora {

template <int kBMode, int MT>
struct PairCfg {
    static_assert(kBMode == kBNf4K || kBMode == kBNf4MN, "pair kernel is for the fused modes");
    static constexpr int BNC = 128;   // weight columns of B per CTA
    static constexpr int NP = 2 * BNC; // MMA N of the pair
    static constexpr int kDeqWarps = 8;
    static constexpr int kEpiWarps = 8;  // warps 4..7 and 16..19: two per TMEM lane quadrant
    static constexpr int kThreads = 256 + 32 * kDeqWarps + 32 * (kEpiWarps - 4);
    static constexpr uint32_t kABytes = MT * 128 * 64 * 2;
    static constexpr uint32_t kBBytes = BNC * 64 * 2;
    static constexpr uint32_t kPBytes = BNC * 32;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes + kPBytes;
    static constexpr int kMaxStages = (232448 - 2048) / kStageBytes;
    static constexpr int kStages = kMaxStages > 6 ? 6 : kMaxStages;
    static constexpr uint32_t kBarOff = kStages * kStageBytes;
    // bf16 epilogue staging: one 32 x 32 bf16 box (2 KB) per epilogue warp
    static constexpr uint32_t kEpiOff = kBarOff + 1024;
    static constexpr uint32_t kEpiBoxBytes = 32 * 32 * 2;
    static constexpr uint32_t kEpiBytes = kEpiWarps * kEpiBoxBytes;
    static constexpr uint32_t kSmemBytes = kEpiOff + kEpiBytes + 1024;
    static constexpr uint32_t kAccCols = MT * NP;
    static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
    static constexpr uint32_t kTmemCols = kAccBufs * kAccCols;
    static constexpr int kTPB = (32 * kDeqWarps) / BNC;   // threads per quantization block
    static_assert(kTmemCols <= 512, "accumulators must fit in TMEM");
    static_assert(kStages >= 2, "shared memory too small");
    static_assert(kSmemBytes + 64 <= 232448, "shared memory per block");
};

template <int kBMode, int kEpi, int MT, bool F16 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<kBMode, MT>::kThreads, 1)
    qgemm_pair_kernel(const __grid_constant__ GemmParams p)
{
    using Cfg = PairCfg<kBMode, MT>;
    using namespace sm100;
    using namespace gemm_detail;
    constexpr int S = Cfg::kStages;
    constexpr int BNC = Cfg::BNC;
    constexpr int NP = Cfg::NP;
    constexpr int BMC = 128 * MT;   // token rows per CTA
    constexpr bool kBMn = kBMode == kBNf4MN;

    extern __shared__ uint8_t smem_raw[];
    __shared__ float lut[16];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_a = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
    uint64_t *pk_full = full_a + S;
    uint64_t *full_b = pk_full + S;
    uint64_t *empty = full_b + S;
    uint64_t *acc_full = empty + S;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    auto sA = [&](int s) { return smem + s * Cfg::kABytes; };
    auto sB = [&](int s) { return smem + S * Cfg::kABytes + s * Cfg::kBBytes; };
    auto sP = [&](int s) { return smem + S * (Cfg::kABytes + Cfg::kBBytes) + s * Cfg::kPBytes; };
    // the leader's copy of a barrier (shared::cluster address)
    auto at_leader = [&](uint64_t *bar) { return mapa_shared(smem_u32(bar), 0); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full_a[s], 1);
            mbar_init(&pk_full[s], 1);
            mbar_init(&full_b[s], 2 * Cfg::kDeqWarps);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * Cfg::kEpiWarps);
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
        if (kEpi == kEpiBf16) tma_prefetch_desc(&p.tm_out);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // barriers of both CTAs initialized before any remote arrive
    tc_fence_after();
    // everything above overlaps the previous kernel's tail; inputs are read below
    pdl_wait();
    pdl_trigger();
    const uint32_t tmem_base = *tmem_slot;
    const int num_tiles = p.m_tiles * p.n_tiles;
    const int cluster_id = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;
    volatile int *vabort = abort_flag;

    auto decode = [&](int t, int &mt, int &nt) {
        mt = t % p.m_tiles;
        nt = t / p.m_tiles;
    };
    const int nst_tile = p.k_stages_total + p.k_stages_lora;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        uint32_t it = 0;
        const uint32_t full_a_leader0 = at_leader(&full_a[0]);
        for (int t = cluster_id; t < num_tiles && !*vabort; t += num_clusters) {
            int mt, nt;
            decode(t, mt, nt);
            const int m0 = mt * 2 * BMC + (int)rank * BMC;       // this CTA's token rows
            const int n0 = nt * NP + (int)rank * BNC;            // this CTA's weight columns
            for (int ks = 0; ks < nst_tile; ks++, it++) {
                const int s = it % S;
                const uint32_t use = it / S;
                if (!mbar_wait_bounded(&empty[s], (use & 1) ^ 1, p.timeout_ns)) {
                    record_timeout(p, abort_flag);
                    break;
                }
                if (*vabort) break;
                const uint32_t fa = full_a_leader0 + (uint32_t)s * 8u;
                if (ks < p.k_stages_total) {
                    const int k0 = ks * 64;
                    mbar_arrive_expect_tx(&pk_full[s], Cfg::kPBytes);
                    if (kBMode == kBNf4K)
                        tma_load_2d(sP(s), &p.tm_b, &pk_full[s], k0 / 2, n0);     // [BNC rows][32 B]
                    else
                        tma_load_2d(sP(s), &p.tm_b, &pk_full[s], n0 / 2, k0);     // [64 rows][BNC/2 B]
                    if (leader) mbar_arrive_expect_tx(&full_a[s], 2 * Cfg::kABytes);
                    tma_load_2d_pair(sA(s), &p.tm_a, fa, k0, m0);
                } else {
                    const int r0 = (ks - p.k_stages_total) * 64;
                    mbar_arrive(&pk_full[s]);   // nothing to expand: lets the dequant warps move on
                    if (leader) mbar_arrive_expect_tx(&full_a[s], 2 * (Cfg::kABytes + Cfg::kBBytes));
                    tma_load_2d_pair(sA(s), &p.tm_a2, fa, (ks - p.k_stages_total) * p.a2_x_step, m0);
                    if (kBMn) {
#pragma unroll
                        for (int j = 0; j < BNC / 64; j++) tma_load_2d_pair(sB(s) + 8192 * j, &p.tm_b2, fa, n0 + 64 * j, r0);
                    } else {
                        tma_load_2d_pair(sB(s), &p.tm_b2, fa, r0, n0);
                    }
                }
            }
        }
        if (*vabort) {
            // after an abort: wait (bounded) for the loads still in flight; the
            // leader's full_a also counts the other CTA's bytes
            for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; j++) {
                mbar_wait_bounded(&pk_full[j % S], (j / S) & 1, p.drain_ns);
                if (leader) mbar_wait_bounded(&full_a[j % S], (j / S) & 1, p.drain_ns);
            }
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // ---------------- MMA issuer (leader only) ----------------
        const uint32_t idesc = idesc_bf16_f32(256, NP, 0, kBMn ? 1 : 0, F16);
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int t = cluster_id; t < num_tiles && ok && !*vabort; t += num_clusters, local++) {
            const uint32_t buf = local % Cfg::kAccBufs, ause = local / Cfg::kAccBufs;
            if (!mbar_wait_bounded_cluster(&acc_empty[buf], (ause & 1) ^ 1, p.timeout_ns)) {
                record_timeout(p, abort_flag);
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + buf * Cfg::kAccCols;
            for (int ks = 0; ks < nst_tile; ks++, it++) {
                const int s = it % S;
                const uint32_t use = it / S;
                if (!mbar_wait_bounded(&full_a[s], use & 1, p.timeout_ns) ||
                    !mbar_wait_bounded_cluster(&full_b[s], use & 1, p.timeout_ns)) {
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
                        const uint64_t adesc = smem_desc_sw128(a_addr + m * 16384 + 32 * kk, 16, 1024);
                        tc_mma_bf16_pair(d_tmem + m * NP, adesc, bdesc, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc_commit_pair(&empty[s], 0x3);
            }
            if (!ok) break;
            tc_commit_pair(&acc_full[buf], 0x3);
        }
        if (*vabort) {
            tc_commit_pair(drain, 0x1);
            mbar_wait_bounded(drain, 0, p.drain_ns);
        }
    } else if ((warp >= 4 && warp < 8) || warp >= 16) {
        // ---------------- epilogue (both CTAs) ----------------
        // warp (q, h): TMEM lanes 32q..32q+31, columns [h * NP/2, (h+1) * NP/2) of each accumulator
        const int q = warp & 3;
        const int h = warp >= 16 ? 1 : 0;
        const uint32_t acc_empty_leader = at_leader(&acc_empty[0]);
        uint8_t *box = smem + Cfg::kEpiOff + (h * 4 + q) * Cfg::kEpiBoxBytes;
        uint32_t epi_it = 0;   // boxes stored by this warp
        uint32_t local = 0;
        for (int t = cluster_id; t < num_tiles && !*vabort; t += num_clusters, local++) {
            int mt, nt;
            decode(t, mt, nt);
            const uint32_t buf = local % Cfg::kAccBufs, ause = local / Cfg::kAccBufs;
            if (!mbar_wait_bounded(&acc_full[buf], ause & 1, p.timeout_ns)) {
                record_timeout(p, abort_flag);
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int m = 0; m < MT; m++) {
                const int row0 = mt * 2 * BMC + (int)rank * BMC + m * 128 + 32 * q;
                const int row = row0 + lane;
                const bool row_ok = row < p.m_total;
#pragma unroll 1
                for (int c = h * (NP / 64); c < (h + 1) * (NP / 64); c++) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + buf * Cfg::kAccCols + m * NP + 32 * c, r);
                    tmem_ld_wait();
                    const int col0 = nt * NP + 32 * c;
                    if (kEpi == kEpiBf16) {
                        // stage the warp's 32 x 32 box in shared memory (64-byte swizzle:
                        // 16-byte chunk j of row i at j ^ ((i >> 1) & 3)), then one TMA
                        // store; the tensor map clips rows and columns past the end
                        if (row0 >= p.m_total || col0 >= p.n_total) continue;
                        if (epi_it >= 1) {
                            // the previous box's store must have read the staging buffer
                            if (lane == 0) bulk_wait_group_read<0>();
                            __syncwarp();
                        }
#pragma unroll
                        for (int g = 0; g < 4; g++) {
                            uint4 v;
                            v.x = nf4::pack16x2<F16>(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]));
                            v.y = nf4::pack16x2<F16>(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
                            v.z = nf4::pack16x2<F16>(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]));
                            v.w = nf4::pack16x2<F16>(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
                            *reinterpret_cast<uint4 *>(box + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4)) = v;
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&p.tm_out, box, col0, row0);
                            bulk_commit_group();
                        }
                        epi_it++;
                    } else {
                        if (!row_ok) continue;
                        float *o = static_cast<float *>(p.out) + (int64_t)row * p.out_ld + col0;
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
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader + buf * 8u);
        }
        // the staging buffers must stay valid until the last stores have read them
        if (kEpi == kEpiBf16 && lane == 0) bulk_wait_group_all();
    } else if (warp >= 8 && warp < 16) {
        // ---------------- dequantization producer (both CTAs) ----------------
        // This CTA expands BNC of the pair's 256 weight columns: forward stages
        // are BNC rows of W x 64 columns, input-gradient stages 64 rows x BNC
        // columns; BNC quantization blocks per stage, kTPB threads per block.
        constexpr int TPB = Cfg::kTPB;
        constexpr int WPT = 8 / TPB;
        const int dt = (warp - 8) * 32 + lane;
        const int blk = dt / TPB, part = dt % TPB;
        const float mu = *p.mean;
        const uint32_t full_b_leader0 = at_leader(&full_b[0]);
        uint32_t it = 0;
        for (int t = cluster_id; t < num_tiles && !*vabort; t += num_clusters) {
            int mt, nt;
            decode(t, mt, nt);
            const int ntc = nt * 2 + (int)rank;   // this CTA's BNC-wide column tile
            auto block_of = [&](int ks, int64_t &n, int64_t &kb) {
                if (kBMode == kBNf4K) {
                    n = (int64_t)ntc * BNC + blk;
                    kb = ks;
                } else {
                    n = (int64_t)ks * 64 + (blk & 63);
                    kb = (int64_t)ntc * (BNC / 64) + (blk >> 6);
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
            const int nmain = p.k_stages_total;
            constexpr int kPre = 4;
            uint8_t qe[kPre];
            float qc2[kPre];
            bool qok[kPre];
#pragma unroll
            for (int i = 0; i < kPre; i++) qok[i] = i < nmain && load_raw(i, qe[i], qc2[i]);
            bool ok = true;
            for (int ks = 0; ks < nst_tile; ks++, it++) {
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
                if (!mbar_wait_bounded(&pk_full[s], use & 1, p.timeout_ns)) {
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
                    if (kBMode == kBNf4K) {
                        // packed tile [BNC rows][32 B], 32-byte swizzle: chunk h at h ^ ((row >> 2) & 1)
                        r = blk;
                        const int sw = (r >> 2) & 1;
#pragma unroll
                        for (int h = 0; h < 2 / TPB; h++) {
                            const int chunk = part * (2 / TPB) + h;
                            const uint4 v = *reinterpret_cast<const uint4 *>(pb + r * 32 + ((chunk ^ sw) << 4));
                            words[4 * h + 0] = v.x; words[4 * h + 1] = v.y; words[4 * h + 2] = v.z; words[4 * h + 3] = v.w;
                        }
                        dst = bb + r * 128;
                    } else {
                        // packed tile [64 rows][BNC/2 B], 64-byte swizzle of its 16-byte chunks
                        r = blk & 63;
                        const int c = blk >> 6;
#pragma unroll
                        for (int h = 0; h < 2 / TPB; h++) {
                            const int chunk = 2 * c + part * (2 / TPB) + h;
                            const int pos = chunk ^ ((r >> 1) & 3);
                            const uint4 v = *reinterpret_cast<const uint4 *>(pb + r * (BNC / 2) + (pos << 4));
                            words[4 * h + 0] = v.x; words[4 * h + 1] = v.y; words[4 * h + 2] = v.z; words[4 * h + 3] = v.w;
                        }
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
                if (lane == 0 && !skip) mbar_arrive_cluster(full_b_leader0 + (uint32_t)s * 8u);
            }
            if (!ok) break;
        }
    }

    __syncthreads();
    cluster_sync();   // both CTAs done with the pair's tensor memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace qlora
