// eva_vq_tcgen.cuh -- the large-batch path on the fifth-generation tensor cores.
//
// The EVA summary (section 2.B) runs its array in GEMM mode where a layer is a
// real matrix product.  Here that is Y[B][N] = X[B][K] W^T with the weight
// rebuilt from the codebook, W[o][4 j + t] = WC[g(o)][WI[o][j]][t] (plus
// alpha[o][k / 128] sigma[o][k] with the 1-bit residual of the 3-bit
// SRAM-lookup article), multiplied by tcgen05.mma (kind::f16: f16 operands,
// fp32 accumulation in tensor memory).
//
// One CTA owns 128 output rows (the MMA's M) and a range of K.  Per stage of
// 64 inputs (16 sub-vectors) every thread rebuilds its row's 64 weights -- one
// 8-byte read of the bank-replicated codebook table per index -- and stores
// them into tensor memory, where the MMA reads its A operand (so the rebuilt
// weights never go through shared memory); one thread then issues the four
// M = 128 x N = Np x K = 16 MMAs of the stage against x (the B operand, in
// shared memory) and commits them to the stage's mbarrier.  Four stages of A
// rotate in tensor memory, so the rebuild of stage s + 1 overlaps the MMAs of
// stage s.  The CTA's index bytes (128 rows x 16 per stage, contiguous in the
// row-block layout) come in by one bulk copy while the kernel waits for its
// predecessor.  The split-K partial sums of the CTAs of a cluster (one row
// block, consecutive K ranges) are combined through distributed shared
// memory in a fixed order.
#pragma once
#include "eva_vq_kernels.cuh"
#include "eva_vq_tc.cuh"

namespace eva {

constexpr int kTcRows = 128;                    // rows per CTA: the MMA's M
constexpr int kTcStageSv = 16;                  // sub-vectors per stage
constexpr int kTcStageK = kTcStageSv * kD;      // 64 inputs per stage: four MMAs of K = 16
constexpr int kTcMaxBufs = 15;                  // A stages in tensor memory, at most
constexpr int kTcStageCols = kTcStageK / 2;     // 32 TMEM columns per A stage (two fp16 each)
constexpr int kTcProducerWarps = 8;             // rebuild the weights (two per TMEM lane quarter)
constexpr int kTcThreads = (kTcProducerWarps + 1) * 32;   // + one warp that issues the MMAs
constexpr int kTcXLoads = 8;                    // x chunks a thread has in flight while staging
constexpr uint32_t kTcIdxStageBytes = kTcRows * kTcStageSv;   // 2048 index bytes per stage
constexpr uint32_t kTcTabBytes = 256u * 16u * 8u;           // codebook table, 16 copies

struct TcParams {
    const uint8_t *wib;      // row-block index layout [R][KB][128][16] bytes (R = ceil(N/128), KB = J/16)
    const __half *wc;        // codebooks [G][256][4]
    const uint8_t *sg;       // row-block sign layout [R][KB][128][8] bytes (residual only)
    const __half *al;        // alpha, canonical [N][K/128] (residual only)
    const void *x;           // [B][K] fp16, or fp32 (x_f32: the rotated input of the allocation-free route)
    void *y;                 // [B][N]
    int N, K, B, Np;         // Np: tokens padded to a multiple of 16 (the MMA's N), <= 64
    int R, KB;               // row blocks, stages over K
    int Gs;                  // CTAs per row block (one cluster, Gs in 1, 2, 4, 8, 16); blockIdx.x = rb * Gs + sg
    int rows_per_cb;         // 0: one codebook; else rows per codebook (a multiple of 128)
    int x_f32, out_f32, independent;
    int resid;               // 1: add alpha * sigma to every rebuilt weight
    int *status;             // device error word (bit 2: a bounded wait of this kernel gave up)
    int wait_rounds;
    int tmem_cols;           // tensor-memory allocation: 256 (two CTAs per SM) or 512 (one)
    int nbuf;                // A stages in flight: (tmem_cols - a_col) / 32, a_col = Np rounded up to 32
#ifdef EVA_TIMELINE
    unsigned long long *timeline;   // [grid][8] %globaltimer stamps of the last run
#endif
};

// Shared-memory layout of one CTA (every CTA of a cluster uses the same
// offsets, sized for the largest K range, because peers write into the
// reduction stage).
struct TcLayout {
    uint32_t tab, idx, sgn, alp, xs, acc, stage, bar, slot, total;
    int ngmax;               // alpha groups per row held for the largest range
    uint32_t xs_sbo;         // bytes between 8-token groups of the x operand
    int kb_max;              // stages of the largest K range
};

__host__ __device__ inline TcLayout tc_layout(int KB, int Gs, int Np, int resid) {
    TcLayout L;
    L.kb_max = (KB + Gs - 1) / Gs;
    const uint32_t kc = (uint32_t)L.kb_max * kTcStageK;        // inputs of the largest range
    L.tab = 0;
    L.idx = L.tab + kTcTabBytes;
    L.sgn = L.idx + (uint32_t)L.kb_max * kTcIdxStageBytes;
    L.alp = L.sgn + (resid ? (uint32_t)L.kb_max * kTcRows * 8u : 0u);
    L.ngmax = resid ? L.kb_max / 2 + 2 : 0;
    L.xs = L.alp + (uint32_t)kTcRows * (uint32_t)L.ngmax * 2u;
    L.xs = (L.xs + 127u) & ~127u;
    L.xs_sbo = (kc / 8u) * 128u;
    // The accumulator copy [128][Np] fp32 reuses the x region once every MMA
    // has completed (or follows it when larger).
    L.acc = L.xs;
    const uint32_t xs_end = L.xs + (uint32_t)(Np / 8) * L.xs_sbo;
    const uint32_t acc_end = L.acc + (uint32_t)kTcRows * (uint32_t)Np * 4u;
    const uint32_t rpo = (uint32_t)(kTcRows / Gs);                     // rows owned per cluster rank
    L.stage = (xs_end > acc_end ? xs_end : acc_end);
    L.bar = L.stage + (uint32_t)Gs * rpo * (uint32_t)Np * 4u;
    L.bar = (L.bar + 15u) & ~15u;
    L.slot = L.bar + 8u * (2 + 2 * kTcMaxBufs);
    L.total = L.slot + 16u;
    return L;
}

template <bool RESID>
__global__ void __launch_bounds__(kTcThreads, 1) eva_tc_kernel(const TcParams p) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    [[maybe_unused]] const int eva_bid = blockIdx.x;   // timeline stamps
    const int rb = blockIdx.x / p.Gs, sg = blockIdx.x % p.Gs;
    const int kb0 = (int)((long long)p.KB * sg / p.Gs), kb1 = (int)((long long)p.KB * (sg + 1) / p.Gs);
    const int ns = kb1 - kb0;
    const TcLayout L = tc_layout(p.KB, p.Gs, p.Np, RESID ? 1 : 0);
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(eva_smem);
    const uint32_t bar_idx = sbase + L.bar, bar_done = bar_idx + 8u;
    auto bar_free = [&](int b) { return bar_idx + 16u + 8u * (uint32_t)b; };
    auto bar_full = [&](int b) { return bar_idx + 16u + 8u * (uint32_t)(kTcMaxBufs + b); };
    const int nbuf = p.nbuf;

    // ---- prologue: weights only ----
    EVA_STAMP(0);
    if (tid == 0) {
        mbar_init(bar_idx, 1);
        mbar_init(bar_done, 1);
        for (int b = 0; b < nbuf; ++b) {
            mbar_init(bar_free(b), 1);
            mbar_init(bar_full(b), kTcProducerWarps);
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(sbase + L.slot, (uint32_t)p.tmem_cols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *reinterpret_cast<const volatile uint32_t *>(eva_smem + L.slot);
    pdl_launch();
    if (p.Gs > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    if (tid == 0) {
        // This CTA's index (and sign) bytes: contiguous in the row-block layouts.
        const uint8_t *src = p.wib + ((size_t)rb * p.KB + kb0) * kTcIdxStageBytes;
        const uint32_t bytes = (uint32_t)ns * kTcIdxStageBytes;
        const uint32_t sbytes = RESID ? (uint32_t)ns * kTcRows * 8u : 0u;
        mbar_arrive_expect_tx(bar_idx, bytes + sbytes);
        for (uint32_t off = 0; off < bytes; off += 32768u)
            bulk_copy_g2s(sbase + L.idx + off, src + off, min(32768u, bytes - off), bar_idx);
        if constexpr (RESID) {
            const uint8_t *ss = p.sg + ((size_t)rb * p.KB + kb0) * kTcRows * 8u;
            for (uint32_t off = 0; off < sbytes; off += 32768u)
                bulk_copy_g2s(sbase + L.sgn + off, ss + off, min(32768u, sbytes - off), bar_idx);
        }
    }
    {
        // Codebook table: entry c, copy r at c * 128 + 8 r (lane reads copy lane % 16).
        const int cb = p.rows_per_cb ? (rb * kTcRows) / p.rows_per_cb : 0;
        const uint2 *src = reinterpret_cast<const uint2 *>(p.wc + (size_t)cb * kCent * kD);
        for (int i = tid; i < kCent * 16; i += kTcThreads) {
            const int c = i >> 4, r = i & 15;
            *reinterpret_cast<uint2 *>(eva_smem + L.tab + (uint32_t)c * 128u + 8u * (uint32_t)r) = __ldg(src + c);
        }
    }
    // alpha of the block's rows for the 128-input groups this K range touches.
    const int g_lo = (kb0 * kTcStageK) / 128;
    if (RESID) {
        const int g_hi = (kb1 * kTcStageK - 1) / 128, ng = g_hi - g_lo + 1, NG = p.K / 128;
        __half *alp = reinterpret_cast<__half *>(eva_smem + L.alp);
        for (int i = tid; i < kTcRows * ng; i += kTcThreads) {
            const int r = i / ng, gi = i - r * ng, o = rb * kTcRows + r;
            alp[r * L.ngmax + gi] = o < p.N ? p.al[(size_t)o * NG + g_lo + gi] : __float2half(0.f);
        }
    }

    if (!p.independent) pdl_wait();
    if (p.Gs > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    EVA_STAMP(1);

    // ---- x: the B operand, K-major core matrices of 8 tokens x 8 inputs ----
    // A warp moves 8 tokens x 4 consecutive chunks of 8 inputs: lane l takes
    // token 8 g8 + (l & 7), chunk 4 c4 + (l >> 3), so its global read is 64
    // contiguous bytes per token and its shared-memory write 512 contiguous
    // bytes (four core matrices, no bank conflict).  Every thread issues its
    // loads (up to kTcXLoads) before it stores any: one round trip to L2.
    {
        const int kbase = kb0 * kTcStageK, kc8 = ns * (kTcStageK / 8), kc4 = kc8 / 4, total = p.Np * kc8;
        for (int i0 = 0; i0 < total; i0 += kTcThreads * kTcXLoads) {
            uint4 v[kTcXLoads];
#pragma unroll
            for (int u = 0; u < kTcXLoads; ++u) {
                const int i = i0 + u * kTcThreads + tid;
                const int q = i >> 5, g8 = q / kc4, c4 = q - g8 * kc4;
                const int n = 8 * g8 + (lane & 7), c8 = 4 * c4 + (lane >> 3);
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (i < total && n < p.B) {
                    const size_t e = (size_t)n * p.K + kbase + 8 * c8;
                    if (p.x_f32) {
                        const float4 *xp = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p.x) + e);
                        const float4 a = __ldcg(xp), b = __ldcg(xp + 1);
                        v[u] = make_uint4(pack_half2(a.x, a.y), pack_half2(a.z, a.w), pack_half2(b.x, b.y),
                                          pack_half2(b.z, b.w));
                    } else {
                        v[u] = __ldcg(reinterpret_cast<const uint4 *>(reinterpret_cast<const __half *>(p.x) + e));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kTcXLoads; ++u) {
                const int i = i0 + u * kTcThreads + tid;
                if (i >= total) break;
                const int q = i >> 5, g8 = q / kc4, c4 = q - g8 * kc4;
                const int n = 8 * g8 + (lane & 7), c8 = 4 * c4 + (lane >> 3);
                *reinterpret_cast<uint4 *>(eva_smem + L.xs + (uint32_t)(n >> 3) * L.xs_sbo + (uint32_t)c8 * 128u +
                                           (uint32_t)(n & 7) * 16u) = v[u];
            }
        }
    }
    // Make the x stage visible to the tensor cores (generic -> async proxy).
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    bool ok = mbar_wait_bounded(bar_idx, 0, p.wait_rounds);
    EVA_STAMP(2);

    const uint32_t idesc = tc::idesc_f16_f32(kTcRows, p.Np);
    const uint32_t acc_col = 0, a_col = (uint32_t)((p.Np + 31) & ~31);
    const int q4 = warp & 3, half = (warp >> 2) & 1;   // TMEM lane quarter; sub-vectors 8 half .. + 7 of a stage
    const int row = q4 * 32 + lane;                    // this thread's row within the block (producers)
    // Producers rebuild stage st into A buffer st % 4 and signal full[buf];
    // the MMA thread waits for it, issues the stage's four MMAs and commits
    // them to free[buf], which the producers wait for before the buffer's
    // next use.  No block-wide barrier inside the loop.
    if (warp < kTcProducerWarps) {
        const uint32_t lofs = 8u * (uint32_t)(lane & 15);
        for (int st = 0; st < ns; ++st) {
            const int buf = st % nbuf;
            if (st >= nbuf) ok &= mbar_wait_bounded(bar_free(buf), (uint32_t)((st / nbuf - 1) & 1), p.wait_rounds);
            tc::fence_after_sync();
            // Rebuild 8 sub-vectors (32 inputs) of this thread's row.
            const uint4 iv = *reinterpret_cast<const uint4 *>(eva_smem + L.idx + (uint32_t)st * kTcIdxStageBytes +
                                                               16u * (uint32_t)row);
            const uint32_t w0 = half ? iv.z : iv.x, w1 = half ? iv.w : iv.y;
            uint32_t a[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t c = ((e < 4 ? w0 : w1) >> (8 * (e & 3))) & 0xFFu;
                const uint2 cw = *reinterpret_cast<const uint2 *>(eva_smem + L.tab + (c << 7) + lofs);
                a[2 * e] = cw.x;
                a[2 * e + 1] = cw.y;
            }
            if (RESID) {
                // sigma bits of the row's 32 inputs (LSB first), alpha of their 128-group.
                const uint32_t sb = *reinterpret_cast<const uint32_t *>(eva_smem + L.sgn + (uint32_t)st * kTcRows * 8u +
                                                                        8u * (uint32_t)row + 4u * (uint32_t)half);
                const int k0 = (kb0 + st) * kTcStageK + 32 * half;
                const __half al = reinterpret_cast<const __half *>(eva_smem + L.alp)[row * L.ngmax + k0 / 128 - g_lo];
                const __half2 ap = __halves2half2(al, al), an = __hneg2(ap);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const uint32_t two = (sb >> (2 * e)) & 3u;
                    const __half2 sgn = __halves2half2((two & 1u) ? __low2half(ap) : __low2half(an),
                                                       (two & 2u) ? __low2half(ap) : __low2half(an));
                    __half2 w = *reinterpret_cast<const __half2 *>(&a[e]);
                    w = __hadd2(w, sgn);
                    a[e] = *reinterpret_cast<const uint32_t *>(&w);
                }
            }
            tc::tmem_st16(tc::taddr(tbase, (uint32_t)(q4 * 32), a_col + (uint32_t)buf * kTcStageCols + 16u * (uint32_t)half),
                          a);
            tc::tmem_st_wait();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_full(buf));
        }
    } else if (lane == 0) {
        for (int st = 0; st < ns; ++st) {
            const int buf = st % nbuf;
            ok &= mbar_wait_bounded(bar_full(buf), (uint32_t)((st / nbuf) & 1), p.wait_rounds);
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t ta = tc::taddr(tbase, 0, a_col + (uint32_t)buf * kTcStageCols + 8u * (uint32_t)kk);
                const uint32_t bo = L.xs + (uint32_t)(st * (kTcStageK / 8) + 2 * kk) * 128u;
                const uint64_t bd = tc::sdesc_kmajor_noswizzle(sbase + bo, 128u, L.xs_sbo);
                tc::mma_ts_f16(tbase + acc_col, ta, bd, idesc, (st > 0 || kk > 0) ? 1u : 0u);
            }
            tc::commit(bar_free(buf));
        }
        tc::commit(bar_done);
    }
    EVA_STAMP(3);
    ok &= mbar_wait_bounded(bar_done, 0, p.wait_rounds);
    tc::fence_after_sync();
    EVA_STAMP(4);
    // ---- accumulator -> shared memory, token-major [Np][128] fp32 ----
    // (thread = row: consecutive threads write consecutive words)
    float *acc = reinterpret_cast<float *>(eva_smem + L.acc);
    if (warp < 4) {
        for (int c0 = 0; c0 < p.Np; c0 += 8) {
            float v[8];
            tc::tmem_ld8(tc::taddr(tbase, (uint32_t)(warp * 32), acc_col + (uint32_t)c0), v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[(c0 + e) * kTcRows + row] = v[e];
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tbase, (uint32_t)p.tmem_cols);
    }
    if (!ok && p.status) atomicOr(p.status, 4);

    EVA_STAMP(5);
    // ---- split-K: rows [rpo r, rpo (r + 1)) belong to cluster rank r (Gs
    // divides 128, so rpo is a multiple of 8); the owner's stage is
    // [Gs sources][Np tokens][rpo rows] ----
    const int rpo = kTcRows / p.Gs;
    if (p.Gs > 1) {
        const uint32_t stage_addr = sbase + L.stage;
        for (int i = tid; i < p.Np * (kTcRows / 4); i += kTcThreads) {
            const int b = i / (kTcRows / 4), r = 4 * (i - b * (kTcRows / 4));
            const int owner = r / rpo, rl = r - owner * rpo;
            const float4 v = *reinterpret_cast<const float4 *>(acc + b * kTcRows + r);
            const uint32_t dst = (uint32_t)(((sg * p.Np + b) * rpo + rl) * 4);
            st_dsmem_v4(stage_addr + dst, (uint32_t)owner, v);
        }
        cluster_sync_all();
    }
    {
        const int r0 = sg * rpo, nr = rpo;
        const float *stage = reinterpret_cast<const float *>(eva_smem + L.stage);
        for (int i = tid; i < nr * p.B; i += kTcThreads) {
            const int rl = i % nr, b = i / nr;
            const int o = rb * kTcRows + r0 + rl;
            if (o >= p.N) continue;
            float sum;
            if (p.Gs > 1) {
                sum = 0.f;
                for (int k = 0; k < p.Gs; ++k) sum += stage[(k * p.Np + b) * rpo + rl];
            } else {
                sum = acc[b * kTcRows + rl];
            }
            const size_t yi = (size_t)b * p.N + o;
            if (p.out_f32) reinterpret_cast<float *>(p.y)[yi] = sum;
            else reinterpret_cast<__half *>(p.y)[yi] = __float2half_rn(sum);
        }
    }
    if (p.independent) pdl_wait();
    EVA_STAMP(6);
#ifdef EVA_TIMELINE
    if (tid == 0) {
        unsigned smid;
        asm volatile("mov.u32 %0, %smid;" : "=r"(smid));
        p.timeline[eva_bid * 8 + 7] = smid;
    }
#endif
}

// Create-time repack of canonical WI [N][J] into the row-block layout
// [R][J/16][128][16]; rows >= N are 0.
__global__ void eva_repack_wi_rowblock_kernel(const uint8_t *__restrict__ wi, uint8_t *__restrict__ out, int N, int J,
                                              long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int KB = J / kTcStageSv;
    const int e = (int)(idx & 15);
    const long long r_all = idx >> 4;                 // (rb * KB + kb) * 128 + r
    const int r = (int)(r_all % kTcRows);
    const long long blk = r_all / kTcRows;
    const int kb = (int)(blk % KB), rb = (int)(blk / KB);
    const int o = rb * kTcRows + r, j = kb * kTcStageSv + e;
    out[idx] = o < N ? wi[(size_t)o * J + j] : (uint8_t)0;
}

// Signs [N][K/8] into [R][J/16][128][8] (the 64 inputs of a stage: 8 bytes per row).
__global__ void eva_repack_signs_rowblock_kernel(const uint8_t *__restrict__ sg, uint8_t *__restrict__ out, int N,
                                                 int K8, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int KB = K8 / 8;
    const int e = (int)(idx & 7);
    const long long r_all = idx >> 3;
    const int r = (int)(r_all % kTcRows);
    const long long blk = r_all / kTcRows;
    const int kb = (int)(blk % KB), rb = (int)(blk / KB);
    const int o = rb * kTcRows + r, m = kb * 8 + e;
    out[idx] = o < N ? sg[(size_t)o * K8 + m] : (uint8_t)0;
}

}  // namespace eva
