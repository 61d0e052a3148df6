// eva_vq_dequant.cuh -- the dequantize-to-tensor-core path for larger batches.
//
// The output-codebook lookups of the EVA summary (section 2.A) cost one
// shared-memory read per index and token pair, so they grow with the batch.
// The alternative the EVA summary's GEMM mode stands for: rebuild the weight
// from the codebook (WC[WI], one 8-byte read per index whatever the batch)
// and let tensor-core MMAs (m16n8k16, f16 in, fp32 accumulate) multiply it
// with up to 16 tokens at a time.  Layers with a shared codebook or one
// codebook per group of rows; with one shared codebook also the 1-bit sign
// residual (w = WC[WI] + alpha sigma, added to the rebuilt pair before its
// MMA) and a rotated input (x~ in fp32 from the rotation kernel).
//
// Same repacked index units and the same CTA grid as the lookup kernel
// (clusters of Gs slice groups x Gt row groups, split-K sums combined in
// distributed shared memory).  Per lane the index bytes of a unit are
// rotated so that MMA block beta (16 inputs = 4 sub-vectors) reads, for lane
// (g, q), sub-vector 4 beta + q (beta < 8) or 4 (beta - 8) + q + 32: the k
// order inside a block is permuted identically in A (the weights) and B (x),
// which leaves the product unchanged.  A fragment: the four fp16 components
// of the lane's centroid for rows g and g + 8, read from a codebook table
// replicated 16 times across the banks (conflict-free); B fragment: the same
// sub-vector of token g, kept in registers for a whole slice.
#pragma once
#include "eva_vq_kernels.cuh"

namespace eva {

constexpr uint32_t kTabBytes = kCent * 16u * 8u;      // 256 centroids x 16 copies x 8 bytes
constexpr uint32_t kXTokStride = 544u;                // bytes per staged token (512 + 32: conflict-free)


// signs [N][K/8] (bit k % 8 of byte k / 8: input k, LSB first) -> sign units.
__global__ void eva_repack_signs_dq_kernel(const uint8_t *__restrict__ sg, uint8_t *__restrict__ out, int N,
                                           int K, int T, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long unit = idx / kDqSignUnitBytes;
    const int b = (int)(idx % kDqSignUnitBytes);
    const int s = (int)(unit / T), tile = (int)(unit % T);
    uint32_t v = 0;
    for (int t = 0; t < 8; ++t) {
        int row, kin;
        dq_sign_pos(b, t, row, kin);
        const int o = kTileRows * tile + row, k = kSliceK * s + kin;
        if (o < N && k < K) v |= (uint32_t)((sg[(size_t)o * (K / 8) + (k >> 3)] >> (k & 7)) & 1u) << t;
    }
    out[idx] = (uint8_t)v;
}

__device__ __forceinline__ uint2 lds64(uint32_t off) { return *reinterpret_cast<const uint2 *>(eva_smem + off); }

// Codebook cb replicated: entry c, copy r at c * 128 + 8 r (r = lane mod 16).
__device__ __forceinline__ void build_codebook_table(const LookupParams &p, int cb, int tid) {
    const uint2 *src = reinterpret_cast<const uint2 *>(p.wc + (size_t)cb * kCent * kD);
    for (int i = tid; i < kCent * 16; i += kThreads) {
        const int c = i >> 4, r = i & 15;
        const uint32_t off = (uint32_t)c * 128u + 8u * (uint32_t)r;
        if (!EVA_BAD_G(BUF_WC, src + c, 8) && !EVA_BAD_S(off) && !EVA_BAD_S(off + 4u))
            *reinterpret_cast<uint2 *>(eva_smem + off) = __ldg(src + c);
    }
}

// x~[ks + 8 lane .. + 7] of token tok for a Sylvester rotation block b
// (p.rot_b), x~ = s . (H_b x) / sqrt(b), computed by one warp from fp16 x:
// b <= 256, the slice holds whole blocks (warp transform of stages < b);
// b > 256, H_b = H_{b/256} (x) H_256, so the slice (sub-block a of its block)
// is sum_sb (-1)^popc(sb & a) H_256 x_sb over the block's sub-blocks, four
// sub-blocks' loads in flight at a time.  Zeros past B and past K.
__device__ __forceinline__ void dq_rotated_x8(const LookupParams &p, int tok, int ks, int lane, float (&acc)[8]) {
    const int b = p.rot_b;
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    if (tok >= p.B) return;
    if (b <= kSliceK) {
        load_x8_f16(p, tok, ks + 8 * lane, acc);
        fwht_warp256(acc, lane, b);
    } else {
        const int nsb = b / kSliceK, blk0 = (ks / b) * b, a = (ks - blk0) / kSliceK;
        for (int sb0 = 0; sb0 < nsb; sb0 += 4) {
            float v[4][8];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (sb0 + u < nsb) {
                    load_x8_f16(p, tok, blk0 + (sb0 + u) * kSliceK + 8 * lane, v[u]);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[u][j] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (sb0 + u >= nsb) break;
                fwht_warp256(v[u], lane, kSliceK);
                const bool neg = (__popc((unsigned)((sb0 + u) & a)) & 1) != 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = neg ? acc[j] - v[u][j] : acc[j] + v[u][j];
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int k = ks + 8 * lane + j;
        acc[j] *= (k < p.K ? (float)p.hs[k] : 0.f) * p.rot_scale;
    }
}

// DIRECT: launched only when every CTA takes one K-slice (Gs = S), so a
// tile's sums are final when its MMAs end and go straight from registers to
// the owning cluster CTA's stage (no running sums in shared memory).
// Two CTAs per SM where the registers allow it without spills (at most 128
// a thread): then the next layer's CTA runs its prologue beside this one.
// The 16-token instances with running sums in shared memory take more than
// half the SM's shared memory anyway, so they keep one CTA per SM and the
// registers that go with it.  The residual instances follow the same rule
// (124-128 registers where it asks for two CTAs per SM, no spills).
template <bool GROUPED, int NTG, bool DIRECT, bool RESID = false>
constexpr int kDequantMinBlocks = (NTG == 2 && (GROUPED || !DIRECT)) ? 1 : 2;

// The whole per-CTA program; eva_bid is the CTA's index within its layer.
// RESID: the 1-bit sign residual of the 3-bit SRAM-lookup article rides on
// the rebuilt weights, w = WC[WI] + alpha sigma (one shared codebook); a
// rotated layer's x~ comes in as fp32 (x_f32) from the rotation kernel.
template <bool GROUPED, int NTG, bool DIRECT, bool RESID = false>
__device__ __forceinline__ void dequant_body(const LookupParams &p, const int eva_bid) {
    static_assert(!(RESID && GROUPED), "the residual rides on one shared codebook");
    constexpr int TT = 8 * NTG;                         // tokens per pass
    constexpr uint32_t BLK = kTileRows * TT * 4u;       // bytes of one tile's running sums
    // A tile's block in the reduction stage.  Sums pushed from registers (8
    // bytes a lane): rows TT + 2 floats apart, so the owners' reads (row
    // fastest, for coalesced y stores) hit distinct banks; running-sum blocks
    // copied 16 bytes at a time: rows TT floats apart, like the running sums.
    constexpr int RS = DIRECT ? TT + 2 : TT;
    constexpr uint32_t BLK_S = kTileRows * RS * 4u;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int ts = eva_bid % p.Gs, tt = eva_bid / p.Gs;
    const int s0 = (int)((long long)p.S * ts / p.Gs), s1 = (int)((long long)p.S * (ts + 1) / p.Gs);
    const int t0 = (int)((long long)p.T * tt / p.Gt), t1 = (int)((long long)p.T * (tt + 1) / p.Gt);
    const int ntw = (t1 - t0 - warp + kWarps - 1) / kWarps;
    const int nsl = s1 - s0, ctiles = t1 - t0;
    const int cb_first = GROUPED ? t0 / p.tiles_per_cb : 0;
    const int cb_last = GROUPED ? (t1 - 1) / p.tiles_per_cb : 0;

    // Shared memory: codebook table | x stage [slice][token] | running sums
    // [tile][16][TT] (only when a CTA takes several slices) | reduction stage
    // [ceil(acc_tiles / Gs)][Gs][16][TT] | the staging mbarrier (128 bytes) |
    // the staged index units (slice-major: unit sl * ctiles + tl) | with the
    // residual, the same units' signs, then their alphas.
    constexpr uint32_t TAB_OFF = 0, XS_OFF = kTabBytes;
    // The layout must be the same in every CTA of a cluster (peers write into
    // the reduction stage at this CTA's offsets): size the x stage for the
    // largest slice count, ceil(S / Gs).
    const int nsl_max = (p.S + p.Gs - 1) / p.Gs;
    constexpr bool direct = DIRECT;
    const uint32_t ACC_OFF = (XS_OFF + (uint32_t)(nsl_max * TT) * kXTokStride + 127u) & ~127u;
    const uint32_t STAGE_OFF = ACC_OFF + (direct ? 0u : (uint32_t)p.acc_tiles * BLK);
    float *acc_s = reinterpret_cast<float *>(eva_smem + ACC_OFF);
    const float *stage = reinterpret_cast<const float *>(eva_smem + STAGE_OFF);
    const uint32_t stage_addr = (uint32_t)__cvta_generic_to_shared(eva_smem + STAGE_OFF);
    const uint32_t BAR_OFF = (STAGE_OFF + (uint32_t)((p.acc_tiles + p.Gs - 1) / p.Gs) * p.Gs * BLK_S + 127u) & ~127u;
    const uint32_t UNITS_OFF = BAR_OFF + 128u;
    const int nst = min(nsl * ctiles, p.wi_staged);   // units copied into shared memory
    const uint32_t SG_OFF = UNITS_OFF + (uint32_t)nst * kUnitBytes;
    const uint32_t AL_OFF = SG_OFF + (uint32_t)nst * kDqSignUnitBytes;
    constexpr uint32_t kStagedUnitBytes = kUnitBytes + (RESID ? kDqResidUnitBytes : 0);
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(eva_smem + BAR_OFF);

    // ---- prologue: weights only ----
    EVA_STAMP(0);
    pdl_launch();
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    // The CTA's first nst index units: bulk copies into shared memory, one per
    // slice (a slice's units of this CTA are contiguous), on one mbarrier.
    if (tid == 0 && nst > 0) {
        mbar_init(bar, 1);
        if (!p.skip_stage_copy && !EVA_BAD_S(UNITS_OFF) &&
            !EVA_BAD_S(UNITS_OFF + (uint32_t)nst * kStagedUnitBytes - 4u)) {
            mbar_arrive_expect_tx(bar, (uint32_t)nst * kStagedUnitBytes);
            const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(eva_smem);
            // One array's units [s][t0, t0 + cnt) of every slice: contiguous in
            // global memory, placed slice-major in shared memory.
            auto copy_units = [&](const uint8_t *base, uint32_t ubytes, uint32_t region) {
                for (int sl = 0; sl < nsl; ++sl) {
                    const int cnt = min(ctiles, nst - sl * ctiles);
                    if (cnt <= 0) break;
                    const uint8_t *src = base + ((size_t)(s0 + sl) * p.T + t0) * ubytes;
                    const uint32_t dst = sbase + region + (uint32_t)(sl * ctiles) * ubytes;
                    const uint32_t bytes = (uint32_t)cnt * ubytes;
                    for (uint32_t off = 0; off < bytes; off += 32768u)
                        bulk_copy_g2s(dst + off, src + off, min(32768u, bytes - off), bar);
                }
            };
            copy_units(p.wi, kUnitBytes, UNITS_OFF);
            if constexpr (RESID) {
                copy_units(p.sgd, kDqSignUnitBytes, SG_OFF);
                copy_units(reinterpret_cast<const uint8_t *>(p.al), kAlphaUnitHalves * 2, AL_OFF);
            }
        } else if (!p.skip_stage_copy) {
            mbar_arrive(bar);
        }
    }
    if (tid < nsl) {
        // L2 prefetch of the slice's units that are not staged.
        const int first = max(0, min(ctiles, nst - tid * ctiles));
        const size_t u = (size_t)(s0 + tid) * p.T + t0 + first;
        const uint32_t nt = (uint32_t)(ctiles - first);
        if (nt > 0 && !EVA_BAD_G(BUF_WI, p.wi + u * kUnitBytes, nt * kUnitBytes))
            prefetch_l2_bulk(p.wi + u * kUnitBytes, nt * kUnitBytes);
        if constexpr (RESID) {
            if (nt > 0 && !EVA_BAD_G(BUF_SG, p.sgd + u * kDqSignUnitBytes, nt * kDqSignUnitBytes))
                prefetch_l2_bulk(p.sgd + u * kDqSignUnitBytes, nt * kDqSignUnitBytes);
            if (nt > 0 && !EVA_BAD_G(BUF_AL, p.al + u * kAlphaUnitHalves, nt * kAlphaUnitHalves * 2))
                prefetch_l2_bulk(p.al + u * kAlphaUnitHalves, nt * kAlphaUnitHalves * 2);
        }
    }
    bool units_ready = nst == 0;
    build_codebook_table(p, cb_first, tid);
    int built_cb = cb_first;

    if (!p.independent) pdl_wait();
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    EVA_STAMP(1);

    const uint32_t lofs = 8u * (uint32_t)(lane & 15);   // this lane's copy in the table
    for (int p0 = 0; p0 < p.B; p0 += TT) {
        // x of this pass's tokens for all the CTA's slices, fp16, zeros past B / K.
        // The residual instances rotate on chip (Sylvester blocks, p.rot_b):
        // one warp per (slice, token).
        const bool rot_x = RESID && p.rot_b != 0;
        if (rot_x) {
            for (int it = warp; it < nsl * TT; it += kWarps) {
                const int sl = it / TT, n = it - sl * TT;
                float v[8];
                dq_rotated_x8(p, p0 + n, (s0 + sl) * kSliceK, lane, v);
                const uint32_t off = XS_OFF + (uint32_t)(sl * TT + n) * kXTokStride + 16u * (uint32_t)lane;
                if (!EVA_BAD_S(off) && !EVA_BAD_S(off + 12u))
                    *reinterpret_cast<uint4 *>(eva_smem + off) =
                        make_uint4(pack_half2(v[0], v[1]), pack_half2(v[2], v[3]), pack_half2(v[4], v[5]),
                                   pack_half2(v[6], v[7]));
            }
        }
        for (int i = tid; i < (rot_x ? 0 : nsl * TT * 32); i += kThreads) {
            const int chunk = i & 31, n = (i >> 5) % TT, sl = i / (32 * TT);
            const int tok = p0 + n, k0 = (s0 + sl) * kSliceK + 8 * chunk;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (p.x_f32 && tok < p.B && k0 + 8 <= p.K) {
                const float4 *xp = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p.x) +
                                                                    (size_t)tok * p.K + k0);
                if (!EVA_BAD_G(BUF_X, xp, 32)) {
                    const float4 a = __ldcg(xp), b = __ldcg(xp + 1);
                    v = make_uint4(pack_half2(a.x, a.y), pack_half2(a.z, a.w), pack_half2(b.x, b.y),
                                   pack_half2(b.z, b.w));
                }
            } else if (p.x_f32 && tok < p.B && k0 < p.K) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float *xp = reinterpret_cast<const float *>(p.x) + (size_t)tok * p.K + k0 + e;
                    f[e] = (k0 + e < p.K && !EVA_BAD_G(BUF_X, xp, 4)) ? __ldcg(xp) : 0.f;
                }
                v = make_uint4(pack_half2(f[0], f[1]), pack_half2(f[2], f[3]), pack_half2(f[4], f[5]),
                               pack_half2(f[6], f[7]));
            } else if (tok < p.B && k0 + 8 <= p.K && ((((size_t)tok * p.K + k0) & 7) == 0)) {
                const uint4 *xp = reinterpret_cast<const uint4 *>(reinterpret_cast<const __half *>(p.x) +
                                                                  (size_t)tok * p.K + k0);
                if (!EVA_BAD_G(BUF_X, xp, 16)) v = __ldcg(xp);
            } else if (tok < p.B && k0 < p.K) {
                unsigned short h[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const unsigned short *xp = reinterpret_cast<const unsigned short *>(p.x) + (size_t)tok * p.K + k0 + e;
                    h[e] = (k0 + e < p.K && !EVA_BAD_G(BUF_X, xp, 2)) ? __ldcg(xp) : (unsigned short)0;
                }
                v = make_uint4(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16),
                               h[4] | ((uint32_t)h[5] << 16), h[6] | ((uint32_t)h[7] << 16));
            }
            const uint32_t off = XS_OFF + (uint32_t)(sl * TT + n) * kXTokStride + 16u * (uint32_t)chunk;
            if (!EVA_BAD_S(off) && !EVA_BAD_S(off + 12u)) *reinterpret_cast<uint4 *>(eva_smem + off) = v;
        }
        __syncthreads();
        EVA_STAMP(2);

        // This warp's tiles of codebook cb: warp + kWarps i for i in [i0, i1).
        auto cb_tiles = [&](int cb, int &i0, int &i1) {
            i0 = 0;
            i1 = ntw;
            if (GROUPED) {
                const int lo = max(cb * p.tiles_per_cb, t0), hi = (cb + 1) * p.tiles_per_cb;
                i0 = max(0, (lo - t0 - warp + kWarps - 1) / kWarps);
                i1 = min(ntw, max(0, (hi - t0 - warp + kWarps - 1) / kWarps));
            }
        };
        // Units [0, nst) of the CTA (slice-major) come from shared memory; the
        // others stream from global memory one unit ahead (nb0, nb1).
        uint4 nb0 = make_uint4(0u, 0u, 0u, 0u), nb1 = nb0;
        uint4 nsv = nb0;                  // residual: the unit's sign words for this lane
        uint2 nav = make_uint2(0u, 0u);   // and the alphas of rows g, g + 8 (groups 0, 1)
        bool have_next = false;   // nb0, nb1 already hold the next (codebook, slice)'s first unit
        auto fetch = [&](int s, int tl) {
            const int u = (s - s0) * ctiles + tl;
            if (u < nst) {
                const uint32_t wo = UNITS_OFF + (uint32_t)u * kUnitBytes + 16u * (uint32_t)lane;
                if (!EVA_BAD_S(wo) && !EVA_BAD_S(wo + 524u)) {
                    nb0 = lds128(wo);
                    nb1 = lds128(wo + 512u);
                }
                if constexpr (RESID) {
                    const uint32_t so = SG_OFF + (uint32_t)u * kDqSignUnitBytes + 16u * (uint32_t)lane;
                    const uint32_t ao = AL_OFF + (uint32_t)u * (kAlphaUnitHalves * 2) + 8u * (uint32_t)g;
                    if (!EVA_BAD_S(so) && !EVA_BAD_S(so + 12u)) nsv = lds128(so);
                    if (!EVA_BAD_S(ao) && !EVA_BAD_S(ao + 4u)) nav = lds64(ao);
                }
            } else {
                const size_t un = (size_t)s * p.T + t0 + tl;
                const uint8_t *up = p.wi + un * kUnitBytes + 16 * lane;
                if (!EVA_BAD_G(BUF_WI, up, 16) && !EVA_BAD_G(BUF_WI, up + 512, 16)) ldg_unit(up, nb0, nb1);
                if constexpr (RESID) {
                    const uint8_t *sp = p.sgd + un * kDqSignUnitBytes + 16 * lane;
                    const __half *ap = p.al + un * kAlphaUnitHalves + 4 * g;
                    if (!EVA_BAD_G(BUF_SG, sp, 16)) nsv = ldg_stream(sp);
                    if (!EVA_BAD_G(BUF_AL, ap, 8)) nav = __ldg(reinterpret_cast<const uint2 *>(ap));
                }
            }
        };
        for (int cb = cb_first; cb <= cb_last; ++cb) {
            int i0, i1;
            cb_tiles(cb, i0, i1);
            if (GROUPED) {
                if (cb != built_cb) {
                    __syncthreads();               // every warp is done with the previous table
                    build_codebook_table(p, cb, tid);
                    __syncthreads();
                    built_cb = cb;
                }
            }
            if constexpr (GROUPED) {
                // Per-group codebooks: a warp has few tiles of a codebook (one
                // when the codebook covers 8 tiles), so it takes each of them
                // through all of the CTA's slices (the slice loop unrolled by
                // two at 8 tokens) and sums them in registers.
                if (!units_ready) {
                    // Bounded: a give-up is recorded; the CTA still finishes.
                    units_ready = true;
                    if (!mbar_wait_bounded(bar, 0, p.wait_rounds) && tid == 0 && p.status) atomicOr(p.status, 1);
                }
                auto load_unit = [&](int s, int tl, uint4 &a, uint4 &b) {
                    const int u = (s - s0) * ctiles + tl;
                    a = b = make_uint4(0u, 0u, 0u, 0u);
                    if (u < nst) {
                        const uint32_t wo = UNITS_OFF + (uint32_t)u * kUnitBytes + 16u * (uint32_t)lane;
                        if (!EVA_BAD_S(wo) && !EVA_BAD_S(wo + 524u)) {
                            a = lds128(wo);
                            b = lds128(wo + 512u);
                        }
                    } else {
                        const uint8_t *up = p.wi + ((size_t)s * p.T + t0 + tl) * kUnitBytes + 16 * lane;
                        if (!EVA_BAD_G(BUF_WI, up, 16) && !EVA_BAD_G(BUF_WI, up + 512, 16)) ldg_unit(up, a, b);
                    }
                };
                constexpr int kSliceUnroll = NTG == 1 ? 2 : 1;
#pragma unroll 1
                for (int i = i0; i < i1; ++i) {
                    const int tl = warp + kWarps * i;
                    float tacc[NTG][4];
#pragma unroll
                    for (int t = 0; t < NTG; ++t)
#pragma unroll
                        for (int e = 0; e < 4; ++e) tacc[t][e] = 0.f;
#pragma unroll kSliceUnroll
                    for (int s = s0; s < s1; ++s) {
                        uint2 xs[NTG][16];
#pragma unroll
                        for (int t = 0; t < NTG; ++t)
#pragma unroll
                            for (int beta = 0; beta < 16; ++beta) {
                                const uint32_t off = XS_OFF + (uint32_t)((s - s0) * TT + 8 * t + g) * kXTokStride +
                                                     8u * (uint32_t)dq_subvec(beta, q);
                                xs[t][beta] = EVA_BAD_S(off) ? make_uint2(0u, 0u) : lds64(off);
                            }
                        uint4 u0, u1;
                        load_unit(s, tl, u0, u1);
                        const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                        uint32_t rot[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) rot[k] = wv[k];
#pragma unroll
                        for (int bit = 1; bit < 8; bit <<= 1) {
                            uint32_t nr[8];
#pragma unroll
                            for (int k = 0; k < 8; ++k) nr[k] = (g & bit) ? rot[(k - bit) & 7] : rot[k];
#pragma unroll
                            for (int k = 0; k < 8; ++k) rot[k] = nr[k];
                        }
                        float acc[NTG][2][4];
#pragma unroll
                        for (int t = 0; t < NTG; ++t)
#pragma unroll
                            for (int h = 0; h < 2; ++h)
#pragma unroll
                                for (int e = 0; e < 4; ++e) acc[t][h][e] = 0.f;
#pragma unroll
                        for (int beta = 0; beta < 16; ++beta) {
                            const uint32_t w = rot[beta & 7];
                            const uint32_t cg = beta < 8 ? (w & 0xFFu) : ((w >> 16) & 0xFFu);
                            const uint32_t ch = beta < 8 ? ((w >> 8) & 0xFFu) : (w >> 24);
                            const uint32_t og = TAB_OFF + (cg << 7) + lofs, oh = TAB_OFF + (ch << 7) + lofs;
                            const uint2 ag = EVA_BAD_S(og) ? make_uint2(0u, 0u) : lds64(og);
                            const uint2 ah = EVA_BAD_S(oh) ? make_uint2(0u, 0u) : lds64(oh);
#pragma unroll
                            for (int t = 0; t < NTG; ++t)
                                mma_f16_k16(acc[t][beta & 1], ag.x, ah.x, ag.y, ah.y, xs[t][beta].x, xs[t][beta].y);
                        }
#pragma unroll
                        for (int t = 0; t < NTG; ++t)
#pragma unroll
                            for (int e = 0; e < 4; ++e) tacc[t][e] += acc[t][0][e] + acc[t][1][e];
                    }
                    // D: (row g, tokens 2q, 2q+1), (row g+8, tokens 2q, 2q+1) of each token group.
                    if (direct) {
                        const uint32_t off = (uint32_t)((tl / p.Gs) * p.Gs + ts) * BLK_S + 4u * (uint32_t)(g * RS + 2 * q);
                        const uint32_t ra = dsmem_map(stage_addr + off, (uint32_t)(tl % p.Gs));
#pragma unroll
                        for (int t = 0; t < NTG; ++t)
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t o = 4u * (uint32_t)(8 * h * RS + 8 * t);
                                if (!EVA_BAD_S(STAGE_OFF + off + o) && !EVA_BAD_S(STAGE_OFF + off + o + 4u))
                                    st_dsmem_v2(ra + o, tacc[t][2 * h], tacc[t][2 * h + 1]);
                            }
                    } else {
#pragma unroll
                        for (int t = 0; t < NTG; ++t)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int row = g + 8 * (e >> 1), tok = 8 * t + 2 * q + (e & 1);
                                const int ai = (tl * kTileRows + row) * TT + tok;
                                if (!EVA_BAD_S(ACC_OFF + 4u * (uint32_t)ai)) acc_s[ai] = tacc[t][e];
                            }
                    }
                }
            } else {
            for (int s = s0; s < s1; ++s) {
                // B fragments of this slice: token 8t + g, sub-vector dq_subvec(beta, q).
                uint2 xb[NTG][16];
#pragma unroll
                for (int t = 0; t < NTG; ++t)
#pragma unroll
                    for (int beta = 0; beta < 16; ++beta) {
                        const uint32_t off = XS_OFF + (uint32_t)((s - s0) * TT + 8 * t + g) * kXTokStride +
                                             8u * (uint32_t)dq_subvec(beta, q);
                        xb[t][beta] = EVA_BAD_S(off) ? make_uint2(0u, 0u) : lds64(off);
                    }
                if (!units_ready) {
                    // Bounded: a give-up is recorded; the CTA still finishes.
                    units_ready = true;
                    if (!mbar_wait_bounded(bar, 0, p.wait_rounds) && tid == 0 && p.status) atomicOr(p.status, 1);
                }
                if (i0 < i1 && !have_next) fetch(s, warp + kWarps * i0);
                have_next = false;
#pragma unroll 1
                for (int i = i0; i < i1; ++i) {
                    const int tl = warp + kWarps * i;
                    const uint32_t wv[8] = {nb0.x, nb0.y, nb0.z, nb0.w, nb1.x, nb1.y, nb1.z, nb1.w};
                    const uint4 sv = nsv;
                    const uint2 av = nav;
                    // One unit ahead, across slices and codebooks too: with
                    // per-group codebooks a warp often has one tile per
                    // (codebook, slice), and its next unit is then in the next one.
                    if (i + 1 < i1) {
                        fetch(s, tl + kWarps);
                    } else if (DIRECT && !GROUPED) {
                        // one slice, one codebook: nothing further ahead
                    } else if (s + 1 < s1) {
                        fetch(s + 1, warp + kWarps * i0);
                        have_next = true;
                    } else if (GROUPED && cb < cb_last) {
                        int n0, n1;
                        cb_tiles(cb + 1, n0, n1);
                        if (n0 < n1) {
                            fetch(s0, warp + kWarps * n0);
                            have_next = true;
                        }
                    }
                    // rot[beta] = wv[(beta - g) mod 8]: the word holding sub-vectors 4 beta + q (+32).
                    uint32_t rot[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) rot[k] = wv[k];
#pragma unroll
                    for (int bit = 1; bit < 8; bit <<= 1) {
                        uint32_t nr[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) nr[k] = (g & bit) ? rot[(k - bit) & 7] : rot[k];
#pragma unroll
                        for (int k = 0; k < 8; ++k) rot[k] = nr[k];
                    }
                    // Two MMA accumulation chains per token group, one where the
                    // registers of two CTAs per SM would not hold two (16 tokens,
                    // sums pushed from registers).
                    constexpr int kChains = (NTG == 2 && DIRECT) ? 1 : 2;
                    float acc[NTG][2][4];
#pragma unroll
                    for (int t = 0; t < NTG; ++t)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int e = 0; e < 4; ++e) acc[t][h][e] = 0.f;
#pragma unroll
                    for (int beta = 0; beta < 16; ++beta) {
                        const uint32_t w = rot[beta & 7];
                        const uint32_t cg = beta < 8 ? (w & 0xFFu) : ((w >> 16) & 0xFFu);
                        const uint32_t ch = beta < 8 ? ((w >> 8) & 0xFFu) : (w >> 24);
                        const uint32_t og = TAB_OFF + (cg << 7) + lofs, oh = TAB_OFF + (ch << 7) + lofs;
                        uint2 ag = EVA_BAD_S(og) ? make_uint2(0u, 0u) : lds64(og);
                        uint2 ah = EVA_BAD_S(oh) ? make_uint2(0u, 0u) : lds64(oh);
                        if constexpr (RESID) {
                            // Sign nibble beta % 8 of word beta / 8 (row g) or 2 + beta / 8
                            // (row g + 8); alpha of the slice's group beta / 8.
                            const int sh = 4 * (beta & 7);
                            const uint32_t alw[2] = {av.x, av.y};
                            auto alpha_of = [&](int h) {
                                const uint32_t w2 = alw[h] >> (16 * (beta >> 3));
                                return __ushort_as_half((unsigned short)(w2 & 0xFFFFu));
                            };
                            auto add_resid = [&](uint2 &w, uint32_t nib, __half a) {
                                const __half na = __hneg(a);
                                const __half2 lo = __halves2half2((nib & 1u) ? a : na, (nib & 2u) ? a : na);
                                const __half2 hi = __halves2half2((nib & 4u) ? a : na, (nib & 8u) ? a : na);
                                __half2 x0 = *reinterpret_cast<const __half2 *>(&w.x), x1 = *reinterpret_cast<const __half2 *>(&w.y);
                                x0 = __hadd2(x0, lo);
                                x1 = __hadd2(x1, hi);
                                w.x = *reinterpret_cast<const uint32_t *>(&x0);
                                w.y = *reinterpret_cast<const uint32_t *>(&x1);
                            };
                            add_resid(ag, ((beta < 8 ? sv.x : sv.y) >> sh) & 0xFu, alpha_of(0));
                            add_resid(ah, ((beta < 8 ? sv.z : sv.w) >> sh) & 0xFu, alpha_of(1));
                        }
#pragma unroll
                        for (int t = 0; t < NTG; ++t)
                            mma_f16_k16(acc[t][kChains == 1 ? 0 : (beta & 1)], ag.x, ah.x, ag.y, ah.y, xb[t][beta].x, xb[t][beta].y);
                    }
                    // D: (row g, tokens 2q, 2q+1), (row g+8, tokens 2q, 2q+1) of each token group.
                    if (direct) {
                        // Into block ts of slot tl / Gs of the owner's (rank tl % Gs) stage.
                        const uint32_t off = (uint32_t)((tl / p.Gs) * p.Gs + ts) * BLK_S + 4u * (uint32_t)(g * RS + 2 * q);
                        const uint32_t ra = dsmem_map(stage_addr + off, (uint32_t)(tl % p.Gs));
#pragma unroll
                        for (int t = 0; t < NTG; ++t)
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t o = 4u * (uint32_t)(8 * h * RS + 8 * t);
                                if (!EVA_BAD_S(STAGE_OFF + off + o) && !EVA_BAD_S(STAGE_OFF + off + o + 4u))
                                    st_dsmem_v2(ra + o, acc[t][0][2 * h] + acc[t][1][2 * h],
                                                acc[t][0][2 * h + 1] + acc[t][1][2 * h + 1]);
                            }
                    } else {
#pragma unroll
                        for (int t = 0; t < NTG; ++t)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int row = g + 8 * (e >> 1), tok = 8 * t + 2 * q + (e & 1);
                                const int ai = (tl * kTileRows + row) * TT + tok;
                                const float v = acc[t][0][e] + acc[t][1][e];
                                if (!EVA_BAD_S(ACC_OFF + 4u * (uint32_t)ai))
                                    acc_s[ai] = (s == s0) ? v : acc_s[ai] + v;
                            }
                    }
                }
            }
            }
        }

        // Split-K sums of this pass: push each tile's block to the owning
        // cluster CTA (rank tl % Gs) with 16-byte remote stores (the direct
        // kernel pushed them from the tile loop), cluster barrier, owners add
        // the Gs blocks in rank order and store y.
        EVA_STAMP(4);
        __syncthreads();
        static_assert(DIRECT || BLK_S == BLK, "running-sum blocks are copied as they are");
        constexpr int CH = (int)(BLK / 16u);               // 16-byte chunks per tile block
        for (int i = tid; !direct && i < ctiles * CH; i += kThreads) {
            const int tl = i / CH, chunk = i % CH;
            const uint32_t src = ACC_OFF + (uint32_t)tl * BLK + 16u * (uint32_t)chunk;
            const uint32_t dst = (uint32_t)((tl / p.Gs) * p.Gs + ts) * BLK_S + 16u * (uint32_t)chunk;
            if (!EVA_BAD_S(src) && !EVA_BAD_S(src + 12u) && !EVA_BAD_S(STAGE_OFF + dst) && !EVA_BAD_S(STAGE_OFF + dst + 12u)) {
                const float4 v = *reinterpret_cast<const float4 *>(eva_smem + src);
                st_dsmem_v4(stage_addr + dst, (uint32_t)(tl % p.Gs), v);
            }
        }
        cluster_sync_all();
        EVA_STAMP(5);
        {
            const int my_tiles = (ctiles - ts + p.Gs - 1) / p.Gs;
            const int nb = min(TT, p.B - p0);               // tokens of this pass
            for (int idx = tid; idx < my_tiles * kTileRows * nb; idx += kThreads) {
                const int row = idx % kTileRows, tok = (idx / kTileRows) % nb, slot = idx / (kTileRows * nb);
                const int tl = ts + p.Gs * slot;
                const int o = kTileRows * (t0 + tl) + row, b = p0 + tok;
                if (o >= p.N) continue;
                float v[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const uint32_t si = (uint32_t)((((slot * p.Gs + k) * kTileRows + row) * RS) + tok);
                    v[k] = (k < p.Gs && !EVA_BAD_S(STAGE_OFF + 4u * si)) ? stage[si] : 0.f;
                }
                float sum = 0.f;
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (k < p.Gs) sum += v[k];
                const size_t yi = (size_t)b * p.N + o;
                if (p.out_f32) {
                    float *yp = reinterpret_cast<float *>(p.y) + yi;
                    if (!EVA_BAD_G(BUF_Y, yp, 4)) *yp = sum;
                } else {
                    __half *yp = reinterpret_cast<__half *>(p.y) + yi;
                    if (!EVA_BAD_G(BUF_Y, yp, 2)) *yp = __float2half_rn(sum);
                }
            }
        }
        // The next pass rewrites the x stage, the sums and the owners' stages.
        if (p0 + TT < p.B) cluster_sync_all();
    }
    // No bulk copy may still be writing this CTA's shared memory at exit.
    if (!units_ready && !mbar_wait_bounded(bar, 0, p.wait_rounds) && tid == 0 && p.status) atomicOr(p.status, 2);
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

template <bool GROUPED, int NTG, bool DIRECT, bool RESID = false>
__global__ void __launch_bounds__(kThreads, kDequantMinBlocks<GROUPED, NTG, DIRECT, RESID>)
    eva_dequant_kernel(const LookupParams p) {
    dequant_body<GROUPED, NTG, DIRECT, RESID>(p, blockIdx.x);
}

// Several layers of one shape (one shared codebook each) in one launch, as
// eva_lookup_group_kernel: layer blockIdx.x / ctas_per_layer.
template <int NTG, bool DIRECT>
__global__ void __launch_bounds__(kThreads, kDequantMinBlocks<false, NTG, DIRECT>)
    eva_dequant_group_kernel(const LookupGroup g) {
    const int li = blockIdx.x / g.ctas_per_layer;
    if (li >= g.count) return;
    dequant_body<false, NTG, DIRECT>(g.p[li], blockIdx.x - li * g.ctas_per_layer);
}

}  // namespace eva
