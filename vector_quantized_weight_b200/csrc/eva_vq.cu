// eva_vq.cu -- C ABI of the VQ decode linear (see include/eva_vq.h).
//
// Host side only: argument validation, device memory owned by a handle, the
// create-time repack, and the launch sequence of run():
//   [Hadamard rotation of x]  ->  fused OC build + lookup + accumulate
// Every launch goes to the caller's stream with programmatic dependent launch
// so a kernel's weight prefetch overlaps the tail of the one before it.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "../../include/eva_vq.h"
#include "eva_vq_kernels.cuh"
#include "eva_vq_plan.h"
#include "eva_vq_quant.cuh"
#include "eva_vq_dequant.cuh"
#include "eva_vq_tcgen.cuh"

using namespace eva;

struct eva_vq_linear {
    eva_vq_desc desc;
    int device = 0, sm_count = 0;
    int ncent = kCent, unit_bytes = kUnitBytes;   // 16 and 512 for 4-bit indices
    int smem_per_sm = 0, smem_reserved = 0, smem_optin = 0;   // shared memory, bytes
    int regs_per_sm = 0;
    int J = 0, S = 0, T = 0, Npad = 0, G = 1, tiles_per_cb = 0;
    // Lookup grid per variant (index: token pair or not): Gs slice groups
    // (one cluster) x Gt row groups, and its dynamic shared memory.
    // `staged` index units per CTA are copied into shared memory up front
    // (`smem`); calls flagged independent skip that copy (`smem_nostage`).
    struct Plan { int Gs = 1, Gt = 1, staged = 0; size_t smem = 0, smem_nostage = 0; };
    // Lookup-path grids for one token and for token pairs: plan[] for calls
    // that wait for their predecessor (one layer's latency), iplan[] for
    // calls flagged independent (CTA-slot time per layer).
    Plan plan[2], iplan[2];
    // Dequantize-to-tensor-core path (no residual, no rotation): plans for 8
    // and 16 tokens per pass.
    bool dq_ok = false;
    Plan dq[2];
    // Fifth-generation tensor-core path (tcgen05): CTAs per 128-row block for
    // 16, 32, 48 and 64 padded tokens, the row-block index / sign layouts, the
    // canonical alpha and, for a rotated layer, the rotated-input workspace.
    bool tc_ok = false;
    int tc_gs[4] = {0, 0, 0, 0};
    uint8_t *wib = nullptr, *sgb = nullptr;
    __half *al_rm = nullptr;
    float *xrot = nullptr;              // also the dequantize path's x~
    uint8_t *sgd = nullptr;             // dequantize path: sign units in its lane order
    uint8_t *wi = nullptr;              // repacked indices
    uint8_t *sg = nullptr;              // repacked signs
    __half *al = nullptr;               // repacked alpha
    __half *wc = nullptr;               // codebooks [G][256][4]
    int8_t *hsign = nullptr;            // Hadamard signs [K]
    int8_t *h28 = nullptr;              // order-28 Paley matrix (Paley rotation blocks)
    int *status = nullptr;              // device error word
    unsigned long long *timeline = nullptr;  // timeline build: [grid][8] stamps
    void *x_stage = nullptr, *y_stage = nullptr;
    // Host-buffer calls: one captured graph (H2D copy, run, D2H copy) per
    // batch size, replayed with the copies' host addresses updated.
    struct HostGraph {
        cudaGraphExec_t exec = nullptr;
        cudaGraphNode_t h2d = nullptr, d2h = nullptr;
        const void *x = nullptr;
        void *y = nullptr;
        bool failed = false;   // capture or instantiation refused: copies one by one
    } host_graph[65];
    cudaStream_t capture_stream = nullptr;
    int64_t workspace_bytes = 0;
    int last_grid = 0, last_kernels = 0, last_path = 0;
    // Failure-detection test hook: > 0 makes the next staging call skip its
    // index copy and give up its wait after this many rounds.
    int inject_wait_rounds = 0;
};

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

eva_status_t cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return EVA_OK;
    if (e == cudaErrorMemoryAllocation) return EVA_ERR_OOM;
    return EVA_ERR_CUDA;
}

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// Rotation blocks: a power of two in [8, 4096] (Sylvester), or b = 28 m with
// m a power of two in [64, 1024] (Paley order 28 (x) Sylvester m; b is then a
// multiple of 256, so every K-slice lies inside one block); b divides K.
int paley_m(int b) { return (b % 28 == 0 && is_pow2(b / 28) && b / 28 >= 64 && b / 28 <= 1024) ? b / 28 : 0; }
bool valid_rotation_block(int b, int K) {
    if (b <= 0 || K % b) return false;
    return (is_pow2(b) && b >= 8 && b <= 4096) || paley_m(b) != 0;
}

// The order-28 Hadamard matrix of Paley's first construction over GF(27):
// GF(27) = GF(3)[t] / (t^3 + 2t + 2), element c0 + 3 c1 + 9 c2 = c0 + c1 t +
// c2 t^2; chi(a) = +1 for a nonzero square, -1 for a non-square, 0 for 0;
// Jacobsthal Q[i][j] = chi(e_i - e_j); H = I + [0, 1; -1, Q].
void paley28_table(int8_t *out) {
    auto mul = [](int a, int b) {
        int x[3], y[3], z[5] = {0, 0, 0, 0, 0};
        for (int i = 0; i < 3; ++i) { x[i] = a % 3; a /= 3; y[i] = b % 3; b /= 3; }
        for (int i = 0; i < 3; ++i)
            for (int j = 0; j < 3; ++j) z[i + j] = (z[i + j] + x[i] * y[j]) % 3;
        for (int d = 4; d >= 3; --d) {          // t^3 = t + 1 (mod 3)
            z[d - 3] = (z[d - 3] + z[d]) % 3;
            z[d - 2] = (z[d - 2] + z[d]) % 3;
            z[d] = 0;
        }
        return z[0] + 3 * z[1] + 9 * z[2];
    };
    bool square[27] = {};
    for (int a = 1; a < 27; ++a) square[mul(a, a)] = true;
    auto sub = [](int a, int b) {
        int r = 0, w = 1;
        for (int i = 0; i < 3; ++i, a /= 3, b /= 3, w *= 3) r += (((a % 3) - (b % 3) + 3) % 3) * w;
        return r;
    };
    for (int i = 0; i < 28; ++i)
        for (int j = 0; j < 28; ++j) {
            int v;
            if (i == 0) v = 1;
            else if (j == 0) v = -1;
            else if (i == j) v = 1;
            else v = square[sub(i - 1, j - 1)] ? 1 : -1;
            out[i * 28 + j] = (int8_t)v;
        }
}

// Layers the tcgen05 path takes: 8-bit indices, K a multiple of 64 (whole
// stages), codebooks shared or per whole 128-row blocks.
bool tc_layer_ok(const eva_vq_desc &d) {
    return d.index_bits == 8 && d.K % kTcStageK == 0 && (d.codebook_rows == 0 || d.codebook_rows % kTcRows == 0);
}

eva_status_t validate_desc(const eva_vq_desc *d) {
    if (!d) return EVA_ERR_INVALID_ARG;
    if (d->N < 1 || d->K < 1 || d->N > (1 << 24) || d->K > (1 << 22)) return EVA_ERR_INVALID_ARG;
    if (d->d != kD || (d->index_bits != 8 && d->index_bits != 4)) return EVA_ERR_UNSUPPORTED;
    if (d->index_bits == 4) {
        // 4-bit indices: the lookup path only, whole index bytes.
        if (d->path == EVA_PATH_DEQUANT_MMA) return EVA_ERR_UNSUPPORTED;
        if (d->K % 8) return EVA_ERR_INVALID_ARG;
    }
    if (d->K % kD) return EVA_ERR_INVALID_ARG;
    if (d->codebook_rows < 0) return EVA_ERR_INVALID_ARG;
    if (d->codebook_rows && (d->codebook_rows % kTileRows || d->N % d->codebook_rows))
        return EVA_ERR_INVALID_ARG;
    if (d->residual_group != 0 && d->residual_group != 128) return EVA_ERR_UNSUPPORTED;
    if (d->residual_group && d->K % d->residual_group) return EVA_ERR_INVALID_ARG;
    if (d->hadamard_block && !valid_rotation_block(d->hadamard_block, d->K)) return EVA_ERR_INVALID_ARG;
    if (d->max_batch < 1 || d->max_batch > 64) return EVA_ERR_INVALID_ARG;
    if (d->out_dtype != EVA_F16 && d->out_dtype != EVA_F32) return EVA_ERR_INVALID_ARG;
    if (d->path != EVA_PATH_AUTO && d->path != EVA_PATH_OC_LOOKUP && d->path != EVA_PATH_DEQUANT_MMA &&
        d->path != EVA_PATH_TCGEN05)
        return EVA_ERR_INVALID_ARG;
    // The dequantize path takes a residual or a rotation with one shared codebook.
    if (d->path == EVA_PATH_DEQUANT_MMA && (d->residual_group || d->hadamard_block) && d->codebook_rows)
        return EVA_ERR_UNSUPPORTED;
    if (d->path == EVA_PATH_TCGEN05 && !tc_layer_ok(*d)) return EVA_ERR_UNSUPPORTED;
    return EVA_OK;
}

// Dynamic shared memory of the lookup kernel: the OC image (with the residual
// table in its unused half for one token, or a second image for a token
// pair), the staged x~ slice of one or two tokens, the staging copy's
// mbarrier, the running sums of `tiles` row tiles, the cluster reduction
// stage and, 128-byte aligned, the fused rotation's scratch (rotation blocks
// b > 256: b floats per token) and the `staged` index units of the first slice.
size_t lookup_smem(bool pair_t, bool resid, int tiles, int gs, int rot_b, int s_total, int staged = 0,
                   size_t unit_bytes = kUnitBytes) {
    const size_t tile_bytes = (size_t)kTileRows * 2 * 4;
    const size_t stage_tiles = (size_t)((tiles + gs - 1) / gs) * gs;   // reduction stage
    // One token without residual table or rotation: x~, mbarrier and running
    // sums sit in the image rows' unused halves; only the stage follows.
    const bool gaps = !pair_t && !resid && !rot_b && !kNaiveOcBuild;
    const size_t base = gaps ? (size_t)kOcBytes + stage_tiles * tile_bytes
                             : (size_t)kOcBytes + ((pair_t && resid) ? (size_t)kOcBytes : 0) +
                                   (pair_t ? kXStageBytes : kXStageBytes / 2) + 128 + (size_t)tiles * tile_bytes +
                                   stage_tiles * tile_bytes;
    const int ntok = pair_t ? 2 : 1;
    const size_t xt = paley_m(rot_b) >= 256 ? (size_t)((s_total + gs - 1) / gs) * ntok * kSliceK * 4 : 0;
    const size_t rot = rot_b ? xt + rot_scratch_bytes(rot_b, paley_m(rot_b), ntok) : 0;
    return ((base + 127) & ~(size_t)127) + rot + (size_t)staged * unit_bytes;
}

// Index units of the first slice a CTA copies into shared memory: as many of
// its `tiles` as fit in what is left of the per-SM budget.  The budget keeps
// two CTAs per SM (this layer's and the next layer's early-launched one)
// wherever the registers and the rest of the footprint allow it, else one.
int staged_tiles(const eva_vq_linear *h, const void *fn, bool pair_t, bool resid, int tiles, int gs) {
    const size_t base = lookup_smem(pair_t, resid, tiles, gs, h->desc.hadamard_block, h->S, 0);
    const size_t per_sm = (size_t)h->smem_per_sm, reserved = (size_t)h->smem_reserved;
    const size_t two = per_sm / 2 - reserved;
    const size_t one = std::min(per_sm - reserved, (size_t)h->smem_optin);
    cudaFuncAttributes fa;
    bool two_fit_regs = false;
    if (cudaFuncGetAttributes(&fa, fn) == cudaSuccess)
        two_fit_regs = 2 * fa.numRegs * kThreads <= h->regs_per_sm;
    else
        cudaGetLastError();
    const size_t budget = (two_fit_regs && base <= two) ? two : one;
    if (base >= budget) return 0;
    return (int)std::min<size_t>((size_t)tiles, (budget - base) / h->unit_bytes);
}

using LookupFn = void (*)(LookupParams);
template <bool ROT, bool NIB>
LookupFn lookup_fn_r(bool pair_t, bool resid, bool grouped) {
    if (grouped) {
        if (!pair_t)
            return resid ? eva_lookup_kernel<false, true, true, ROT, NIB> : eva_lookup_kernel<false, false, true, ROT, NIB>;
        return resid ? eva_lookup_kernel<true, true, true, ROT, NIB> : eva_lookup_kernel<true, false, true, ROT, NIB>;
    }
    if (!pair_t)
        return resid ? eva_lookup_kernel<false, true, false, ROT, NIB> : eva_lookup_kernel<false, false, false, ROT, NIB>;
    return resid ? eva_lookup_kernel<true, true, false, ROT, NIB> : eva_lookup_kernel<true, false, false, ROT, NIB>;
}
// rot: the instance that computes the Hadamard rotation while staging x;
// nib: 4-bit indices.
LookupFn lookup_fn(bool pair_t, bool resid, bool grouped, bool rot, bool nib = false) {
    if (nib) return rot ? lookup_fn_r<true, true>(pair_t, resid, grouped) : lookup_fn_r<false, true>(pair_t, resid, grouped);
    return rot ? lookup_fn_r<true, false>(pair_t, resid, grouped) : lookup_fn_r<false, false>(pair_t, resid, grouped);
}

// Three CTAs per SM (eva_lookup_kernel3): one token, no residual table, no
// rotation, and few enough tiles per CTA that the tighter register budget
// costs less than the third layer in flight gains (measured: 37 tiles of a
// 4096 x 4096 layer gain, 77 tiles of 11008 x 4096 lose).
constexpr int kThreePerSmMaxTiles = 48;
LookupFn lookup_fn3(bool grouped, bool nib) {
    if (nib) return grouped ? eva_lookup_kernel3<true, true> : eva_lookup_kernel3<false, true>;
    return grouped ? eva_lookup_kernel3<true, false> : eva_lookup_kernel3<false, false>;
}

// Largest number of clusters of `cs` CTAs of this kernel resident at once.
int max_active_clusters(LookupFn fn, size_t smem, int cs, int threads = kThreads) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs * 64);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeClusterDimension;
    a[0].val.clusterDim.x = cs;
    a[0].val.clusterDim.y = 1;
    a[0].val.clusterDim.z = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (const void *)fn, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

// Pick the CTA rectangle: Gs slice groups (one thread-block cluster, Gs <=
// 16) x Gt row groups, every cluster resident in one wave with at most one
// CTA of this layer per SM (the second slot stays free for the next layer's
// prologue), at most kMaxCtaTiles row tiles per CTA.  The cost model counts
// the latency-bound phases of a CTA: per slice the x~ staging and the image
// build, per unit of lookups a share of the warps' tile loop, and the
// cluster reduction.
eva_vq_linear::Plan latency_plan(const eva_vq_linear *h, int pair_t) {
    const int S = h->S, T = h->T, P = h->sm_count;
    const bool resid = h->desc.residual_group != 0;
    const LookupFn fn = lookup_fn(pair_t != 0, resid, h->tiles_per_cb != 0, h->desc.hadamard_block != 0,
                                  h->desc.index_bits == 4);
    double best = 1e300;
    eva_vq_linear::Plan pl;
    pl.Gs = 1;
    pl.Gt = std::min(T, P);
    for (int gs = 1; gs <= std::min(S, 16); ++gs) {
        const int gt_min = (T + kMaxCtaTiles - 1) / kMaxCtaTiles;
        // Capacity with one CTA per SM: the occupancy query counts CTA slots,
        // so ask with a footprint that leaves room for a single CTA per SM.
        const size_t smem_one = std::max(lookup_smem(pair_t, resid, (T + gt_min - 1) / gt_min, gs,
                                                     h->desc.hadamard_block, S),
                                         (size_t)120 * 1024);
        const int clusters = max_active_clusters(fn, smem_one, gs);
        // One CTA of this layer per SM: no more clusters than P / gs either.
        // With per-group codebooks the image builds dominate and two CTAs of
        // the layer per SM interleave them (measured, Llama-2-70B 8192^2 at
        // one token: 24.1 us on 16 x 7, 21.3 on 16 x 13), at the cost of the
        // next layer's early prologue.
        const int per_sm = h->tiles_per_cb ? 2 : 1;
        const int gt_max = std::min({T, per_sm * clusters, per_sm * (P / gs)});
        for (int gt = gt_min; gt <= gt_max; ++gt) {
            const int tiles = (T + gt - 1) / gt, slices = (S + gs - 1) / gs;
            int builds = 1;
            if (h->tiles_per_cb) builds = (tiles + h->tiles_per_cb - 1) / h->tiles_per_cb + 1;
            double cost = (double)slices * (1300.0 + 900.0 * builds + 250.0 * ((tiles + kWarps - 1) / kWarps));
            cost += (gs > 1) ? 600.0 + 40.0 * gs : 0.0;
            if (cost < best) {
                best = cost;
                pl.Gs = gs;
                pl.Gt = gt;
            }
        }
    }
    const int tiles = (T + pl.Gt - 1) / pl.Gt;
    pl.staged = staged_tiles(h, (const void *)fn, pair_t != 0, resid, tiles, pl.Gs);
    pl.smem = lookup_smem(pair_t, resid, tiles, pl.Gs, h->desc.hadamard_block, S, pl.staged, h->unit_bytes);
    pl.smem_nostage = lookup_smem(pair_t, resid, tiles, pl.Gs, h->desc.hadamard_block, S, 0);
    return pl;
}

void plan_grid(eva_vq_linear *h, int pair_t) {
    const int S = h->S, T = h->T;
    const bool resid = h->desc.residual_group != 0;
    const eva_vq_linear::Plan pl = latency_plan(h, pair_t);
    h->plan[pair_t] = pl;

    // Calls flagged independent: their own grid (eva_vq_plan.h), preferring
    // 128 row tiles per CTA, 64 with per-group codebooks (there more tiles per
    // CTA also mean more image builds per CTA), at most what the running-sum
    // layout holds (kMaxGapTiles in the row-gap layout, kMaxCtaTiles
    // otherwise), within a footprint of two CTAs per SM (or the latency
    // plan's own); if nothing qualifies it is the latency plan.
    eva_vq_linear::Plan ip = pl;
    ip.staged = 0;
    ip.smem = ip.smem_nostage = pl.smem_nostage;
    {
        const bool gaps = !pair_t && !resid && !h->desc.hadamard_block && !kNaiveOcBuild;
        const int hard = gaps ? kMaxGapTiles : kMaxCtaTiles;
        const int soft = h->tiles_per_cb ? kMaxCtaTiles / 2 : kMaxCtaTiles;
        const size_t two = (size_t)h->smem_per_sm / 2 - (size_t)h->smem_reserved;
        const size_t fit = std::min(std::max(pl.smem_nostage, two), (size_t)h->smem_optin);
        auto smem = [&](int tiles, int gs) {
            return lookup_smem(pair_t, resid, tiles, gs, h->desc.hadamard_block, S, 0, h->unit_bytes);
        };
        int gs = 0, gt = 0;
        size_t sm = 0;
        if (independent_grid(T, pl.Gs, pl.Gt, hard, soft, fit, smem, &gs, &gt, &sm)) {
            ip.Gs = gs;
            ip.Gt = gt;
            ip.smem = ip.smem_nostage = sm;
        }
    }
    h->iplan[pair_t] = ip;
}

// The grid of a lookup-path call.
const eva_vq_linear::Plan &call_plan(const eva_vq_linear *h, int B, int independent) {
    return independent ? h->iplan[B > 1 ? 1 : 0] : h->plan[B > 1 ? 1 : 0];
}

// Launch with programmatic dependent launch (and a cluster shape when
// cluster > 0) on the caller's stream.
template <typename K, typename... Args>
cudaError_t launch_pdl(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n = 1;
    if (cluster > 0) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}


using DequantFn = void (*)(LookupParams);
// `direct`: every CTA takes one K-slice (Gs = S), see eva_dequant_kernel;
// `resid`: the sign residual (one shared codebook only).
DequantFn dequant_fn(bool grouped, int ntg, bool direct, bool resid = false) {
    if (resid) {
        if (direct) return ntg == 2 ? eva_dequant_kernel<false, 2, true, true> : eva_dequant_kernel<false, 1, true, true>;
        return ntg == 2 ? eva_dequant_kernel<false, 2, false, true> : eva_dequant_kernel<false, 1, false, true>;
    }
    if (direct) {
        if (grouped) return ntg == 2 ? eva_dequant_kernel<true, 2, true> : eva_dequant_kernel<true, 1, true>;
        return ntg == 2 ? eva_dequant_kernel<false, 2, true> : eva_dequant_kernel<false, 1, true>;
    }
    if (grouped) return ntg == 2 ? eva_dequant_kernel<true, 2, false> : eva_dequant_kernel<true, 1, false>;
    return ntg == 2 ? eva_dequant_kernel<false, 2, false> : eva_dequant_kernel<false, 1, false>;
}

// Calls with at least this many tokens take the dequantize path (when the
// layer allows it and the descriptor leaves the choice to the library); layers
// with per-group codebooks from kDequantMinBatchGrouped on.  Measured on B200
// (us per layer, each call waiting for the one before it, lookup against
// dequantize path): 4096 x 4096 at 3 tokens 10.3 against 5.7, at 2 5.8 against
// 5.7; 11008 x 4096 at 3 15.9 against 14.6, at 2 8.8 against 14.4; 4096 x
// 11008 at 3 21.7 against 11.4; 8192 x 8192 with 128-row codebooks at 2 39.0
// against 22.7, at 3 75.6 against 22.7.
constexpr int kDequantMinBatch = 3;
constexpr int kDequantMinBatchGrouped = 2;
int dequant_min_batch(const eva_vq_desc &d) { return d.codebook_rows ? kDequantMinBatchGrouped : kDequantMinBatch; }

// Dynamic shared memory of the dequantize kernel: the replicated codebook,
// the x stage of up to nsl slices, the running sums, the reduction stage, the
// staging mbarrier and `staged` index units (with their sign and alpha units
// when the layer has the residual).
size_t dequant_smem(int nsl, int tiles, int gs, int ntg, int staged = 0, bool resid = false) {
    const size_t blk = (size_t)kTileRows * 8 * ntg * 4;
    const size_t xs = ((size_t)nsl * 8 * ntg * kXTokStride + 127) & ~(size_t)127;
    const size_t nslot = (size_t)(tiles + gs - 1) / gs;
    // With one slice per CTA the tiles' sums go straight to the owners'
    // stages, whose rows are then padded by two floats.
    const size_t acc = nsl == 1 ? 0 : (size_t)tiles * blk;
    const size_t blk_s = nsl == 1 ? (size_t)kTileRows * (8 * ntg + 2) * 4 : blk;
    const size_t base = (size_t)kTabBytes + xs + acc + nslot * gs * blk_s;
    return ((base + 127) & ~(size_t)127) + 128 + (size_t)staged * (kUnitBytes + (resid ? kDqResidUnitBytes : 0));
}

// Same search as plan_grid, for the dequantize kernel (one CTA per SM, every
// cluster in one wave when the shared memory allows it).
void plan_dequant(eva_vq_linear *h, int ntg) {
    const int S = h->S, T = h->T, P = h->sm_count;
    double best = 1e300;
    eva_vq_linear::Plan pl;
    pl.Gs = 0;
    for (int gs = 1; gs <= std::min(S, 16); ++gs) {
        const int nsl = (S + gs - 1) / gs;
        const DequantFn fn = dequant_fn(h->tiles_per_cb != 0, ntg, nsl == 1, h->desc.residual_group != 0);
        const int gt_min = (T + kMaxCtaTiles - 1) / kMaxCtaTiles;
        const int clusters = max_active_clusters((LookupFn)fn, (size_t)h->smem_optin, gs);
        const int gt_max = std::min({T, std::max(clusters, gt_min), std::max(P / gs, gt_min)});
        for (int gt = gt_min; gt <= gt_max; ++gt) {
            const int tiles = (T + gt - 1) / gt;
            if (dequant_smem(nsl, tiles, gs, ntg) > (size_t)h->smem_optin) continue;
            int builds = 1;
            if (h->tiles_per_cb) builds = (tiles + h->tiles_per_cb - 1) / h->tiles_per_cb + 1;
            double cost = (double)nsl * (700.0 + (250.0 + 150.0 * ntg) * ((tiles + kWarps - 1) / kWarps)) +
                          600.0 * builds + ((gs > 1) ? 600.0 + 40.0 * gs : 0.0);
            if (gt > clusters) cost *= 2.0;   // beyond one wave
            if (cost < best) {
                best = cost;
                pl.Gs = gs;
                pl.Gt = gt;
            }
        }
    }
    if (pl.Gs == 0) {   // nothing fits: the lookup path serves every batch
        h->dq[ntg - 1] = pl;
        return;
    }
    const int tiles = (T + pl.Gt - 1) / pl.Gt, nsl = (S + pl.Gs - 1) / pl.Gs;
    // Index units copied into shared memory in the prologue: as many of the
    // CTA's units as fit while the CTA still leaves half the SM to the next
    // layer's early-launched CTA (whose prologue then overlaps this one);
    // none when the rest of the footprint already takes more than half
    // (measured: staging past that point costs the overlap, 6.1 -> 11.4 us
    // for 4096^2 at 4 tokens).
    // With per-group codebooks the tile loop, not the prologue, sets the
    // layer's time: the CTA takes the whole SM instead -- every unit that fits
    // is staged, and at least half the SM's shared memory keeps a second CTA
    // of the same layer off the SM (two on one SM stretched the slowest CTA's
    // tile loop from 12.8 to 19.8 us for 8192^2 at one token).
    const bool resid = h->desc.residual_group != 0;
    const size_t base = dequant_smem(nsl, tiles, pl.Gs, ntg);
    const size_t half = (size_t)h->smem_per_sm / 2 - (size_t)h->smem_reserved;
    const size_t budget = h->tiles_per_cb ? (size_t)h->smem_optin : half;
    const size_t ubytes = kUnitBytes + (resid ? kDqResidUnitBytes : 0);
    pl.staged = base < budget ? (int)std::min<size_t>((size_t)nsl * tiles, (budget - base) / ubytes) : 0;
    pl.smem = dequant_smem(nsl, tiles, pl.Gs, ntg, pl.staged, resid);
    pl.smem_nostage = dequant_smem(nsl, tiles, pl.Gs, ntg);
    if (h->tiles_per_cb) pl.smem = std::max(pl.smem, half + 1024);
    h->dq[ntg - 1] = pl;
}

cudaError_t set_smem_attrs(int smem_optin) {
    cudaError_t e;
    for (int v = 0; v < 4; ++v) {
        const void *fn = v == 0 ? (const void *)eva_dequant_group_kernel<1, false>
                       : v == 1 ? (const void *)eva_dequant_group_kernel<2, false>
                       : v == 2 ? (const void *)eva_dequant_group_kernel<1, true>
                                : (const void *)eva_dequant_group_kernel<2, true>;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
        if (e != cudaSuccess) return e;
    }
    for (int v = 0; v < 12; ++v) {
        const DequantFn fn = v < 8 ? dequant_fn(v & 1, 1 + ((v >> 1) & 1), (v >> 2) & 1)
                                   : dequant_fn(false, 1 + (v & 1), (v >> 1) & 1, true);
        e = cudaFuncSetAttribute((const void *)fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute((const void *)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
        if (e != cudaSuccess) return e;
    }
    for (int v = 0; v < 32; ++v) {
        const LookupFn fn = lookup_fn(v & 1, (v >> 1) & 1, (v >> 2) & 1, (v >> 3) & 1, (v >> 4) & 1);
        e = cudaFuncSetAttribute((const void *)fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        // The device's per-block limit: it covers the one-CTA-per-SM footprint
        // the planner's occupancy query uses and any index staging; launches
        // request only what they need.
        e = cudaFuncSetAttribute((const void *)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
        if (e != cudaSuccess) return e;
    }
    for (int v = 0; v < 4; ++v) {
        const LookupFn fn = lookup_fn3(v & 1, (v >> 1) & 1);
        e = cudaFuncSetAttribute((const void *)fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute((const void *)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
        if (e != cudaSuccess) return e;
    }
    for (int v = 0; v < 4; ++v) {
        const void *fn = v == 0 ? (const void *)eva_lookup_group_kernel<false, false>
                       : v == 1 ? (const void *)eva_lookup_group_kernel<false, true>
                       : v == 2 ? (const void *)eva_lookup_group_kernel<true, false>
                                : (const void *)eva_lookup_group_kernel<true, true>;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
        if (e != cudaSuccess) return e;
    }
    for (int v = 0; v < 2; ++v) {
        const void *fn = v ? (const void *)eva_tc_kernel<true> : (const void *)eva_tc_kernel<false>;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
        if (e != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(eva_paley_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 28 * 1024 * 4);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(eva_hadamard_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 4096 * 4);
}

// Failure-detection test hook (eva_vq_debug_inject_wait_timeout): a launch
// that stages index units skips their copy and gives up its wait early, once.
void apply_injection(eva_vq_linear *h, LookupParams &p) {
    if (h->inject_wait_rounds > 0 && p.wi_staged > 0) {
        p.skip_stage_copy = 1;
        p.wait_rounds = h->inject_wait_rounds;
        h->inject_wait_rounds = 0;
    }
}

bool dequant_direct(const eva_vq_linear *h, int B) {
    const eva_vq_linear::Plan &pl = h->dq[B > 8 ? 1 : 0];
    return (h->S + pl.Gs - 1) / pl.Gs == 1;   // the same rule as dequant_smem's
}

// The dequantize kernel's residual instances rotate x on chip (the 3.125-bit
// format has both) where that is cheap: a Sylvester block of at most 1024
// inputs (one round of four sub-block loads per slice and token), one slice
// per CTA and at most kOnChipRotMaxTiles row tiles per CTA.  Measured on
// B200, 3.125-bit layers (block 512), one layer waiting for the previous
// one: 3584 x 3584 (32 tiles a CTA) 8.7 against 11.0 us at 4 tokens, 12.0
// against 19.4 at 16; 14336 x 3584 (128 tiles a CTA) 29.0 against 27.7 at 4,
// 35.7 against 33.5 at 16 -- with long tile loops the rotation kernel's
// launch costs less than the rotation on the CTAs' critical path.  Otherwise
// x~ comes from the standalone rotation kernel: with several slices per CTA
// of a 2048 block the warps redo the sub-block transforms one latency after
// the other (3584 x 14336 at 16 tokens: 64.0 on chip against 41.2 us); a
// Paley block's transform spans the whole block; a rotated layer without the
// residual keeps the other instances' registers as they are.
constexpr int kOnChipRotMaxTiles = 64;
bool dq_rotates_on_chip(const eva_vq_linear *h, int B) {
    const eva_vq_desc &d = h->desc;
    if (!d.hadamard_block || d.hadamard_block > 1024 || paley_m(d.hadamard_block) || !d.residual_group) return false;
    const eva_vq_linear::Plan &pl = h->dq[B > 8 ? 1 : 0];
    return dequant_direct(h, B) && (h->T + pl.Gt - 1) / pl.Gt <= kOnChipRotMaxTiles;
}

// The dequantize kernel's fields of a call's parameters (its plan for B);
// p.x is fp16 x, or x~ in fp32 (x_f32) from the rotation kernel.
void dequant_params(eva_vq_linear *h, LookupParams &p, int B) {
    const int ntg = B > 8 ? 2 : 1;
    const eva_vq_linear::Plan &pl = h->dq[ntg - 1];
    p.Gs = pl.Gs;
    p.Gt = pl.Gt;
    p.acc_tiles = (h->T + pl.Gt - 1) / pl.Gt;
    p.wi_staged = pl.staged;
    p.rot_b = 0;
    p.rot_m = 0;
    if (dq_rotates_on_chip(h, B) && !p.x_f32) {
        p.rot_b = h->desc.hadamard_block;
        p.hs = h->hsign;
        p.rot_scale = (float)(1.0 / std::sqrt((double)h->desc.hadamard_block));
    }
    p.sgd = h->sgd;
    p.al = h->al;
    apply_injection(h, p);
#ifdef EVA_DEVICE_CHECKS
    p.smem_bytes = (unsigned)pl.smem;
    if (h->desc.residual_group) {
        const unsigned long long units = (unsigned long long)h->S * h->T;
        p.chk_base[BUF_SG] = h->sgd;
        p.chk_bytes[BUF_SG] = units * kDqSignUnitBytes;
        p.chk_base[BUF_AL] = h->al;
        p.chk_bytes[BUF_AL] = units * kAlphaUnitHalves * 2;
    }
    p.chk_base[BUF_X] = p.x;
    p.chk_bytes[BUF_X] = (unsigned long long)B * h->desc.K * (p.x_f32 ? 4 : 2);
#endif
}

cudaError_t launch_dequant(eva_vq_linear *h, LookupParams p, int B, cudaStream_t s, size_t *smem_out,
                           int *grid_out) {
    const int ntg = B > 8 ? 2 : 1;
    const eva_vq_linear::Plan &pl = h->dq[ntg - 1];
    dequant_params(h, p, B);
    *smem_out = pl.smem;
    *grid_out = pl.Gs * pl.Gt;
    return launch_pdl(dequant_fn(h->tiles_per_cb != 0, ntg, dequant_direct(h, B), h->desc.residual_group != 0),
                      dim3(pl.Gs * pl.Gt), dim3(kThreads), pl.smem, s, pl.Gs, p);
}

bool use_three_per_sm(const eva_vq_linear *h, int B, int independent) {
    const eva_vq_desc &d = h->desc;
    if (B > 1 || d.residual_group || d.hadamard_block || kNaiveOcBuild) return false;
    const eva_vq_linear::Plan &pl = call_plan(h, B, independent);
    return (h->T + pl.Gt - 1) / pl.Gt <= kThreePerSmMaxTiles;
}

// The tcgen05 path: forced, or AUTO from kDequantMinBatch tokens on.
// AUTO (measured per batch on B200, one layer waiting for the previous one):
//  - the warp-level dequantize path from kDequantMinBatch tokens on, except
//    with one shared codebook past two 16-token passes (kTcMinBatch), where
//    tcgen05 wins (4096 x 4096: 16.3 against 17.0 us at 32 tokens, 19.1
//    against 24.2 at 48, 21.3 against 32.0 at 64; 11008 x 4096: 35.0 against
//    49.0 at 32, 62.0 against 65.1 at 64); with per-group codebooks the
//    warp-level path stays ahead (8192 x 8192: 62.3 against 85.2 us at 32
//    tokens).  The same split holds for 3.125-bit layers (Hadamard blocks,
//    sign residual): 3584 x 3584 at 4 tokens 11.1 us against 16.0 (lookup)
//    and 20.5 (tcgen05), at 16 19.4 against 24.1 (tcgen05), at 48 47.7
//    against 30.6; 14336 x 3584 at 16 34.3 against 60.4, at 64 116.9 against
//    110.6;
//  - layers the warp-level path cannot take (residual or rotation with
//    per-group codebooks): the lookup path below kTcResidMinBatch tokens,
//    tcgen05 from there.
// A tcgen05.mma of M = 128 rows takes about as long for N = 16 tokens as for
// N = 64 (54-100 cycles per instruction in two single-thread probes), so the
// tensor-core path pays off as the batch grows, while the warp-level MMA of 8
// tokens scales with the batch.
constexpr int kTcMinBatch = 33;
constexpr int kTcResidMinBatch = 8;

// Whether AUTO can ever pick the tcgen05 path for this handle (the rule of
// use_tc at the handle's largest batch): only then does create plan it and
// keep its row-block copies of the indices and signs.
bool auto_may_use_tc(const eva_vq_linear *h) {
    if (h->dq_ok) return h->desc.codebook_rows == 0 && h->desc.max_batch >= kTcMinBatch;
    return h->desc.max_batch >= kTcResidMinBatch;
}

bool use_tc(const eva_vq_linear *h, int B) {
    if (!h->tc_ok) return false;
    if (h->desc.path == EVA_PATH_TCGEN05) return true;
    if (h->desc.path != EVA_PATH_AUTO || B < kDequantMinBatch) return false;
    if (!h->dq_ok) return B >= kTcResidMinBatch;
    return B >= kTcMinBatch && h->desc.codebook_rows == 0;
}

bool use_dequant(const eva_vq_linear *h, int B) {
    if (!h->dq_ok || use_tc(h, B)) return false;
    if (h->desc.path == EVA_PATH_DEQUANT_MMA) return true;
    return h->desc.path == EVA_PATH_AUTO && B >= dequant_min_batch(h->desc);
}

// Tensor memory per tcgen05-path CTA (columns) and the dynamic shared memory
// that goes with it: with 256 columns at least 80 KB, so no more than two
// CTAs share an SM; with 512 at least 116 KB, so one CTA has the SM.  Either
// way the allocations of the CTAs on an SM fit in its 512 columns together,
// and an allocation never waits for another CTA's.
constexpr int kTcTmemCols = 256;
size_t tc_smem(const TcLayout &L, int tmem_cols = kTcTmemCols) {
    return std::max((size_t)L.total, (size_t)(tmem_cols > 256 ? 116 : 80) * 1024);
}

using TcFn = void (*)(TcParams);
TcFn tc_fn(bool resid) { return resid ? eva_tc_kernel<true> : eva_tc_kernel<false>; }

// CTAs per 128-row block (one cluster of Gs, consecutive K ranges) for Np
// padded tokens: the fewest rounds of resident CTAs times the stages of the
// longest K range, plus a share for the cluster reduction; 0 if nothing fits.
int plan_tc(eva_vq_linear *h, int Np) {
    const eva_vq_desc &d = h->desc;
    const int R = (d.N + kTcRows - 1) / kTcRows, KB = d.K / kTcStageK;
    const bool resid = d.residual_group != 0;
    const TcFn fn = tc_fn(resid);
    double best = 1e300;
    int pick = 0;
    for (int gs = 1; gs <= std::min(16, KB); gs *= 2) {   // a power of two: it divides the 128 rows
        const TcLayout L = tc_layout(KB, gs, Np, resid ? 1 : 0);
        if (tc_smem(L) > (size_t)h->smem_optin) continue;
        int resident = 0;
        if (gs > 1) {
            resident = max_active_clusters((LookupFn)fn, tc_smem(L), gs, kTcThreads) * gs;
        } else {
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, (const void *)fn, kTcThreads, tc_smem(L)) !=
                cudaSuccess) {
                cudaGetLastError();
                per_sm = 0;
            }
            resident = per_sm * h->sm_count;
        }
        // One CTA per SM of this layer at a time: in a chain of calls the next
        // layer's early-launched CTAs (programmatic dependent launch) hold the
        // other slot while they wait.
        resident = std::min(resident, h->sm_count);
        if (resident <= 0) continue;
        const int rounds = (R * gs + resident - 1) / resident;
        const double cost = (double)rounds * (300.0 + 160.0 * ((KB + gs - 1) / gs)) + (gs > 1 ? 700.0 + 40.0 * gs : 0.0);
        if (cost < best) {
            best = cost;
            pick = gs;
        }
    }
    return pick;
}

void free_handle(eva_vq_linear *h) {
    if (!h) return;
    for (auto &hg : h->host_graph)
        if (hg.exec) cudaGraphExecDestroy(hg.exec);
    if (h->capture_stream) cudaStreamDestroy(h->capture_stream);
    void *ptrs[] = {h->wi, h->sg, h->al, h->wc, h->hsign, h->h28, h->status, h->x_stage,
                    h->y_stage, h->timeline, h->wib, h->sgb, h->al_rm, h->xrot, h->sgd};
    for (void *p : ptrs)
        if (p) cudaFree(p);
    delete h;
}

template <typename T>
cudaError_t dalloc(T **p, size_t bytes, int64_t *acc) {
    *p = nullptr;
    if (bytes == 0) return cudaSuccess;
    cudaError_t e = cudaMalloc(reinterpret_cast<void **>(p), bytes);
    if (e == cudaSuccess && acc) *acc += (int64_t)bytes;
    return e;
}

unsigned blocks_for(long long total, int threads) { return (unsigned)((total + threads - 1) / threads); }

}  // namespace

extern "C" {

const char *eva_vq_status_string(eva_status_t s) {
    switch (s) {
        case EVA_OK: return "ok";
        case EVA_ERR_INVALID_ARG: return "invalid argument";
        case EVA_ERR_UNSUPPORTED: return "unsupported configuration";
        case EVA_ERR_CUDA: return "CUDA runtime error";
        case EVA_ERR_OOM: return "device allocation failed";
        case EVA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case EVA_ERR_NO_DEVICE: return "no sm_100 device";
        case EVA_ERR_DEVICE_CHECK: return "device-side bounds check failed (checked build)";
        case EVA_ERR_SCRATCH_TOO_SMALL:
            return "B * K * 4 bytes exceed the 4 MiB static scratch of eva_vq_linear_run_noalloc";
    }
    return "unknown status";
}

eva_status_t eva_vq_linear_create(eva_vq_linear_t *out, const eva_vq_desc *desc, const void *wc,
                                  const uint8_t *wi, const uint8_t *signs, const void *alpha,
                                  const int8_t *hsign, eva_stream_t stream) {
    if (!out) return EVA_ERR_INVALID_ARG;
    *out = nullptr;
    eva_status_t st = validate_desc(desc);
    if (st != EVA_OK) return st;
    if (!wc || !wi || !aligned16(wc) || !aligned16(wi)) return EVA_ERR_INVALID_ARG;
    if (desc->residual_group) {
        if (!signs || !alpha || !aligned16(signs) || !aligned16(alpha)) return EVA_ERR_INVALID_ARG;
    } else if (signs || alpha) {
        return EVA_ERR_INVALID_ARG;
    }
    if (desc->hadamard_block) {
        if (!hsign || !aligned16(hsign)) return EVA_ERR_INVALID_ARG;
    } else if (hsign) {
        return EVA_ERR_INVALID_ARG;
    }

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return EVA_ERR_NO_DEVICE;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return EVA_ERR_NO_DEVICE;
    if (prop.major != 10) return EVA_ERR_NO_DEVICE;

    eva_vq_linear *h = new (std::nothrow) eva_vq_linear();
    if (!h) return EVA_ERR_OOM;
    h->desc = *desc;
    h->device = dev;
    h->sm_count = prop.multiProcessorCount;
    h->smem_per_sm = (int)prop.sharedMemPerMultiprocessor;
    h->smem_reserved = (int)prop.reservedSharedMemPerBlock;
    h->smem_optin = (int)prop.sharedMemPerBlockOptin;
    h->regs_per_sm = prop.regsPerMultiprocessor;
    const int N = desc->N, K = desc->K;
    h->J = K / kD;
    h->S = (h->J + kSliceJ - 1) / kSliceJ;
    h->T = (N + kTileRows - 1) / kTileRows;
    h->Npad = h->T * kTileRows;
    h->G = desc->codebook_rows ? N / desc->codebook_rows : 1;
    h->tiles_per_cb = desc->codebook_rows ? desc->codebook_rows / kTileRows : 0;
    h->ncent = 1 << desc->index_bits;
    h->unit_bytes = desc->index_bits == 4 ? kUnitBytes4 : kUnitBytes;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long units = (long long)h->S * h->T;
    int64_t ws = 0;
    cudaError_t e = cudaSuccess;
    auto chk = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
    chk(set_smem_attrs(h->smem_optin));
    plan_grid(h, 0);
    if (desc->max_batch > 1) plan_grid(h, 1);
    int max_grid = std::max(h->plan[0].Gs * h->plan[0].Gt, h->plan[1].Gs * h->plan[1].Gt);
    // Residual and rotated layers on the dequantize path (one shared codebook):
    // its own sign units beside the lookup's alpha units, and the rotated x in
    // the workspace the tcgen05 path uses too.
    const bool dq_resrot = desc->residual_group || desc->hadamard_block;
    if (desc->index_bits == 8 && (!dq_resrot || !desc->codebook_rows) &&
        (desc->path == EVA_PATH_DEQUANT_MMA ||
         (desc->path == EVA_PATH_AUTO && desc->max_batch >= dequant_min_batch(*desc)))) {
        plan_dequant(h, 1);
        plan_dequant(h, 2);
        h->dq_ok = h->dq[0].Gs > 0 && h->dq[1].Gs > 0;
        if (h->dq_ok) max_grid = std::max({max_grid, h->dq[0].Gs * h->dq[0].Gt, h->dq[1].Gs * h->dq[1].Gt});
        else if (desc->path == EVA_PATH_DEQUANT_MMA) {
            free_handle(h);
            return EVA_ERR_UNSUPPORTED;
        }
    }
    if (tc_layer_ok(*desc) && (desc->path == EVA_PATH_TCGEN05 || (desc->path == EVA_PATH_AUTO && auto_may_use_tc(h)))) {
        // Plans for the padded batches up to max_batch; a batch whose padded
        // size has no plan (its x range does not fit in shared memory) runs
        // as several launches of the largest size that has one.
        for (int i = 0; i < 4 && 16 * i < desc->max_batch; ++i) {
            h->tc_gs[i] = plan_tc(h, 16 * (i + 1));
            max_grid = std::max(max_grid, h->tc_gs[i] * ((N + kTcRows - 1) / kTcRows));
        }
        h->tc_ok = h->tc_gs[0] > 0;
        if (!h->tc_ok && desc->path == EVA_PATH_TCGEN05) {
            free_handle(h);
            return EVA_ERR_UNSUPPORTED;
        }
    }
    chk(dalloc(&h->wi, (size_t)units * h->unit_bytes, nullptr));
    const int R128 = (N + kTcRows - 1) / kTcRows;
    if (h->tc_ok) {
        chk(dalloc(&h->wib, (size_t)R128 * kTcRows * h->J, nullptr));
        if (desc->residual_group) {
            chk(dalloc(&h->sgb, (size_t)R128 * kTcRows * (K / 8), nullptr));
            chk(dalloc(&h->al_rm, (size_t)N * (K / desc->residual_group) * sizeof(__half), nullptr));
        }
    }
    if ((h->tc_ok || h->dq_ok) && desc->hadamard_block)
        chk(dalloc(&h->xrot, (size_t)desc->max_batch * K * sizeof(float), &ws));
    if (h->dq_ok && desc->residual_group) chk(dalloc(&h->sgd, (size_t)units * kDqSignUnitBytes, nullptr));
    chk(dalloc(&h->wc, (size_t)h->G * h->ncent * kD * sizeof(__half), nullptr));
    if (desc->residual_group) {
        chk(dalloc(&h->sg, (size_t)units * kSignUnitBytes, nullptr));
        chk(dalloc(&h->al, (size_t)units * kAlphaUnitHalves * sizeof(__half), nullptr));
    }
    if (desc->hadamard_block) {
        chk(dalloc(&h->hsign, (size_t)K, nullptr));
    }
    chk(dalloc(&h->status, 8 * sizeof(int), &ws));
#ifdef EVA_TIMELINE
    chk(dalloc(&h->timeline, (size_t)max_grid * 8 * sizeof(unsigned long long), &ws));
    if (e == cudaSuccess) chk(cudaMemsetAsync(h->timeline, 0, (size_t)max_grid * 8 * 8, s));
#endif
    const size_t ybytes = (size_t)desc->max_batch * N * (desc->out_dtype == EVA_F32 ? 4 : 2);
    chk(dalloc(&h->x_stage, (size_t)desc->max_batch * K * sizeof(__half), &ws));
    chk(dalloc(&h->y_stage, ybytes, &ws));
    h->workspace_bytes = ws;
    if (e != cudaSuccess) {
        free_handle(h);
        return cuda_status(e);
    }

    const int thr = 256;
    const long long wib = units * h->unit_bytes;
    if (desc->index_bits == 4)
        eva_repack_wi4_kernel<<<blocks_for(wib, thr), thr, 0, s>>>(wi, h->wi, N, h->J, h->T, wib);
    else
        eva_repack_wi_kernel<<<blocks_for(wib, thr), thr, 0, s>>>(wi, h->wi, N, h->J, h->T, wib);
    chk(cudaGetLastError());
    chk(cudaMemcpyAsync(h->wc, wc, (size_t)h->G * h->ncent * kD * sizeof(__half), cudaMemcpyDeviceToDevice, s));
    if (desc->residual_group) {
        const long long sb = units * kSignUnitBytes, ab = units * kAlphaUnitHalves;
        eva_repack_signs_kernel<<<blocks_for(sb, thr), thr, 0, s>>>(signs, h->sg, N, K / 8, h->T, sb);
        chk(cudaGetLastError());
        eva_repack_alpha_kernel<<<blocks_for(ab, thr), thr, 0, s>>>(
            reinterpret_cast<const __half *>(alpha), h->al, N, K / desc->residual_group, h->T, ab);
        chk(cudaGetLastError());
    }
    if (h->dq_ok && desc->residual_group) {
        const long long sb = units * kDqSignUnitBytes;
        eva_repack_signs_dq_kernel<<<blocks_for(sb, thr), thr, 0, s>>>(signs, h->sgd, N, K, h->T, sb);
        chk(cudaGetLastError());
    }
    if (h->tc_ok) {
        const long long nb = (long long)R128 * kTcRows * h->J;
        eva_repack_wi_rowblock_kernel<<<blocks_for(nb, thr), thr, 0, s>>>(wi, h->wib, N, h->J, nb);
        chk(cudaGetLastError());
        if (desc->residual_group) {
            const long long ns = (long long)R128 * kTcRows * (K / 8);
            eva_repack_signs_rowblock_kernel<<<blocks_for(ns, thr), thr, 0, s>>>(signs, h->sgb, N, K / 8, ns);
            chk(cudaGetLastError());
            chk(cudaMemcpyAsync(h->al_rm, alpha, (size_t)N * (K / desc->residual_group) * sizeof(__half),
                                cudaMemcpyDeviceToDevice, s));
        }
    }
    if (desc->hadamard_block) chk(cudaMemcpyAsync(h->hsign, hsign, (size_t)K, cudaMemcpyDeviceToDevice, s));
    if (paley_m(desc->hadamard_block)) {
        int8_t tab[28 * 28];
        paley28_table(tab);
        chk(dalloc(&h->h28, sizeof(tab), nullptr));
        if (e == cudaSuccess) chk(cudaMemcpy(h->h28, tab, sizeof(tab), cudaMemcpyHostToDevice));
    }
    chk(cudaMemsetAsync(h->status, 0, 8 * sizeof(int), s));
    if (e != cudaSuccess) {
        cudaStreamSynchronize(s);
        free_handle(h);
        return cuda_status(e);
    }
    *out = h;
    return EVA_OK;
}

eva_status_t eva_vq_linear_run(eva_vq_linear_t h, const void *x, int32_t B, void *y, eva_stream_t stream) {
    return eva_vq_linear_run_ex(h, x, B, y, stream, 0u);
}

}  // extern "C"

namespace {
// Parameters of one call of the lookup kernel (arguments already checked).
LookupParams call_params(eva_vq_linear *h, const void *x, int32_t B, void *y, int independent, size_t *smem) {
    const eva_vq_desc &d = h->desc;
    LookupParams p;
    std::memset(&p, 0, sizeof(p));
    p.wi = h->wi;
    p.sg = h->sg;
    p.al = h->al;
    p.wc = h->wc;
    p.x = x;
    p.x_f32 = 0;
    p.y = y;
    p.N = d.N;
    p.Npad = h->Npad;
    p.K = d.K;
    p.S = h->S;
    p.T = h->T;
    p.B = B;
    const eva_vq_linear::Plan &pl = call_plan(h, B, independent);
    p.Gs = pl.Gs;
    p.Gt = pl.Gt;
    p.acc_tiles = (h->T + pl.Gt - 1) / pl.Gt;
    // A call that waits for its predecessor copies its first indices into
    // shared memory while it waits.  An independent call starts at once and
    // streams them through registers, leaving the shared-memory bandwidth to
    // the lookups of the calls it overlaps with.
    p.wi_staged = independent ? 0 : pl.staged;
    p.status = h->status;
    p.wait_rounds = kWaitRounds;
    p.tiles_per_cb = h->tiles_per_cb;
    p.ncent = h->ncent;
    p.out_f32 = d.out_dtype == EVA_F32 ? 1 : 0;
    p.independent = independent;
    if (d.hadamard_block) {   // the rotation runs inside the lookup kernel
        p.rot_b = d.hadamard_block;
        p.rot_m = paley_m(d.hadamard_block);
        p.h28 = h->h28;
        p.hs = h->hsign;
        p.rot_scale = (float)(1.0 / std::sqrt((double)d.hadamard_block));
    }
    *smem = p.wi_staged ? pl.smem : pl.smem_nostage;
#ifdef EVA_TIMELINE
    p.timeline = h->timeline;
#endif
#ifdef EVA_DEVICE_CHECKS
    {
        const long long units = (long long)h->S * h->T;
        const void *base[8] = {h->wi, h->sg, h->al, h->wc, p.x, nullptr, nullptr, y};
        const unsigned long long bytes[8] = {
            (unsigned long long)units * h->unit_bytes,
            h->sg ? (unsigned long long)units * kSignUnitBytes : 0ull,
            h->al ? (unsigned long long)units * kAlphaUnitHalves * 2 : 0ull,
            (unsigned long long)h->G * h->ncent * kD * 2,
            (unsigned long long)B * d.K * (p.x_f32 ? 4 : 2),
            0ull,
            0ull,
            (unsigned long long)B * d.N * (p.out_f32 ? 4 : 2)};
        for (int i = 0; i < 8; ++i) {
            p.chk_base[i] = base[i];
            p.chk_bytes[i] = bytes[i];
        }
        p.smem_bytes = (unsigned)*smem;
        p.chk_record = h->status;
    }
#endif
    return p;
}

// The layers a grouped launch can take: one lookup-kernel instance for all
// (8-bit indices, shared codebook, no rotation, the lookup path at this B).
bool groupable(const eva_vq_linear *h, int B) {
    const eva_vq_desc &d = h->desc;
    return d.index_bits == 8 && !d.codebook_rows && !d.hadamard_block && !use_dequant(h, B) && !use_tc(h, B);
}

using GroupFn = void (*)(LookupGroup);
GroupFn group_fn(bool pair_t, bool resid) {
    if (pair_t) return resid ? eva_lookup_group_kernel<true, true> : eva_lookup_group_kernel<true, false>;
    return resid ? eva_lookup_group_kernel<false, true> : eva_lookup_group_kernel<false, false>;
}
}  // namespace

namespace {
// One call on the tcgen05 path: for a rotated layer the standalone rotation
// kernel first writes x~ (fp32) into `xrot`, then the tensor-core kernel.
// x~ of a rotated layer into `xrot` (fp32 [B][K]) with the standalone
// rotation kernel (Sylvester or Paley blocks).
cudaError_t launch_rotation(const eva_vq_linear *h, const void *x, int B, cudaStream_t s, int independent,
                            float *xrot) {
    const eva_vq_desc &d = h->desc;
    const int b = d.hadamard_block, m = paley_m(b), thr = std::min(b / 2, 1024);
    const float scale = (float)(1.0 / std::sqrt((double)b));
    if (m)
        return launch_pdl(eva_paley_x_kernel, dim3(28 * (d.K / b), B), dim3(m), (size_t)m * sizeof(float), s, 0,
                          reinterpret_cast<const __half *>(x), (const int8_t *)h->hsign, (const int8_t *)h->h28,
                          xrot, d.K, b, m, scale, independent);
    return launch_pdl(eva_hadamard_kernel, dim3(d.K / b, B), dim3(thr), (size_t)b * sizeof(float), s, 0,
                      reinterpret_cast<const __half *>(x), (const int8_t *)h->hsign, xrot, d.K, b, scale,
                      independent);
}

cudaError_t launch_tc(eva_vq_linear *h, const void *x, int B, void *y, cudaStream_t s, int independent,
                      float *xrot) {
    const eva_vq_desc &d = h->desc;
    int kernels = 0;
    cudaError_t e;
    const void *xin = x;
    int x_f32 = 0;
    if (d.hadamard_block) {
        e = launch_rotation(h, x, B, s, independent, xrot);
        if (e != cudaSuccess) return e;
        xin = xrot;
        x_f32 = 1;
        independent = 0;    // the tensor-core kernel reads the rotation kernel's output
        ++kernels;
    }
    // The largest padded batch with a plan takes the tokens in chunks.
    int imax = 0;
    for (int i = 0; i < 4; ++i)
        if (h->tc_gs[i]) imax = i;
    const int ybytes = d.out_dtype == EVA_F32 ? 4 : 2, xbytes = x_f32 ? 4 : 2;
    int grid = 0;
    for (int b0 = 0; b0 < B; b0 += 16 * (imax + 1)) {
        const int nb = std::min(B - b0, 16 * (imax + 1));
        const int Np = ((nb + 15) / 16) * 16;
        const int gs = h->tc_gs[Np / 16 - 1];
        TcParams p;
        std::memset(&p, 0, sizeof(p));
        p.wib = h->wib;
        p.wc = h->wc;
        p.sg = h->sgb;
        p.al = h->al_rm;
        p.x = static_cast<const char *>(xin) + (size_t)b0 * d.K * xbytes;
        p.y = static_cast<char *>(y) + (size_t)b0 * d.N * ybytes;
        p.N = d.N;
        p.K = d.K;
        p.B = nb;
        p.Np = Np;
        p.R = (d.N + kTcRows - 1) / kTcRows;
        p.KB = d.K / kTcStageK;
        p.Gs = gs;
        p.rows_per_cb = d.codebook_rows;
        p.x_f32 = x_f32;
        p.out_f32 = d.out_dtype == EVA_F32 ? 1 : 0;
        p.independent = independent;
        p.resid = d.residual_group != 0;
        p.status = h->status;
        p.wait_rounds = kWaitRounds;
        p.tmem_cols = kTcTmemCols;
        p.nbuf = std::min(kTcMaxBufs, (p.tmem_cols - ((Np + 31) & ~31)) / kTcStageCols);
#ifdef EVA_TIMELINE
        p.timeline = h->timeline;
#endif
        const TcLayout L = tc_layout(p.KB, gs, Np, p.resid);
        e = launch_pdl(tc_fn(p.resid != 0), dim3(p.R * gs), dim3(kTcThreads), tc_smem(L, p.tmem_cols), s,
                       gs > 1 ? gs : 0, p);
        if (e != cudaSuccess) return e;
        grid = p.R * gs;
        ++kernels;
    }
    h->last_grid = grid;
    h->last_kernels = kernels;
    h->last_path = EVA_PATH_TCGEN05;
    return cudaSuccess;
}
}  // namespace

extern "C" {

eva_status_t eva_vq_linear_run_ex(eva_vq_linear_t h, const void *x, int32_t B, void *y, eva_stream_t stream,
                                  uint32_t flags) {
    if (!h || !x || !y || !aligned16(x) || !aligned16(y)) return EVA_ERR_INVALID_ARG;
    if (flags & ~(uint32_t)EVA_RUN_INDEPENDENT) return EVA_ERR_INVALID_ARG;
    const int independent = (flags & EVA_RUN_INDEPENDENT) ? 1 : 0;
    if (B < 1 || B > h->desc.max_batch) return EVA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const eva_vq_desc &d = h->desc;
    size_t smem = 0;
    cudaError_t e;
    if (use_tc(h, B)) return cuda_status(launch_tc(h, x, B, y, s, independent, h->xrot));
    LookupParams p = call_params(h, x, B, y, independent, &smem);
    if (use_dequant(h, B)) {
        size_t dsmem = 0;
        int dgrid = 0;
        const bool rot_kernel = d.hadamard_block && !dq_rotates_on_chip(h, B);
        if (rot_kernel) {
            // The dequantize kernel reads x~ (fp32) from the rotation kernel.
            e = launch_rotation(h, x, B, s, independent, h->xrot);
            if (e != cudaSuccess) return cuda_status(e);
            p.x = h->xrot;
            p.x_f32 = 1;
            p.independent = 0;
        }
        e = launch_dequant(h, p, B, s, &dsmem, &dgrid);
        if (e != cudaSuccess) return cuda_status(e);
        h->last_grid = dgrid;
        h->last_kernels = rot_kernel ? 2 : 1;
        h->last_path = EVA_PATH_DEQUANT_MMA;
        return EVA_OK;
    }
    const bool pair_t = B > 1, resid = d.residual_group != 0;
    const eva_vq_linear::Plan &pl = call_plan(h, B, independent);
    LookupFn fn = lookup_fn(pair_t, resid, h->tiles_per_cb != 0, p.rot_b != 0, d.index_bits == 4);
    if (independent && use_three_per_sm(h, B, independent)) fn = lookup_fn3(h->tiles_per_cb != 0, d.index_bits == 4);
    apply_injection(h, p);
    e = launch_pdl(fn, dim3(pl.Gs * pl.Gt), dim3(kThreads), smem, s, pl.Gs, p);
    if (e != cudaSuccess) return cuda_status(e);
    h->last_grid = pl.Gs * pl.Gt;
    h->last_kernels = 1;
    h->last_path = EVA_PATH_OC_LOOKUP;
    return EVA_OK;
}

eva_status_t eva_vq_linear_run_group(const eva_vq_linear_t *hs, const void *const *xs, void *const *ys,
                                     int32_t count, int32_t B, eva_stream_t stream, uint32_t flags) {
    if (!hs || !xs || !ys || count < 1 || count > kMaxGroup) return EVA_ERR_INVALID_ARG;
    if (flags & ~(uint32_t)EVA_RUN_INDEPENDENT) return EVA_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        const eva_vq_linear_t h = hs[i];
        if (!h || !xs[i] || !ys[i] || !aligned16(xs[i]) || !aligned16(ys[i])) return EVA_ERR_INVALID_ARG;
        if (B < 1 || B > h->desc.max_batch || h->device != hs[0]->device) return EVA_ERR_INVALID_ARG;
    }
    const eva_vq_desc &d0 = hs[0]->desc;
    const int independent = (flags & EVA_RUN_INDEPENDENT) ? 1 : 0;
    // Layers of one shape on the dequantize path (one shared codebook each, no
    // residual, no rotation): one launch of the dequantize kernel.
    const auto dq_plain = [](const eva_vq_desc &d) {
        return !d.codebook_rows && !d.residual_group && !d.hadamard_block;
    };
    bool dq_one = use_dequant(hs[0], B) && dq_plain(d0) && count > 1;
    for (int i = 1; i < count && dq_one; ++i) {
        const eva_vq_desc &d = hs[i]->desc;
        dq_one = use_dequant(hs[i], B) && dq_plain(d) && d.N == d0.N && d.K == d0.K &&
                 d.out_dtype == d0.out_dtype && hs[i]->dq[B > 8 ? 1 : 0].Gs == hs[0]->dq[B > 8 ? 1 : 0].Gs &&
                 hs[i]->dq[B > 8 ? 1 : 0].Gt == hs[0]->dq[B > 8 ? 1 : 0].Gt &&
                 hs[i]->dq[B > 8 ? 1 : 0].smem == hs[0]->dq[B > 8 ? 1 : 0].smem;
    }
    if (dq_one) {
        LookupGroup g;
        std::memset(&g, 0, sizeof(g));
        size_t smem = 0;
        for (int i = 0; i < count; ++i) {
            g.p[i] = call_params(hs[i], xs[i], B, ys[i], independent, &smem);
            dequant_params(hs[i], g.p[i], B);
        }
        const int ntg = B > 8 ? 2 : 1;
        const eva_vq_linear::Plan &pl = hs[0]->dq[ntg - 1];
        g.count = count;
        g.ctas_per_layer = pl.Gs * pl.Gt;
        const bool direct = dequant_direct(hs[0], B);
        using DqGroupFn = void (*)(LookupGroup);
        const DqGroupFn fn = ntg == 2 ? (direct ? eva_dequant_group_kernel<2, true> : eva_dequant_group_kernel<2, false>)
                                      : (direct ? eva_dequant_group_kernel<1, true> : eva_dequant_group_kernel<1, false>);
        const cudaError_t e = launch_pdl(fn, dim3(count * pl.Gs * pl.Gt), dim3(kThreads), pl.smem,
                                         reinterpret_cast<cudaStream_t>(stream), pl.Gs, g);
        if (e != cudaSuccess) return cuda_status(e);
        for (int i = 0; i < count; ++i) {
            hs[i]->last_grid = pl.Gs * pl.Gt;
            hs[i]->last_kernels = 1;
            hs[i]->last_path = EVA_PATH_DEQUANT_MMA;
        }
        return EVA_OK;
    }
    // One launch when every layer has the first one's shape and format.
    bool one = groupable(hs[0], B);
    for (int i = 1; i < count && one; ++i) {
        const eva_vq_desc &d = hs[i]->desc;
        one = groupable(hs[i], B) && d.N == d0.N && d.K == d0.K && d.residual_group == d0.residual_group &&
              d.out_dtype == d0.out_dtype;
    }
    if (!one) {
        for (int i = 0; i < count; ++i) {
            const eva_status_t st = eva_vq_linear_run_ex(hs[i], xs[i], B, ys[i], stream, flags);
            if (st != EVA_OK) return st;
        }
        return EVA_OK;
    }
    LookupGroup g;
    std::memset(&g, 0, sizeof(g));
    size_t smem = 0;
    for (int i = 0; i < count; ++i) g.p[i] = call_params(hs[i], xs[i], B, ys[i], independent, &smem);
    const bool pair_t = B > 1;
    const eva_vq_linear::Plan &pl = call_plan(hs[0], B, independent);
    g.count = count;
    g.ctas_per_layer = pl.Gs * pl.Gt;
    const cudaError_t e = launch_pdl(group_fn(pair_t, d0.residual_group != 0), dim3(count * pl.Gs * pl.Gt),
                                     dim3(kThreads), smem, reinterpret_cast<cudaStream_t>(stream), pl.Gs, g);
    if (e != cudaSuccess) return cuda_status(e);
    for (int i = 0; i < count; ++i) {
        hs[i]->last_grid = pl.Gs * pl.Gt;
        hs[i]->last_kernels = 1;
        hs[i]->last_path = EVA_PATH_OC_LOOKUP;
    }
    return EVA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free run.  eva_vq_linear_run computes the rotated input of a
// 3.125-bit layer on chip, inside the lookup kernel; this variant keeps the
// two-kernel route (a standalone rotation kernel, then the lookups), whose
// rotated input goes through one file-scope device array rather than memory
// anyone allocates, so the call never goes near the device allocator.
namespace {
constexpr size_t kStaticScratchBytes = (size_t)4 << 20;   // 4 MiB: B * K * 4 bytes at most
}
static __device__ __align__(256) float eva_static_scratch[kStaticScratchBytes / sizeof(float)];

namespace {
std::mutex g_scratch_mu;
float *g_scratch_dev[128] = {};   // device address of eva_static_scratch, per device ordinal

// The host-side symbol is a stand-in, not a device address: look the real
// address up once per device, with that device current.
eva_status_t static_scratch(int dev, float **out) {
    if (dev < 0 || dev >= 128) return EVA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_dev[dev]) {
        void *ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, eva_static_scratch);
        if (e != cudaSuccess || !ptr) return EVA_ERR_CUDA;
        g_scratch_dev[dev] = static_cast<float *>(ptr);
    }
    *out = g_scratch_dev[dev];
    return EVA_OK;
}
}  // namespace

extern "C" {

eva_status_t eva_vq_linear_run_noalloc(eva_vq_linear_t h, const void *x, int32_t B, void *y,
                                       eva_stream_t stream) {
    if (!h || !x || !y || !aligned16(x) || !aligned16(y)) return EVA_ERR_INVALID_ARG;
    if (B < 1 || B > h->desc.max_batch) return EVA_ERR_INVALID_ARG;
    const eva_vq_desc &d = h->desc;
    if (use_tc(h, B)) {
        // The tensor-core path of a rotated layer always runs the standalone
        // rotation first; its x~ goes through the static scratch.
        if (d.hadamard_block && (size_t)B * d.K * sizeof(float) > kStaticScratchBytes)
            return EVA_ERR_SCRATCH_TOO_SMALL;
        int dev = -1;
        if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return EVA_ERR_INVALID_ARG;
        float *scratch = nullptr;
        if (d.hadamard_block) {
            const eva_status_t st = static_scratch(dev, &scratch);
            if (st != EVA_OK) return st;
        }
        return cuda_status(launch_tc(h, x, B, y, reinterpret_cast<cudaStream_t>(stream), 0, scratch));
    }
    // A Paley rotation block has no standalone-kernel route that matches the
    // fused rotation bit for bit at every size, so it stays fused (no scratch).
    const bool fused_rot = paley_m(d.hadamard_block) != 0;
    // The dequantize path rotates Sylvester blocks on chip and reads a Paley
    // block's x~ from the standalone rotation kernel; the lookup path the
    // other way round.
    const bool dq = use_dequant(h, B);
    const bool rot_scratch = d.hadamard_block && (dq ? !dq_rotates_on_chip(h, B) : !fused_rot);
    if (rot_scratch && (size_t)B * d.K * sizeof(float) > kStaticScratchBytes) return EVA_ERR_SCRATCH_TOO_SMALL;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return EVA_ERR_INVALID_ARG;
    float *scratch = nullptr;
    if (rot_scratch) {
        const eva_status_t st = static_scratch(dev, &scratch);
        if (st != EVA_OK) return st;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool pair_t = B > 1;
    const eva_vq_linear::Plan &pl = h->plan[pair_t ? 1 : 0];
    LookupParams p;
    std::memset(&p, 0, sizeof(p));
    p.wi = h->wi;
    p.sg = h->sg;
    p.al = h->al;
    p.wc = h->wc;
    p.x = x;
    p.x_f32 = 0;
    p.y = y;
    p.N = d.N;
    p.Npad = h->Npad;
    p.K = d.K;
    p.S = h->S;
    p.T = h->T;
    p.B = B;
    p.tiles_per_cb = h->tiles_per_cb;
    p.ncent = h->ncent;
    p.out_f32 = d.out_dtype == EVA_F32 ? 1 : 0;
    p.independent = 0;
    p.Gs = pl.Gs;
    p.Gt = pl.Gt;
    p.acc_tiles = (h->T + pl.Gt - 1) / pl.Gt;
    p.wi_staged = pl.staged;
    p.status = h->status;
    p.wait_rounds = kWaitRounds;
#ifdef EVA_TIMELINE
    p.timeline = h->timeline;
#endif
#ifdef EVA_DEVICE_CHECKS
    return EVA_ERR_UNSUPPORTED;   // the checked build validates the handle path only
#endif
    cudaError_t e;
    if (dq) {
        if (rot_scratch) {
            e = launch_rotation(h, x, B, s, 0, scratch);
            if (e != cudaSuccess) return cuda_status(e);
            p.x = scratch;
            p.x_f32 = 1;
        }
    } else if (fused_rot) {
        p.rot_b = d.hadamard_block;
        p.rot_m = paley_m(d.hadamard_block);
        p.h28 = h->h28;
        p.hs = h->hsign;
        p.rot_scale = (float)(1.0 / std::sqrt((double)d.hadamard_block));
    } else if (d.hadamard_block) {
        const int b = d.hadamard_block;
        const int thr = std::min(b / 2, 1024);
        e = launch_pdl(eva_hadamard_kernel, dim3(d.K / b, B), dim3(thr), (size_t)b * sizeof(float), s, 0,
                       reinterpret_cast<const __half *>(x), (const int8_t *)h->hsign, scratch, d.K, b,
                       (float)(1.0 / std::sqrt((double)b)), 0);
        if (e != cudaSuccess) return cuda_status(e);
        p.x = scratch;
        p.x_f32 = 1;
    }
    if (dq) {
        size_t dsmem = 0;
        int dgrid = 0;
        e = launch_dequant(h, p, B, s, &dsmem, &dgrid);
        if (e != cudaSuccess) return cuda_status(e);
        h->last_grid = dgrid;
        h->last_kernels = rot_scratch ? 2 : 1;
        h->last_path = EVA_PATH_DEQUANT_MMA;
        return EVA_OK;
    }
    const bool resid = d.residual_group != 0;
    e = launch_pdl(lookup_fn(pair_t, resid, h->tiles_per_cb != 0, fused_rot, d.index_bits == 4), dim3(pl.Gs * pl.Gt),
                   dim3(kThreads),
                   pl.smem, s, pl.Gs, p);
    if (e != cudaSuccess) return cuda_status(e);
    h->last_grid = pl.Gs * pl.Gt;
    h->last_kernels = (d.hadamard_block && !fused_rot) ? 2 : 1;   // standalone rotation, then the lookups
    h->last_path = EVA_PATH_OC_LOOKUP;
    return EVA_OK;
}

// Inputs up to this size are read by the kernels straight from mapped host
// memory in eva_vq_linear_run_host; larger ones are copied in first (every
// row-group CTA reads x, so a large x would cross the bus several times).
constexpr size_t kZeroCopyMaxBytes = 64 * 1024;

eva_status_t eva_vq_linear_run_host(eva_vq_linear_t h, const void *x_host, int32_t B, void *y_host,
                                    eva_stream_t stream) {
    if (!h || !x_host || !y_host) return EVA_ERR_INVALID_ARG;
    if (B < 1 || B > h->desc.max_batch) return EVA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t xb = (size_t)B * h->desc.K * sizeof(__half);
    const size_t yb = (size_t)B * h->desc.N * (h->desc.out_dtype == EVA_F32 ? 4 : 2);
    // Page-locked host buffers: one graph launch (copy in, run, copy out).
    // Pageable ones: the three operations one by one.
    cudaPointerAttributes ax, ay;
    const bool pinned = cudaPointerGetAttributes(&ax, x_host) == cudaSuccess && ax.type == cudaMemoryTypeHost &&
                        cudaPointerGetAttributes(&ay, y_host) == cudaSuccess && ay.type == cudaMemoryTypeHost;
    cudaGetLastError();
    // Small batches with page-locked buffers: no copies at all -- the kernel
    // reads x from and writes y to the mapped host memory (the same bytes
    // cross the bus, without two copy operations around the launch).
    if (pinned && ax.devicePointer && ay.devicePointer && xb <= kZeroCopyMaxBytes &&
        aligned16(ax.devicePointer) && aligned16(ay.devicePointer)) {
        const eva_status_t st = eva_vq_linear_run(h, ax.devicePointer, B, ay.devicePointer, stream);
        if (st != EVA_OK) return st;
        return cuda_status(cudaStreamSynchronize(s));
    }
    if (pinned && !h->host_graph[B].failed) {
        eva_vq_linear::HostGraph &hg = h->host_graph[B];
        cudaError_t e = cudaSuccess;
        if (!hg.exec) {
            if (!h->capture_stream) {
                e = cudaStreamCreateWithFlags(&h->capture_stream, cudaStreamNonBlocking);
                if (e != cudaSuccess) return cuda_status(e);
            }
            cudaStream_t cs = h->capture_stream;
            e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
            if (e != cudaSuccess) return cuda_status(e);
            cudaError_t e1 = cudaMemcpyAsync(h->x_stage, x_host, xb, cudaMemcpyHostToDevice, cs);
            const eva_status_t st = e1 == cudaSuccess ? eva_vq_linear_run(h, h->x_stage, B, h->y_stage, cs)
                                                      : EVA_ERR_CUDA;
            cudaError_t e2 = st == EVA_OK ? cudaMemcpyAsync(y_host, h->y_stage, yb, cudaMemcpyDeviceToHost, cs)
                                          : cudaSuccess;
            cudaGraph_t graph = nullptr;
            e = cudaStreamEndCapture(cs, &graph);
            if (st == EVA_ERR_INVALID_ARG) {
                if (graph) cudaGraphDestroy(graph);
                return st;
            }
            if (st != EVA_OK || e1 != cudaSuccess || e2 != cudaSuccess || e != cudaSuccess) {
                if (graph) cudaGraphDestroy(graph);
                cudaGetLastError();
                hg.failed = true;
                return eva_vq_linear_run_host(h, x_host, B, y_host, stream);
            }
            // The two memcpy nodes: the first is the copy in, the last the copy out.
            size_t n = 0;
            cudaGraphGetNodes(graph, nullptr, &n);
            cudaGraphNode_t nodes[16];
            if (n > 16) n = 16;
            cudaGraphGetNodes(graph, nodes, &n);
            for (size_t i = 0; i < n; ++i) {
                cudaGraphNodeType t;
                cudaGraphNodeGetType(nodes[i], &t);
                if (t != cudaGraphNodeTypeMemcpy) continue;
                cudaMemcpy3DParms mp;
                if (cudaGraphMemcpyNodeGetParams(nodes[i], &mp) != cudaSuccess) continue;
                if (mp.srcPtr.ptr == x_host || mp.dstPtr.ptr == h->x_stage) hg.h2d = nodes[i];
                else if (mp.dstPtr.ptr == y_host || mp.srcPtr.ptr == h->y_stage) hg.d2h = nodes[i];
            }
            e = cudaGraphInstantiate(&hg.exec, graph, 0);
            cudaGraphDestroy(graph);
            if (e != cudaSuccess || !hg.h2d || !hg.d2h) {
                if (hg.exec) cudaGraphExecDestroy(hg.exec);
                cudaGetLastError();
                hg = eva_vq_linear::HostGraph();
                hg.failed = true;
                return eva_vq_linear_run_host(h, x_host, B, y_host, stream);
            }
            hg.x = x_host;
            hg.y = y_host;
        }
        if (hg.x != x_host || hg.y != y_host) {
            // New host buffers: update the two copies in place, or, where the
            // runtime refuses that, capture the graph again for them.
            e = cudaGraphExecMemcpyNodeSetParams1D(hg.exec, hg.h2d, h->x_stage, x_host, xb, cudaMemcpyHostToDevice);
            if (e == cudaSuccess)
                e = cudaGraphExecMemcpyNodeSetParams1D(hg.exec, hg.d2h, y_host, h->y_stage, yb, cudaMemcpyDeviceToHost);
            if (e != cudaSuccess) {
                cudaGetLastError();
                cudaGraphExecDestroy(hg.exec);
                hg = eva_vq_linear::HostGraph();
                return eva_vq_linear_run_host(h, x_host, B, y_host, stream);
            }
            hg.x = x_host;
            hg.y = y_host;
        }
        e = cudaGraphLaunch(hg.exec, s);
        if (e != cudaSuccess) return cuda_status(e);
        return cuda_status(cudaStreamSynchronize(s));
    }
    cudaError_t e = cudaMemcpyAsync(h->x_stage, x_host, xb, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_status(e);
    eva_status_t st = eva_vq_linear_run(h, h->x_stage, B, h->y_stage, stream);
    if (st != EVA_OK) return st;
    e = cudaMemcpyAsync(y_host, h->y_stage, yb, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(cudaStreamSynchronize(s));
}

eva_status_t eva_vq_linear_destroy(eva_vq_linear_t h) {
    free_handle(h);
    return EVA_OK;
}

eva_status_t eva_vq_unpack_indices(eva_vq_linear_t h, uint8_t *wi_out, eva_stream_t stream) {
    if (!h || !wi_out) return EVA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (h->desc.index_bits == 4) {   // canonical packed [N][J/2]
        const long long total = (long long)h->desc.N * (h->J / 2);
        eva_unpack_wi4_kernel<<<blocks_for(total, 256), 256, 0, s>>>(h->wi, wi_out, h->desc.N, h->J, h->T, total);
        return cuda_status(cudaGetLastError());
    }
    const long long total = (long long)h->S * h->T * kUnitBytes;
    eva_unpack_wi_kernel<<<blocks_for(total, 256), 256, 0, s>>>(h->wi, wi_out, h->desc.N, h->J, h->T, total);
    return cuda_status(cudaGetLastError());
}

eva_status_t eva_vq_sync_status(eva_vq_linear_t h) {
    if (!h) return EVA_ERR_INVALID_ARG;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e);
    int word = 0;
    e = cudaMemcpy(&word, h->status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
#ifdef EVA_DEVICE_CHECKS
    return word ? EVA_ERR_DEVICE_CHECK : EVA_OK;
#else
    return word ? EVA_ERR_DEVICE_TIMEOUT : EVA_OK;
#endif
}

eva_status_t eva_vq_debug_inject_wait_timeout(eva_vq_linear_t h, int32_t rounds) {
    if (!h || rounds < 1 || rounds > kWaitRounds) return EVA_ERR_INVALID_ARG;
    h->inject_wait_rounds = rounds;
    return EVA_OK;
}

eva_status_t eva_vq_device_check_record(eva_vq_linear_t h, int32_t *out8) {
    if (!h || !out8) return EVA_ERR_INVALID_ARG;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(cudaMemcpy(out8, h->status, 8 * sizeof(int), cudaMemcpyDeviceToHost));
}

eva_status_t eva_vq_debug_timeline(eva_vq_linear_t h, uint64_t *out, int32_t max_entries, int32_t *count) {
    if (!h || !out || !count || max_entries < 0) return EVA_ERR_INVALID_ARG;
    *count = 0;
#ifdef EVA_TIMELINE
    const int n = std::min(max_entries, h->last_grid * 8);
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(out, h->timeline, (size_t)n * 8, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    *count = n;
    return EVA_OK;
#else
    return EVA_ERR_UNSUPPORTED;
#endif
}

eva_status_t eva_vq_linear_info(eva_vq_linear_t h, eva_vq_info *info) {
    if (!h || !info) return EVA_ERR_INVALID_ARG;
    const eva_vq_desc &d = h->desc;
    std::memset(info, 0, sizeof(*info));
    info->wi_bytes = (int64_t)d.N * (d.K / kD) * d.index_bits / 8;
    info->sign_bytes = d.residual_group ? (int64_t)d.N * (d.K / 8) : 0;
    info->alpha_bytes = d.residual_group ? (int64_t)d.N * (d.K / d.residual_group) * 2 : 0;
    info->codebook_bytes = (int64_t)h->G * h->ncent * kD * 2;
    info->stream_bytes = info->wi_bytes + info->sign_bytes + info->alpha_bytes + (int64_t)d.K * 2;
    info->workspace_bytes = h->workspace_bytes;
    info->slices = h->S;
    info->row_tiles = h->T;
    info->grid = h->last_grid ? h->last_grid : h->plan[0].Gs * h->plan[0].Gt;
    info->kernels_per_run = h->last_kernels ? h->last_kernels : 1;
    info->path = h->last_path ? h->last_path : EVA_PATH_OC_LOOKUP;
    info->sm_count = h->sm_count;
    info->staged_units = call_plan(h, 1, 0).staged;
    return EVA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Offline quantizer (3-bit SRAM-lookup article, quantize() sample).
namespace {

bool aligned16c(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

eva_status_t kmeans_args(const float *v, int64_t M, int32_t d, const float *cent, int32_t ncent,
                         int64_t vecs_per_cb) {
    if (d != 4) return EVA_ERR_UNSUPPORTED;
    if (!v || !cent || M < 0 || ncent < 1 || ncent > kMaxCent || vecs_per_cb < 0) return EVA_ERR_INVALID_ARG;
    if (!aligned16c(v) || !aligned16c(cent)) return EVA_ERR_INVALID_ARG;
    const int64_t G = vecs_per_cb ? (M + vecs_per_cb - 1) / vecs_per_cb : 1;
    if (G > 65535) return EVA_ERR_INVALID_ARG;
    return EVA_OK;
}

int64_t codebooks_of(int64_t M, int64_t vecs_per_cb) {
    return vecs_per_cb ? std::max<int64_t>(1, (M + vecs_per_cb - 1) / vecs_per_cb) : 1;
}

template <typename IdxT>
cudaError_t launch_assign(const float *v, int64_t M, const float *cent, int ncent, int64_t vecs_per_cb,
                          IdxT *idx, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    const int64_t G = codebooks_of(M, vecs_per_cb);
    const int64_t per = vecs_per_cb ? vecs_per_cb : M;
    const int64_t bx = std::min<int64_t>(std::max<int64_t>(1, (per + 4 * kQThreads - 1) / (4 * kQThreads)), 2048);
    eva_kmeans_assign_kernel<IdxT><<<dim3((unsigned)bx, (unsigned)G), kQThreads, 0, s>>>(
        reinterpret_cast<const float4 *>(v), M, reinterpret_cast<const float4 *>(cent), ncent,
        vecs_per_cb ? vecs_per_cb : M, idx);
    return cudaGetLastError();
}

cudaError_t launch_update(const float *v, int64_t M, const int32_t *idx, int ncent, int64_t vecs_per_cb,
                          const float *old, float *out, int64_t *counts_out, double *sums,
                          unsigned long long *counts, cudaStream_t s) {
    const int64_t G = codebooks_of(M, vecs_per_cb);
    const int n = (int)(G * ncent);
    cudaError_t e = cudaMemsetAsync(sums, 0, (size_t)n * 4 * sizeof(double), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, (size_t)n * sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
    if (M > 0) {
        const int64_t per = vecs_per_cb ? vecs_per_cb : M;
        const int64_t bx = std::min<int64_t>(std::max<int64_t>(1, (per + kQThreads - 1) / kQThreads), 592);
        eva_kmeans_accum_kernel<<<dim3((unsigned)bx, (unsigned)G), kQThreads, 0, s>>>(
            reinterpret_cast<const float4 *>(v), M, idx, ncent, vecs_per_cb ? vecs_per_cb : M, sums, counts);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    eva_kmeans_finish_kernel<<<blocks_for(n, 256), 256, 0, s>>>(sums, counts, old, out,
                                                                 reinterpret_cast<long long *>(counts_out), n);
    return cudaGetLastError();
}

cudaError_t launch_residual(const float *wrot, int N, int K, const __half *wc, int ncent, const uint8_t *wi,
                            int codebook_rows, int group, uint8_t *signs, __half *alpha, cudaStream_t s) {
    const long long warps = (long long)N * (K / group);
    const long long threads = warps * 32;
    eva_residual_kernel<<<(unsigned)((threads + kQThreads - 1) / kQThreads), kQThreads, 0, s>>>(
        reinterpret_cast<const float4 *>(wrot), N, K, wc, ncent, wi, codebook_rows, group, signs, alpha);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

eva_status_t eva_vq_kmeans_assign(const float *v, int64_t M, int32_t d, const float *centroids, int32_t ncent,
                                  int64_t vecs_per_cb, int32_t *idx_out, eva_stream_t stream) {
    const eva_status_t st = kmeans_args(v, M, d, centroids, ncent, vecs_per_cb);
    if (st != EVA_OK) return st;
    if (!idx_out) return EVA_ERR_INVALID_ARG;
    return cuda_status(launch_assign(v, M, centroids, ncent, vecs_per_cb, idx_out,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

eva_status_t eva_vq_kmeans_update(const float *v, int64_t M, int32_t d, const int32_t *idx, int32_t ncent,
                                  int64_t vecs_per_cb, const float *old, float *new_out, int64_t *counts_out,
                                  eva_stream_t stream) {
    const eva_status_t st = kmeans_args(v, M, d, old, ncent, vecs_per_cb);
    if (st != EVA_OK) return st;
    if (!idx || !new_out) return EVA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t n = codebooks_of(M, vecs_per_cb) * ncent;
    double *sums = nullptr;
    cudaError_t e = cudaMallocAsync(reinterpret_cast<void **>(&sums),
                                    (size_t)n * (4 * sizeof(double) + sizeof(unsigned long long)), s);
    if (e != cudaSuccess) return e == cudaErrorMemoryAllocation ? EVA_ERR_OOM : cuda_status(e);
    e = launch_update(v, M, idx, ncent, vecs_per_cb, old, new_out, counts_out, sums,
                      reinterpret_cast<unsigned long long *>(sums + 4 * n), s);
    const cudaError_t ef = cudaFreeAsync(sums, s);
    return cuda_status(e != cudaSuccess ? e : ef);
}

eva_status_t eva_vq_residual(const float *wrot, int32_t N, int32_t K, const void *wc, int32_t ncent,
                             const uint8_t *wi, int32_t codebook_rows, int32_t group, uint8_t *signs_out,
                             void *alpha_out, eva_stream_t stream) {
    if (!wrot || !wc || !wi || !signs_out || !alpha_out || !aligned16c(wrot)) return EVA_ERR_INVALID_ARG;
    if (N < 1 || K < 8 || K % 8 || ncent < 1 || ncent > kMaxCent || group < 8 || group % 8 || K % group)
        return EVA_ERR_INVALID_ARG;
    if (codebook_rows < 0 || (codebook_rows && N % codebook_rows)) return EVA_ERR_INVALID_ARG;
    return cuda_status(launch_residual(wrot, N, K, reinterpret_cast<const __half *>(wc), ncent, wi, codebook_rows,
                                       group, signs_out, reinterpret_cast<__half *>(alpha_out),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

eva_status_t eva_vq_quantize(const eva_quant_desc *desc, const void *w, const int8_t *hsign,
                             const int32_t *init_index, void *wc_out, uint8_t *wi_out, uint8_t *signs_out,
                             void *alpha_out, float *wrot_out, float *cent_out, eva_stream_t stream) {
    if (!desc) return EVA_ERR_INVALID_ARG;
    const eva_quant_desc &d = *desc;
    if (d.d != 4) return EVA_ERR_UNSUPPORTED;
    if (d.index_bits < 1 || d.index_bits > 8) return EVA_ERR_UNSUPPORTED;
    if (d.N < 1 || d.K < 4 || d.K % 4 || d.iters < 0) return EVA_ERR_INVALID_ARG;
    if (d.index_bits == 4 && d.K % 8) return EVA_ERR_INVALID_ARG;   // whole packed bytes
    if (d.codebook_rows < 0 || (d.codebook_rows && d.N % d.codebook_rows)) return EVA_ERR_INVALID_ARG;
    if (d.residual_group && (d.residual_group < 8 || d.residual_group % 8 || d.K % d.residual_group))
        return EVA_ERR_INVALID_ARG;
    if (d.hadamard_block) {
        if (!valid_rotation_block(d.hadamard_block, d.K) || !hsign) return EVA_ERR_INVALID_ARG;
    } else if (hsign) {
        return EVA_ERR_INVALID_ARG;
    }
    if (!w || !init_index || !wc_out || !wi_out) return EVA_ERR_INVALID_ARG;
    if (d.residual_group ? (!signs_out || !alpha_out) : (signs_out || alpha_out)) return EVA_ERR_INVALID_ARG;
    if (wrot_out && !aligned16c(wrot_out)) return EVA_ERR_INVALID_ARG;
    if (cent_out && !aligned16c(cent_out)) return EVA_ERR_INVALID_ARG;
    const int ncent = 1 << d.index_bits;
    const int64_t N = d.N, K = d.K, J = K / 4, M = N * J;
    const int64_t vpc = d.codebook_rows ? (int64_t)d.codebook_rows * J : 0;
    const int64_t G = d.codebook_rows ? N / d.codebook_rows : 1;
    if (G > 65535) return EVA_ERR_INVALID_ARG;
    const int64_t nc = G * ncent;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    // Work buffers, one stream-ordered allocation:
    // [wrot][cent][cent16][sums][counts][idx][wi8][err] (wi8: the byte-per-pointer
    // indices when the output packs them two per byte).
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const bool packed = d.index_bits == 4;
    const size_t b_wrot = wrot_out ? 0 : up((size_t)M * 16), b_cent = up((size_t)nc * 16);
    const size_t b_sums = up((size_t)nc * 32), b_cnt = up((size_t)nc * 8), b_idx = up((size_t)M * 4);
    const size_t b_wi8 = packed ? up((size_t)M) : 0;
    const size_t total = b_wrot + 2 * b_cent + b_sums + b_cnt + b_idx + b_wi8 + 256;
    uint8_t *ws = nullptr;
    cudaError_t e = cudaMallocAsync(reinterpret_cast<void **>(&ws), total, s);
    if (e != cudaSuccess) return e == cudaErrorMemoryAllocation ? EVA_ERR_OOM : cuda_status(e);
    uint8_t *q = ws;
    float *wrot = wrot_out ? wrot_out : reinterpret_cast<float *>(q);
    q += b_wrot;
    float *cent = reinterpret_cast<float *>(q);
    q += b_cent;
    float *cent16 = reinterpret_cast<float *>(q);
    q += b_cent;
    double *sums = reinterpret_cast<double *>(q);
    q += b_sums;
    unsigned long long *counts = reinterpret_cast<unsigned long long *>(q);
    q += b_cnt;
    int32_t *idx = reinterpret_cast<int32_t *>(q);
    q += b_idx;
    uint8_t *wi8 = packed ? q : wi_out;
    q += b_wi8;
    int *err = reinterpret_cast<int *>(q);
    auto chk = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
    chk(cudaMemsetAsync(err, 0, sizeof(int), s));

    // 1. W_rot = W Q (rows rotated like x~), or W in fp32.
    int8_t *h28 = nullptr;
    if (paley_m(d.hadamard_block)) {
        int8_t tab[28 * 28];
        paley28_table(tab);
        chk(cudaMallocAsync(reinterpret_cast<void **>(&h28), sizeof(tab), s));
        if (e == cudaSuccess) chk(cudaMemcpyAsync(h28, tab, sizeof(tab), cudaMemcpyHostToDevice, s));
        if (e == cudaSuccess) chk(cudaStreamSynchronize(s));   // tab is on this stack frame
    }
    if (d.hadamard_block && e == cudaSuccess) {
        const int b = d.hadamard_block, thr = std::min(b / 2, 1024), m = paley_m(b);
        const float scale = (float)(1.0 / std::sqrt((double)b));
        if (m) chk(cudaFuncSetAttribute(eva_paley_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)std::min<size_t>((size_t)b * sizeof(float), 232448)));
        for (int64_t r0 = 0; r0 < N && e == cudaSuccess; r0 += 65535) {
            const int rows = (int)std::min<int64_t>(65535, N - r0);
            if (m)
                eva_paley_rows_kernel<<<dim3((unsigned)(K / b), (unsigned)rows), thr, (size_t)b * sizeof(float), s>>>(
                    reinterpret_cast<const __half *>(w) + r0 * K, hsign, h28, wrot + r0 * K, (int)K, b, m, scale);
            else
                eva_hadamard_kernel<<<dim3((unsigned)(K / b), (unsigned)rows), thr, (size_t)b * sizeof(float), s>>>(
                    reinterpret_cast<const __half *>(w) + r0 * K, hsign, wrot + r0 * K, (int)K, b, scale, 1);
            chk(cudaGetLastError());
        }
    } else if (!d.hadamard_block) {
        eva_rows_to_f32_kernel<<<(unsigned)std::min<int64_t>(blocks_for(N * K, 256), 4096), 256, 0, s>>>(
            reinterpret_cast<const __half *>(w), wrot, N * K);
        chk(cudaGetLastError());
    }
    // 2.-3. blocks of 4, starting centroids, Lloyd iterations.
    eva_gather_init_kernel<<<blocks_for(nc, 256), 256, 0, s>>>(
        reinterpret_cast<const float4 *>(wrot), M, init_index, ncent, vpc ? vpc : M, (int)G,
        reinterpret_cast<float4 *>(cent), err);
    chk(cudaGetLastError());
    for (int it = 0; it < d.iters && e == cudaSuccess; ++it) {
        chk(launch_assign(wrot, M, cent, ncent, vpc, idx, s));
        chk(launch_update(wrot, M, idx, ncent, vpc, cent, cent, nullptr, sums, counts, s));
    }
    if (cent_out) chk(cudaMemcpyAsync(cent_out, cent, (size_t)nc * 16, cudaMemcpyDeviceToDevice, s));
    // fp16 codebook; pointers = nearest fp16 centroids.
    eva_centroids_to_f16_kernel<<<blocks_for(nc * 4, 256), 256, 0, s>>>(cent, reinterpret_cast<__half *>(wc_out),
                                                                        cent16, (int)(nc * 4));
    chk(cudaGetLastError());
    chk(launch_assign(wrot, M, cent16, ncent, vpc, wi8, s));
    // 4.-7. residual signs and scales.
    if (d.residual_group)
        chk(launch_residual(wrot, (int)N, (int)K, reinterpret_cast<const __half *>(wc_out), ncent, wi8,
                            d.codebook_rows, d.residual_group, signs_out, reinterpret_cast<__half *>(alpha_out), s));
    if (packed) {   // two pointers per byte, the even sub-vector in the low nibble
        eva_pack_nibbles_kernel<<<blocks_for(M / 2, 256), 256, 0, s>>>(wi8, wi_out, M / 2);
        chk(cudaGetLastError());
    }
    int herr = 0;
    chk(cudaMemcpyAsync(&herr, err, sizeof(int), cudaMemcpyDeviceToHost, s));
    if (h28) cudaFreeAsync(h28, s);
    chk(cudaFreeAsync(ws, s));
    chk(cudaStreamSynchronize(s));
    if (e != cudaSuccess) return cuda_status(e);
    return herr ? EVA_ERR_INVALID_ARG : EVA_OK;
}

}  // extern "C"
