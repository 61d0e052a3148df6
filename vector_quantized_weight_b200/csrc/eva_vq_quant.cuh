// eva_vq_quant.cuh -- kernels of the offline quantizer (3-bit SRAM-lookup
// article, the quantize() sample): rotate the weight rows, Lloyd K-means over
// the d = 4 blocks, residual signs and per-group scales.
//
//  eva_rows_to_f32_kernel    W fp16 -> fp32 (layers without rotation); with a
//                            rotation the rows go through eva_hadamard_kernel
//                            (W_rot = W Q is the x~ transform applied row-wise)
//  eva_gather_init_kernel    starting centroids = chosen blocks of W_rot
//  eva_kmeans_assign_kernel  nearest centroid of every block, decided in fp32
//                            with the distance summed component by component
//                            (no contraction) and the first minimum winning
//  eva_kmeans_accum_kernel   per-centroid sums (double) and counts
//  eva_kmeans_finish_kernel  centroid = mean, an empty cluster keeps its value
//  eva_residual_kernel       r = W_rot - codebook[pointer] (fp32), sign bits
//                            LSB-first (zero counts as +1), alpha = mean |r|
//                            per group (double sum) rounded to fp16
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace eva {

constexpr int kQThreads = 256;
constexpr int kMaxCent = 256;

__global__ void eva_rows_to_f32_kernel(const __half *__restrict__ w, float *__restrict__ out, long long n) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        out[i] = __half2float(w[i]);
}

// Codebook g's centroid c starts as block init_index[g][c] of the codebook's
// own blocks [g * vecs_per_cb, min(M, (g + 1) * vecs_per_cb)).  An index
// outside that range is not read: it sets *err and the centroid starts at 0.
__global__ void eva_gather_init_kernel(const float4 *__restrict__ v, long long M,
                                       const int32_t *__restrict__ init_index, int ncent, long long vecs_per_cb,
                                       int G, float4 *__restrict__ cent, int *__restrict__ err) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= G * ncent) return;
    const int g = i / ncent;
    const long long lo = (long long)g * vecs_per_cb, n = min(M, lo + vecs_per_cb) - lo;
    const long long k = init_index[i];
    if (k < 0 || k >= n) {
        atomicOr(err, 1);
        cent[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        return;
    }
    cent[i] = v[lo + k];
}

// Squared distance of block a to centroid c, exactly as the oracle sums it:
// each difference, square and partial sum rounded to fp32, in component order.
__device__ __forceinline__ float dist4(const float4 a, const float4 c) {
    const float d0 = __fsub_rn(a.x, c.x), d1 = __fsub_rn(a.y, c.y);
    const float d2 = __fsub_rn(a.z, c.z), d3 = __fsub_rn(a.w, c.w);
    float s = __fmul_rn(d0, d0);
    s = __fadd_rn(s, __fmul_rn(d1, d1));
    s = __fadd_rn(s, __fmul_rn(d2, d2));
    return __fadd_rn(s, __fmul_rn(d3, d3));
}

// grid (blocks, G): the blocks of codebook g = blockIdx.y are
// [g * vecs_per_cb, min(M, (g + 1) * vecs_per_cb)).  Each thread takes four
// blocks at a time; every lane reads the same centroid (a broadcast).
template <typename IdxT>
__global__ void __launch_bounds__(kQThreads) eva_kmeans_assign_kernel(const float4 *__restrict__ v, long long M,
                                                                      const float4 *__restrict__ cent, int ncent,
                                                                      long long vecs_per_cb, IdxT *__restrict__ idx) {
    __shared__ float4 cs[kMaxCent];
    const int g = blockIdx.y;
    for (int c = threadIdx.x; c < ncent; c += blockDim.x) cs[c] = cent[(long long)g * ncent + c];
    __syncthreads();
    const long long lo = (long long)g * vecs_per_cb, hi = min(M, lo + vecs_per_cb);
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long m0 = lo + (long long)blockIdx.x * blockDim.x + threadIdx.x; m0 < hi; m0 += 4 * stride) {
        float4 a[4];
        int best[4];
        float bd[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const long long m = m0 + u * stride;
            a[u] = m < hi ? v[m] : make_float4(0.f, 0.f, 0.f, 0.f);
            best[u] = 0;
            bd[u] = dist4(a[u], cs[0]);
        }
        for (int c = 1; c < ncent; ++c) {
            const float4 cc = cs[c];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float dd = dist4(a[u], cc);
                if (dd < bd[u]) {
                    bd[u] = dd;
                    best[u] = c;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const long long m = m0 + u * stride;
            if (m < hi) idx[m] = (IdxT)best[u];
        }
    }
}

// Per-centroid sums in double and counts: shared-memory accumulation per
// block, then one global atomic per centroid and component.  sums [G][ncent][4],
// counts [G][ncent] must start at zero.
__global__ void __launch_bounds__(kQThreads) eva_kmeans_accum_kernel(const float4 *__restrict__ v, long long M,
                                                                     const int32_t *__restrict__ idx, int ncent,
                                                                     long long vecs_per_cb, double *__restrict__ sums,
                                                                     unsigned long long *__restrict__ counts) {
    __shared__ double ss[kMaxCent * 4];
    __shared__ unsigned int sc[kMaxCent];
    const int g = blockIdx.y;
    for (int i = threadIdx.x; i < ncent * 4; i += blockDim.x) ss[i] = 0.0;
    for (int i = threadIdx.x; i < ncent; i += blockDim.x) sc[i] = 0u;
    __syncthreads();
    const long long lo = (long long)g * vecs_per_cb, hi = min(M, lo + vecs_per_cb);
    for (long long m = lo + (long long)blockIdx.x * blockDim.x + threadIdx.x; m < hi;
         m += (long long)gridDim.x * blockDim.x) {
        const int c = idx[m];
        if (c < 0 || c >= ncent) continue;   // indices come from the assign kernel
        const float4 a = v[m];
        atomicAdd(&ss[4 * c + 0], (double)a.x);
        atomicAdd(&ss[4 * c + 1], (double)a.y);
        atomicAdd(&ss[4 * c + 2], (double)a.z);
        atomicAdd(&ss[4 * c + 3], (double)a.w);
        atomicAdd(&sc[c], 1u);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < ncent; c += blockDim.x) {
        if (!sc[c]) continue;
        const long long gc = (long long)g * ncent + c;
#pragma unroll
        for (int t = 0; t < 4; ++t) atomicAdd(&sums[4 * gc + t], ss[4 * c + t]);
        atomicAdd(&counts[gc], (unsigned long long)sc[c]);
    }
}

__global__ void eva_kmeans_finish_kernel(const double *__restrict__ sums, const unsigned long long *__restrict__ counts,
                                         const float *__restrict__ old_cent, float *__restrict__ new_cent,
                                         long long *__restrict__ counts_out, int n) {
    const int gc = blockIdx.x * blockDim.x + threadIdx.x;
    if (gc >= n) return;
    const unsigned long long k = counts[gc];
#pragma unroll
    for (int t = 0; t < 4; ++t)
        new_cent[4 * gc + t] = k ? (float)(sums[4 * gc + t] / (double)k) : old_cent[4 * gc + t];
    if (counts_out) counts_out[gc] = (long long)k;
}

// fp32 centroids -> the stored fp16 codebook, and its values back in fp32 for
// the final pointer assignment.
__global__ void eva_centroids_to_f16_kernel(const float *__restrict__ cent, __half *__restrict__ wc,
                                            float *__restrict__ cent16, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const __half h = __float2half_rn(cent[i]);
    wc[i] = h;
    cent16[i] = __half2float(h);
}

// One warp per (row o, group q of 128 inputs): lane L takes block
// 32 q + L (inputs 128 q + 4L .. +3).  Signs: a nibble per lane, two lanes per
// byte.  alpha: |r| summed in double across the warp, / 128, to fp16.
__global__ void __launch_bounds__(kQThreads) eva_residual_kernel(const float4 *__restrict__ wrot, int N, int K,
                                                                 const __half *__restrict__ wc, int ncent,
                                                                 const uint8_t *__restrict__ wi, int codebook_rows,
                                                                 int group, uint8_t *__restrict__ signs,
                                                                 __half *__restrict__ alpha) {
    const int lane = threadIdx.x & 31;
    const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int gpr = K / group;                       // groups per row
    if (wid >= (long long)N * gpr) return;
    const int o = (int)(wid / gpr), q = (int)(wid % gpr);
    const int J = K / 4, cb = codebook_rows ? o / codebook_rows : 0;
    const int bpg = group / 4;                       // blocks per group (32 for 128)
    double acc = 0.0;
    for (int jb = lane; jb < bpg; jb += 32) {
        const int j = q * bpg + jb;
        const float4 w = wrot[(long long)o * J + j];
        const int c = wi[(long long)o * J + j];
        const __half *e = wc + ((long long)cb * ncent + (c < ncent ? c : 0)) * 4;
        const float r0 = __fsub_rn(w.x, __half2float(e[0])), r1 = __fsub_rn(w.y, __half2float(e[1]));
        const float r2 = __fsub_rn(w.z, __half2float(e[2])), r3 = __fsub_rn(w.w, __half2float(e[3]));
        const unsigned nib = (r0 >= 0.f ? 1u : 0u) | (r1 >= 0.f ? 2u : 0u) | (r2 >= 0.f ? 4u : 0u) |
                             (r3 >= 0.f ? 8u : 0u);
        acc += fabs((double)r0) + fabs((double)r1) + fabs((double)r2) + fabs((double)r3);
        const unsigned hi = __shfl_down_sync(__activemask(), nib, 1);
        if (!(jb & 1)) signs[(long long)o * (K / 8) + j / 2] = (uint8_t)(nib | (hi << 4));
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) alpha[(long long)o * gpr + q] = __double2half(acc / (double)group);
}

// Pointers < 16, one per byte -> two per byte, sub-vector 2t in the low nibble
// of byte t (the 4-bit index layout of the layer).
__global__ void eva_pack_nibbles_kernel(const uint8_t *__restrict__ wi8, uint8_t *__restrict__ out, long long n) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n) return;
    out[t] = (uint8_t)((wi8[2 * t] & 15u) | ((wi8[2 * t + 1] & 15u) << 4));
}

}  // namespace eva
