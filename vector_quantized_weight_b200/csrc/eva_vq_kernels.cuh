// eva_vq_kernels.cuh -- sm_100a kernels of the VQ decode linear.
//
//  eva_lookup_kernel   fused output-codebook build + conflict-free lookup +
//                      accumulation (EVA summary section 2.A, both steps; the
//                      Epilogue Unit of section 2.B that overlaps lookups with
//                      the codebook product is played here by one CTA doing
//                      both on one slice), with the optional 1-bit sign
//                      residual of the 3-bit SRAM-lookup article.
//  eva_hadamard_kernel randomized block Hadamard rotation of x (3-bit article,
//                      quantize() sample: W_rot = W Q, so x~ = Q^T x).
//  eva_repack_*        create-time repack of WI / signs / alpha into the
//                      unit-major lane order the lookup kernel streams.
//
// Accumulation: the looked-up fp16 OC entries are summed by tensor-core MMAs
// against a constant 0/1 "routing" matrix (f16 inputs, fp32 accumulation).
// That is the adder tree: the MMA sums across the 16 k-columns supplied by
// the four lanes of a row, so no warp shuffles are needed and the shared-
// memory pipe carries only the lookups.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "eva_vq_layout.cuh"

namespace eva {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCtaTiles = 128;  // row tiles per CTA (shared-memory accumulator size)
constexpr int kLookahead = 3;      // units of index bytes in flight per warp
constexpr uint32_t kAccBytes = kMaxCtaTiles * kTileRows * 2 * 4;

extern __shared__ __align__(1024) uint8_t eva_smem[];

struct LookupParams {
    const uint8_t *wi;       // repacked index units, [S][T] x 1024 B
    const uint8_t *sg;       // repacked sign units, [S][T] x 512 B (residual only)
    const __half *al;        // repacked alpha units, [S][T] x 32 halves (residual only)
    const __half *wc;        // codebooks [G][256][4]
    const void *x;           // activations [B][K]: fp16, or fp32 when x_f32
    void *y;                 // output [B][N]
    int N, Npad, K, S, T, B;
    int Gs, Gt;              // CTA grid: blockIdx.x = tt * Gs + ts; clusters of Gs CTAs
    int tiles_per_cb;        // 0: shared codebook; else row tiles per codebook
    int x_f32, out_f32;
    int independent;         // neither x nor y is touched by the preceding kernel:
                             // run without waiting for it (wait only before exit)
    int acc_tiles;           // row tiles of the largest CTA (shared-memory layout)
    const uint8_t *sgd;      // dequantize path with residual: sign units in its own lane
                             // order, [S][T][512] bytes (alpha: the lookup's units, al)
    int wi_staged;           // leading row tiles whose first-slice indices are copied
                             // into shared memory by one bulk copy in the prologue
    int *status;             // device error word (bit 0: the wait for the staged index
                             // copy gave up; bit 1: the same wait at exit gave up)
    int wait_rounds;         // try_wait rounds before a bounded wait gives up (> 0)
    int skip_stage_copy;     // failure-detection test only: issue neither the staging
                             // copy nor its arrival, so the bounded wait runs out
    const int8_t *hs;        // randomized Hadamard signs s [K] (fused rotation only)
    int rot_b;               // 0, or the rotation block b: x~ = s . (H_b x) / sqrt(b) is
                             // computed in the lookup kernel from fp16 x
    float rot_scale;         // 1 / sqrt(b), rounded to fp32
    int ncent;               // centroids per codebook: 256, or 16 for 4-bit indices
    int rot_m;               // 0: Sylvester block; m: b = 28 m, H_b = H28 (x) H_m
    const int8_t *h28;       // the order-28 Paley matrix [28][28] (rot_m != 0)
#ifdef EVA_DEVICE_CHECKS
    // Debug build only: bounds of every buffer the kernel touches.  A
    // violating access is skipped and the first one is recorded.
    const void *chk_base[8];
    unsigned long long chk_bytes[8];
    unsigned smem_bytes;
    int *chk_record;         // [0] count, [1] line, [2] buffer, [3] block, [4] thread,
                             // [5] offset low, [6] offset high, [7] size
#endif
#ifdef EVA_TIMELINE
    unsigned long long *timeline;   // [grid][8] %globaltimer stamps of the last run
#endif
};

// Timeline build only: thread 0 of each CTA stamps phase boundaries.
#ifdef EVA_TIMELINE
__device__ __forceinline__ unsigned long long eva_globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
#define EVA_STAMP(ph) do { if (threadIdx.x == 0) p.timeline[eva_bid * 8 + (ph)] = eva_globaltimer(); } while (0)
#else
#define EVA_STAMP(ph) do { } while (0)
#endif

enum { BUF_WI = 0, BUF_SG, BUF_AL, BUF_WC, BUF_X, BUF_PARTIAL, BUF_COUNTERS, BUF_Y, BUF_SMEM };

#ifdef EVA_DEVICE_CHECKS
__device__ __noinline__ bool eva_check_fail(const LookupParams &p, int line, int buf, long long off,
                                            unsigned long long n) {
    if (atomicAdd(p.chk_record, 1) == 0) {
        p.chk_record[1] = line;
        p.chk_record[2] = buf;
        p.chk_record[3] = (int)blockIdx.x;
        p.chk_record[4] = (int)threadIdx.x;
        p.chk_record[5] = (int)(off & 0xffffffffll);
        p.chk_record[6] = (int)(off >> 32);
        p.chk_record[7] = (int)n;
    }
    return true;
}
// True when [ptr, ptr + n) is outside buffer `buf` or misaligned for an
// n-byte access (n up to 16).
__device__ __forceinline__ bool eva_bad_g(const LookupParams &p, int buf, const void *ptr,
                                          unsigned long long n, int line) {
    const char *b = static_cast<const char *>(p.chk_base[buf]);
    const char *q = static_cast<const char *>(ptr);
    const long long off = (long long)(q - b);
    const unsigned long long al = n >= 16 ? 16 : (n >= 8 ? 8 : (n >= 4 ? 4 : (n >= 2 ? 2 : 1)));
    if (b && off >= 0 && (unsigned long long)off + n <= p.chk_bytes[buf] &&
        (reinterpret_cast<uintptr_t>(q) % al) == 0)
        return false;
    return eva_check_fail(p, line, buf, off, n);
}
__device__ __forceinline__ bool eva_bad_s(const LookupParams &p, uint32_t off, int line) {
    if (off + 4u <= p.smem_bytes && (off & 3u) == 0) return false;
    return eva_check_fail(p, line, BUF_SMEM, off, 4);
}
#define EVA_BAD_G(buf, ptr, n) eva_bad_g(p, buf, ptr, n, __LINE__)
#define EVA_BAD_S(off) eva_bad_s(p, off, __LINE__)
#else
#define EVA_BAD_G(buf, ptr, n) false
#define EVA_BAD_S(off) false
#endif

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ uint32_t lds32(uint32_t off) {
    return *reinterpret_cast<const uint32_t *>(eva_smem + off);
}
__device__ __forceinline__ void sts32(uint32_t off, uint32_t v) {
    *reinterpret_cast<uint32_t *>(eva_smem + off) = v;
}

// Streamed read-only 16-byte load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

// The 32 index bytes of one lane in one unit (two 16-byte halves 512 bytes
// apart, see wi_unit_pos).  Volatile with a memory
// clobber so the compiler keeps it where it is written: the tile loop issues
// exactly one unit of lookahead instead of hoisting every tile's load.
__device__ __forceinline__ void ldg_unit(const void *p, uint4 &a, uint4 &b) {
    asm volatile(
        "ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%8];\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%4,%5,%6,%7}, [%8+512];"
        : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
        : "l"(p)
        : "memory");
}

__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Programmatic dependent launch: wait for the preceding kernel's writes /
// allow the next kernel to start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Thread-block-cluster barrier (release/acquire): every CTA of the cluster
// has arrived and its shared-memory writes are visible cluster-wide.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---- one-shot mbarrier + bulk copy (global -> own shared memory, no multicast)
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Bounded wait for phase `parity` of the barrier: gives up (returns false)
// after `rounds` tries (each try suspends for a short, hardware-chosen time).
constexpr int kWaitRounds = 1 << 20;
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int rounds) {
    for (int it = 0; it < rounds; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t off) {
    return *reinterpret_cast<const uint4 *>(eva_smem + off);
}

// 16-byte store into the shared memory of cluster CTA `rank`, at the address
// this CTA uses for the same variable (distributed shared memory).
__device__ __forceinline__ void st_dsmem_v4(uint32_t local_addr, uint32_t rank, float4 v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_addr), "r"(rank));
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(ra), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

// The address of this CTA's shared-memory location `local_addr` in cluster
// CTA `rank`, and an 8-byte store there.
__device__ __forceinline__ uint32_t dsmem_map(uint32_t local_addr, uint32_t rank) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_addr), "r"(rank));
    return ra;
}
__device__ __forceinline__ void st_dsmem_v2(uint32_t remote_addr, float x, float y) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(remote_addr), "f"(x), "f"(y) : "memory");
}

__device__ __forceinline__ uint32_t to_tf32(float f) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(f));
    return r;
}

// D = A(16x4, tf32) * B(4x8, tf32), fp32 accumulate from zero.
__device__ __forceinline__ void mma_tf32_k4(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm("mma.sync.aligned.m16n8k4.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
        "{%7,%7,%7,%7};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0), "f"(0.f));
}

// D += A(16x16, f16) * B(16x8, f16), fp32 accumulate.
__device__ __forceinline__ void mma_f16_k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t half2_bits(float lo, float hi) { return pack_half2(lo, hi); }

__device__ __forceinline__ void swap_if(bool c, uint32_t &a, uint32_t &b) {
    uint32_t ta = c ? b : a, tb = c ? a : b;
    a = ta;
    b = tb;
}

// After the call v[r] holds the input v[r ^ q] (q in 0..3): lane q stores its
// bank class r ^ q in round r, so the 32 lanes of a store hit 32 banks.
__device__ __forceinline__ void xor_permute(uint32_t (&v)[4], int q) {
    swap_if(q & 1, v[0], v[1]);
    swap_if(q & 1, v[2], v[3]);
    swap_if(q & 2, v[0], v[2]);
    swap_if(q & 2, v[1], v[3]);
}

// x~[tok][k], zero outside [0, B) x [0, K).  Read through L2 (x may have
// been written by the kernel this one waited for).
__device__ __forceinline__ float load_x(const LookupParams &p, int tok, int k) {
    if (tok >= p.B || k >= p.K) return 0.f;
    size_t i = (size_t)tok * p.K + k;
    if (p.x_f32) {
        const float *xp = reinterpret_cast<const float *>(p.x) + i;
        return EVA_BAD_G(BUF_X, xp, 4) ? 0.f : __ldcg(xp);
    }
    const unsigned short *xp = reinterpret_cast<const unsigned short *>(p.x) + i;
    if (EVA_BAD_G(BUF_X, xp, 2)) return 0.f;
    unsigned short b = __ldcg(xp);
    return __half2float(__ushort_as_half(b));
}

// ------------------------------------------------------------- x staging
//
// The x~ values of one K-slice (256 inputs per token, as fp32) are staged once
// per CTA in shared memory: one warp per token, 8 consecutive inputs per lane
// with 128-bit loads when aligned; zeros past K or past B.
constexpr uint32_t kXStageBytes = 2u * kSliceK * 4u;   // room for a token pair

// Layout of a one-token image without residual table: only columns 0..31 of
// its 256-byte rows are lookups; the other 128 bytes of each row ("gaps")
// hold the running sums (row tl: tile tl, tl < kMaxGapTiles), the staging
// mbarrier (row 247) and the x~ slice (rows 248..255, 32 floats each).
// x_off == kXGaps selects that x~ layout.
constexpr uint32_t kXGaps = 0xFFFF0000u;
constexpr int kMaxGapTiles = 247;   // row tiles per CTA in this layout
__host__ __device__ constexpr uint32_t gap_off(int row) { return (uint32_t)row * kOcRowBytes + 128u; }
__device__ __forceinline__ uint32_t x_addr(uint32_t x_off, int idx) {
    return x_off == kXGaps ? gap_off(248 + (idx >> 5)) + 4u * (uint32_t)(idx & 31) : x_off + 4u * (uint32_t)idx;
}

template <bool PAIR_T>
__device__ __forceinline__ void stage_x(const LookupParams &p, int s, int pr, int warp, int lane,
                                        uint32_t x_off) {
    constexpr int NTOK = PAIR_T ? 2 : 1;
    if (warp >= NTOK) return;
    const int tok = PAIR_T ? 2 * pr + warp : 0;
    const int k0 = s * kSliceK + 8 * lane;
    float v[8];
    const size_t i = (size_t)tok * p.K + k0;
    bool done = false;
    if (tok < p.B && k0 + 8 <= p.K) {
        if (p.x_f32 && (i & 3) == 0) {
            const float4 *xp = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p.x) + i);
            if (!EVA_BAD_G(BUF_X, xp, 32)) {
                const float4 a = __ldcg(xp), b = __ldcg(xp + 1);
                v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
                v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
                done = true;
            }
        } else if (!p.x_f32 && (i & 7) == 0) {
            const uint4 *xp = reinterpret_cast<const uint4 *>(reinterpret_cast<const __half *>(p.x) + i);
            if (!EVA_BAD_G(BUF_X, xp, 16)) {
                const uint4 r = __ldcg(xp);
                const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __half2 h2 = *reinterpret_cast<const __half2 *>(&w[j]);
                    v[2 * j] = __low2float(h2);
                    v[2 * j + 1] = __high2float(h2);
                }
                done = true;
            }
        }
    }
    if (!done) {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = load_x(p, tok, k0 + j);
    }
    const uint32_t off = x_addr(x_off, warp * kSliceK + 8 * lane);   // 8 floats, inside one gap
    if (!EVA_BAD_S(off) && !EVA_BAD_S(off + 28u)) {
        *reinterpret_cast<float4 *>(eva_smem + off) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4 *>(eva_smem + off + 16) = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// ------------------------------------------------- fused Hadamard rotation
//
// The randomized block rotation of the 3-bit article (x~ = Q^T x with
// Q = blockdiag(H_b) diag(s) / sqrt(b)) computed while staging x: each CTA
// transforms the whole b-block its slice falls in and keeps its 256 outputs.
// The butterflies are those of the in-order fast Walsh-Hadamard transform
// (stage h pairs positions lo and lo + h, lo with bit h clear, into
// (a + c, a - c)), stage by stage, so every value is bitwise that of the
// standalone rotation kernel below.

// Eight consecutive fp16 inputs of token `tok` from k0 on, as fp32; zeros past
// K or past B.
__device__ __forceinline__ void load_x8_f16(const LookupParams &p, int tok, int k0, float (&v)[8]) {
    const size_t i = (size_t)tok * p.K + k0;
    if (tok < p.B && k0 + 8 <= p.K && (i & 7) == 0) {
        const uint4 *xp = reinterpret_cast<const uint4 *>(reinterpret_cast<const __half *>(p.x) + i);
        if (!EVA_BAD_G(BUF_X, xp, 16)) {
            const uint4 r = __ldcg(xp);
            const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __half2 h2 = *reinterpret_cast<const __half2 *>(&w[j]);
                v[2 * j] = __low2float(h2);
                v[2 * j + 1] = __high2float(h2);
            }
            return;
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = load_x(p, tok, k0 + j);
}

// Stages h = 1 .. min(b, 256) / 2 over 256 consecutive inputs held by one
// warp, eight per lane (lane L holds 8L .. 8L + 7).
__device__ __forceinline__ void fwht_warp256(float (&v)[8], int lane, int b) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
        if (h >= b) break;
#pragma unroll
        for (int lo = 0; lo < 8; ++lo)
            if (!(lo & h)) {
                const float a = v[lo], c = v[lo + h];
                v[lo] = a + c;
                v[lo + h] = a - c;
            }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {      // h = 8 m: partner lane L ^ m
        if (8 * m >= b) break;
        const bool hi = (lane & m) != 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, v[j], m);
            v[j] = hi ? o - v[j] : v[j] + o;
        }
    }
}

// Scratch of the fused rotation, in bytes: the transformed 256-input chunks of
// one block for every token (Sylvester b > 256, Paley m <= 128), or eight
// warps' partial sums of up to four slices (Paley m >= 256, one token at a
// time).
__host__ __device__ __forceinline__ uint32_t rot_scratch_bytes(int b, int m, int ntok) {
    if (m >= 256) return 8u * 4u * kSliceK * 4u;
    return (m > 0 || b > kSliceK) ? (uint32_t)ntok * (uint32_t)b * 4u : 0u;
}

// Paley blocks with m >= 256 (b >= 7168: a block holds 28 or more slices):
// the rotated input x~ = s . (H_b^T x) / sqrt(b), H_b = H28 (x) H_m, of every
// slice s0 .. s1-1 of this CTA, for the pair's tokens, into xt
// [slice][token][256] (fp32).  With k = a m + c inside a block,
// (H_b^T x)[a m + c] = sum_a' H28[a'][a] (H_m x_a')[c]; per group of up to
// four slices of one block and per token, each warp transforms 256-input
// chunks (a', c') once and adds them, with sign H28[a'][a] sylvester(c', c),
// into partial sums of every slice of the group; the partials are added in
// warp order.
template <bool PAIR_T>
__device__ __forceinline__ void stage_x_rot_all(const LookupParams &p, int s0, int s1, int pr, int warp, int lane,
                                                int tid, uint32_t xt_off, uint32_t scr_off) {
    constexpr int NTOK = PAIR_T ? 2 : 1;
    const int b = p.rot_b, m = p.rot_m, nsl = s1 - s0;
    auto finish = [&](int sl, int tk, int i, float acc) {
        const int k = (s0 + sl) * kSliceK + i;
        const uint32_t off = xt_off + (uint32_t)((sl * NTOK + tk) * kSliceK + i) * 4u;
        if (!EVA_BAD_S(off)) *reinterpret_cast<float *>(eva_smem + off) = (k < p.K ? (float)p.hs[k] : 0.f) * acc * p.rot_scale;
    };
    auto tok_of = [&](int tk) { return PAIR_T ? 2 * pr + tk : 0; };
    {
        const int cpm = m / kSliceK, nch = 28 * cpm;
        for (int g0 = 0; g0 < nsl;) {
            // up to four consecutive slices inside one block
            const int blk = (s0 + g0) * kSliceK / b;
            int gn = 1;
            while (gn < 4 && g0 + gn < nsl && (s0 + g0 + gn) * kSliceK / b == blk) ++gn;
            const int blk0 = blk * b;
            for (int tk = 0; tk < NTOK; ++tk) {
                float acc[4][8];
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
                for (int ch = warp; ch < nch; ch += kWarps) {
                    const int a2 = ch / cpm, c2 = ch - a2 * cpm;
                    float v[8];
                    load_x8_f16(p, tok_of(tk), blk0 + ch * kSliceK + 8 * lane, v);
                    fwht_warp256(v, lane, kSliceK);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        if (j >= gn) break;
                        const int kb = (s0 + g0 + j) * kSliceK - blk0;
                        const int a = kb / m, c = (kb - a * m) / kSliceK;
                        const bool neg = (__ldg(p.h28 + a2 * 28 + a) < 0) != ((__popc((unsigned)(c2 & c)) & 1) != 0);
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[j][e] = neg ? acc[j][e] - v[e] : acc[j][e] + v[e];
                    }
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (j >= gn) break;
                    const uint32_t off = scr_off + (uint32_t)((warp * 4 + j) * kSliceK + 8 * lane) * 4u;
                    if (!EVA_BAD_S(off) && !EVA_BAD_S(off + 28u)) {
                        *reinterpret_cast<float4 *>(eva_smem + off) = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
                        *reinterpret_cast<float4 *>(eva_smem + off + 16) = make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]);
                    }
                }
                __syncthreads();
                for (int e = tid; e < gn * kSliceK; e += kThreads) {
                    const int j = e / kSliceK, i = e - j * kSliceK;
                    float sum = 0.f;
                    for (int w = 0; w < kWarps; ++w) {
                        const uint32_t off = scr_off + (uint32_t)((w * 4 + j) * kSliceK + i) * 4u;
                        sum += EVA_BAD_S(off) ? 0.f : *reinterpret_cast<const float *>(eva_smem + off);
                    }
                    finish(g0 + j, tk, i, sum);
                }
                __syncthreads();
            }
            g0 += gn;
        }
        return;
    }
}

// Per-slice form of the rotation (one slice's outputs at a time): the
// blocks' transforms are redone for every slice, which costs nothing extra
// when a CTA has one slice or the blocks are small.
// Rotation scratch in bytes per token: the b / 256 transformed sub-blocks of a
// Sylvester block b > 256 or a Paley block with m <= 128; eight warps'
// partial sums for a Paley block with m >= 256.
__host__ __device__ __forceinline__ uint32_t rot_scratch_per_token_slice(int b, int m) {
    if (m >= 256) return 8u * kSliceK * 4u;
    return (m > 0 || b > kSliceK) ? (uint32_t)b * 4u : 0u;
}

// Paley blocks b = 28 m (m a power of two >= 64, so every slice lies in one
// block): x~ = s . (H_b^T x) / sqrt(b), H_b = H28 (x) H_m.  With k = a m + c
// inside the block, (H_b^T x)[a m + c] = sum_a' H28[a'][a] (H_m x_a')[c].
//  m <= 128: the H_m transforms of all 28 sub-blocks (warp FWHT stages below
//    m over 256-input chunks) go to shared memory, then each output sums its
//    28 terms in order a' = 0..27 -- the same operations, in the same order,
//    as the standalone row kernel, so the values are bitwise equal;
//  (m >= 256 takes stage_x_rot_all, which serves all of a CTA's slices.)
template <bool PAIR_T>
__device__ __forceinline__ void stage_x_paley(const LookupParams &p, int s, int pr, int warp, int lane, int tid,
                                              uint32_t x_off, uint32_t rot_off) {
    constexpr int NTOK = PAIR_T ? 2 : 1;
    const int b = p.rot_b, m = p.rot_m, ks = s * kSliceK;
    const int blk0 = (ks / b) * b, kb = ks - blk0;       // block start, slice offset in the block
    const uint32_t per_tok = rot_scratch_per_token_slice(b, m);
    {
        const int nch = b / kSliceK;
        for (int w = warp; w < NTOK * nch; w += kWarps) {
            const int tk = w / nch, ch = w - tk * nch;
            float v[8];
            load_x8_f16(p, PAIR_T ? 2 * pr + tk : 0, blk0 + ch * kSliceK + 8 * lane, v);
            fwht_warp256(v, lane, m);
            const uint32_t off = rot_off + (uint32_t)tk * per_tok + (uint32_t)(ch * kSliceK + 8 * lane) * 4u;
            if (!EVA_BAD_S(off) && !EVA_BAD_S(off + 28u)) {
                *reinterpret_cast<float4 *>(eva_smem + off) = make_float4(v[0], v[1], v[2], v[3]);
                *reinterpret_cast<float4 *>(eva_smem + off + 16) = make_float4(v[4], v[5], v[6], v[7]);
            }
        }
        __syncthreads();
        for (int e = tid; e < NTOK * kSliceK; e += kThreads) {
            const int tk = e / kSliceK, i = e - tk * kSliceK;
            const int a = (kb + i) / m, c = (kb + i) - a * m;
            float acc = 0.f;
            for (int a2 = 0; a2 < 28; ++a2) {
                const uint32_t off = rot_off + (uint32_t)tk * per_tok + (uint32_t)(a2 * m + c) * 4u;
                const float y = EVA_BAD_S(off) ? 0.f : *reinterpret_cast<const float *>(eva_smem + off);
                acc = __ldg(p.h28 + a2 * 28 + a) > 0 ? acc + y : acc - y;
            }
            const uint32_t off = x_off + (uint32_t)(tk * kSliceK + i) * 4u;
            if (!EVA_BAD_S(off)) *reinterpret_cast<float *>(eva_smem + off) = (float)p.hs[ks + i] * acc * p.rot_scale;
        }
        return;
    }
}

template <bool PAIR_T>
__device__ __forceinline__ void stage_x_rot(const LookupParams &p, int s, int pr, int warp, int lane, int tid,
                                            uint32_t x_off, uint32_t rot_off) {
    constexpr int NTOK = PAIR_T ? 2 : 1;
    if (p.rot_m) {
        stage_x_paley<PAIR_T>(p, s, pr, warp, lane, tid, x_off, rot_off);
        return;
    }
    const int b = p.rot_b, ks = s * kSliceK;
    if (b <= kSliceK) {
        // Whole blocks inside the slice: one warp per token.
        if (warp >= NTOK) return;
        const int tok = PAIR_T ? 2 * pr + warp : 0;
        float v[8];
        load_x8_f16(p, tok, ks + 8 * lane, v);
        fwht_warp256(v, lane, b);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int k = ks + 8 * lane + j;
            v[j] = (k < p.K ? (float)p.hs[k] : 0.f) * v[j] * p.rot_scale;
        }
        const uint32_t off = x_off + (uint32_t)(warp * kSliceK + 8 * lane) * 4u;
        if (!EVA_BAD_S(off) && !EVA_BAD_S(off + 28u)) {
            *reinterpret_cast<float4 *>(eva_smem + off) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4 *>(eva_smem + off + 16) = make_float4(v[4], v[5], v[6], v[7]);
        }
        return;
    }
    // b > 256 (K is a multiple of b): the slice is sub-block `a` of its block.
    // Stages h < 256 run per sub-block in one warp each; h >= 256 combine the
    // nsb = b / 256 sub-blocks through shared memory.
    const int nsb = b / kSliceK, blk0 = (ks / b) * b, a = (ks - blk0) / kSliceK;
    for (int w = warp; w < NTOK * nsb; w += kWarps) {
        const int tk = w / nsb, sb = w - tk * nsb;
        float v[8];
        load_x8_f16(p, PAIR_T ? 2 * pr + tk : 0, blk0 + sb * kSliceK + 8 * lane, v);
        fwht_warp256(v, lane, kSliceK);
        const uint32_t off = rot_off + (uint32_t)(w * kSliceK + 8 * lane) * 4u;
        if (!EVA_BAD_S(off) && !EVA_BAD_S(off + 28u)) {
            *reinterpret_cast<float4 *>(eva_smem + off) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4 *>(eva_smem + off + 16) = make_float4(v[4], v[5], v[6], v[7]);
        }
    }
    __syncthreads();
    for (int e = tid; e < NTOK * kSliceK; e += kThreads) {
        const int tk = e / kSliceK, i = e - tk * kSliceK;
        float u[16];
#pragma unroll
        for (int sb = 0; sb < 16; ++sb) {
            const uint32_t off = rot_off + (uint32_t)((tk * nsb + sb) * kSliceK + i) * 4u;
            u[sb] = (sb < nsb && !EVA_BAD_S(off)) ? *reinterpret_cast<const float *>(eva_smem + off) : 0.f;
        }
#pragma unroll
        for (int m = 1; m < 16; m <<= 1) {  // h = 256 m
            if (m >= nsb) break;
#pragma unroll
            for (int lo = 0; lo < 16; ++lo)
                if (!(lo & m)) {
                    const float x0 = u[lo], x1 = u[lo + m];
                    u[lo] = x0 + x1;
                    u[lo + m] = x0 - x1;
                }
        }
        float r = u[0];
#pragma unroll
        for (int sb = 1; sb < 16; ++sb)
            if (sb == a) r = u[sb];
        const int k = ks + i;
        const uint32_t off = x_off + (uint32_t)(tk * kSliceK + i) * 4u;
        if (!EVA_BAD_S(off)) *reinterpret_cast<float *>(eva_smem + off) = (float)p.hs[k] * r * p.rot_scale;
    }
}

__device__ __forceinline__ float lds_x(const LookupParams &p, uint32_t x_off, int idx) {
    const uint32_t off = x_addr(x_off, idx);
    return EVA_BAD_S(off) ? 0.f : *reinterpret_cast<const float *>(eva_smem + off);
}

// B fragments of the codebook product for this warp's centroid tiles
// nt = warp + kWarps j: lane (g, q) holds WC[cb][8 nt + g][q] as tf32.  The
// raw fp16 bits are loaded first (load_codebook_raw) and converted when
// used (frag_from_raw), so a later pass's codebook can be in flight while
// the current one is used.
__device__ __forceinline__ void load_codebook_raw(const LookupParams &p, int cb, int warp, int g, int q,
                                                  uint32_t (&raw)[4]) {
    const __half *wcb = p.wc + (size_t)cb * p.ncent * kD;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int c = 8 * (warp + kWarps * j) + g;
        const __half *wp = wcb + c * kD + q;
        raw[j] = (c >= p.ncent || EVA_BAD_G(BUF_WC, wp, 2))
                     ? 0u
                     : (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(wp));
    }
}
__device__ __forceinline__ void frag_from_raw(const uint32_t (&raw)[4], uint32_t (&bf)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) bf[j] = to_tf32(__half2float(__ushort_as_half((unsigned short)raw[j])));
}
__device__ __forceinline__ void load_codebook_frag(const LookupParams &p, int cb, int warp, int g, int q,
                                                   uint32_t (&bf)[4]) {
    uint32_t raw[4];
    load_codebook_raw(p, cb, warp, g, q, raw);
    frag_from_raw(raw, bf);
}

// --------------------------------------------------- output-codebook build
//
// OC[j][c] = sum_{u<4} x~[256 s + 4 j + u] * WC[cb][c][u] for the 64 sub-vectors
// of slice s: a 64 x 4 by 4 x 256 product on tensor cores (m16n8k4, tf32),
// rounded to fp16 and stored in the conflict-free image.  fp16 operands are
// exact in tf32 and their products exact in fp32; the rotated input x~ of a
// 3.125-bit layer is fp32 and is rounded to tf32 (11 significant bits, the
// precision of the fp16 image entries themselves) before the product.  Warp
// w builds the centroid columns 8 nt .. 8 nt + 7 of nt = w + kWarps j, j = 0..3.
// Diagnostics build only (EVA_NAIVE_OC_LAYOUT): the one-token image of a
// layer without residual is stored the naive way, word(c, w) at row w,
// column c, so that a warp's 32 lookups land on banks chosen by the indices
// (bank = c mod 32).  It exists to measure the bank conflicts the
// column-per-sub-vector layout removes; results are the same.
#ifdef EVA_NAIVE_OC_LAYOUT
constexpr bool kNaiveOcBuild = true;
#else
constexpr bool kNaiveOcBuild = false;
#endif

template <bool PAIR_T, bool NAIVE = false>
__device__ __forceinline__ void build_oc(const LookupParams &p, int warp, int g, int q,
                                         const uint32_t (&bf)[4], uint32_t x_off) {
    constexpr int NTOK = PAIR_T ? 2 : 1;
    uint32_t ax[NTOK][4][2];
#pragma unroll
    for (int tk = 0; tk < NTOK; ++tk)
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            const int idx = tk * kSliceK + kD * (16 * mt + g) + q;
            ax[tk][mt][0] = to_tf32(lds_x(p, x_off, idx));
            ax[tk][mt][1] = to_tf32(lds_x(p, x_off, idx + 8 * kD));
        }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int nt = warp + kWarps * j;
        if (8 * nt >= p.ncent) continue;   // 16-centroid codebooks: two column tiles
        const uint32_t b0 = bf[j];
        if (!PAIR_T) {
            // D[mt][2h + cc] = OC[16 mt + g + 8 h][8 nt + 2 q + cc]; the word of
            // class i pairs sub-vector g + 8 i (m-tile i/2) with +32 (m-tile i/2 + 2).
            float D[4][4];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) mma_tf32_k4(D[mt], ax[0][mt][0], ax[0][mt][1], b0);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const uint32_t row = (uint32_t)(8 * nt + 2 * q + cc) * kOcRowBytes;
                uint32_t W[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    W[i] = pack_half2(D[i >> 1][2 * (i & 1) + cc], D[(i >> 1) + 2][2 * (i & 1) + cc]);
                xor_permute(W, q);
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const uint32_t off = NAIVE ? 1024u * (uint32_t)(g + 8 * (r ^ q)) + 4u * (8 * nt + 2 * q + cc)
                                               : row + 4u * (g + 8 * (r ^ q));
                    if (!EVA_BAD_S(off)) sts32(off, W[r]);
                }
            }
        } else {
            // Token pair: sub-vectors 0..31 (m-tiles 0,1) then 32..63 (m-tiles 2,3).
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                float D[2][2][4];
#pragma unroll
                for (int tk = 0; tk < 2; ++tk)
#pragma unroll
                    for (int m = 0; m < 2; ++m)
                        mma_tf32_k4(D[tk][m], ax[tk][2 * hi + m][0], ax[tk][2 * hi + m][1], b0);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t row = (uint32_t)(8 * nt + 2 * q + cc) * kOcRowBytes;
                    uint32_t W[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int e = 2 * (i & 1) + cc;
                        W[i] = pack_half2(D[0][i >> 1][e], D[NTOK - 1][i >> 1][e]);
                    }
                    xor_permute(W, q);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const uint32_t off = row + 4u * (g + 8 * (r ^ q) + 32 * hi);
                        if (!EVA_BAD_S(off)) sts32(off, W[r]);
                    }
                }
            }
        }
    }
}

// ------------------------------------------------------ sign-residual table
//
// The residual of a sign byte v at position m of the slice is
// T[v][m] = sum_{i<8} sigma_i(v) x~[256 s + 8 m + i], sigma_i(v) = +1 if bit i
// of v is set, else -1 -- the LUT of "input block x codebook" dot products of
// the 3-bit SRAM-lookup article with the 256 sign patterns as codebook.
// Warp w writes the rows v whose high nibble is w, w + kWarps, ...; lane =
// position m, so every store hits its own bank.  T = P_lo[v & 15] +
// P_hi[v >> 4] with 4-input partial sums.
template <bool PAIR_T>
__device__ __forceinline__ void build_sign_table(const LookupParams &p, int warp, int lane,
                                                 uint32_t t_off, uint32_t x_off) {
    constexpr int NTOK = PAIR_T ? 2 : 1;
    float xv[NTOK][8];
#pragma unroll
    for (int tk = 0; tk < NTOK; ++tk)
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[tk][i] = lds_x(p, x_off, tk * kSliceK + 8 * lane + i);
#pragma unroll 1
    for (int hn = warp; hn < 16; hn += kWarps) {
        float phi[NTOK];
#pragma unroll
        for (int tk = 0; tk < NTOK; ++tk) {
            phi[tk] = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) phi[tk] += ((hn >> i) & 1) ? xv[tk][4 + i] : -xv[tk][4 + i];
        }
#pragma unroll
        for (int a = 0; a < 16; ++a) {
            float tv[NTOK];
#pragma unroll
            for (int tk = 0; tk < NTOK; ++tk) {
                float plo = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) plo += ((a >> i) & 1) ? xv[tk][i] : -xv[tk][i];
                tv[tk] = plo + phi[tk];
            }
            const uint32_t w = PAIR_T ? pack_half2(tv[0], tv[NTOK - 1]) : pack_half2(tv[0], 0.f);
            const uint32_t off = t_off + (uint32_t)(16 * hn + a) * kOcRowBytes + 4u * lane;
            if (!EVA_BAD_S(off)) sts32(off, w);
        }
    }
}

// One unit's bytes for this lane: 8-bit indices, 16 bytes at p and 16 at
// p + 512; 4-bit indices, the 16 bytes at p (b stays zero).
template <bool NIB>
__device__ __forceinline__ void load_unit(const LookupParams &p, const uint8_t *up, uint4 &a, uint4 &b) {
    if constexpr (NIB) {
        if (!EVA_BAD_G(BUF_WI, up, 16)) a = ldg_stream(up);
    } else {
        if (!EVA_BAD_G(BUF_WI, up, 16) && !EVA_BAD_G(BUF_WI, up + 512, 16)) ldg_unit(up, a, b);
    }
}

// The residual operands of one unit: its sign bytes (16 per lane) and, in
// lanes q = 0, the alpha halves of rows g and g + 8.
__device__ __forceinline__ void load_resid(const LookupParams &p, size_t unit, int lane, int g, int q, uint4 &sv,
                                           uint2 &av) {
    const uint8_t *sp = p.sg + unit * kSignUnitBytes + lane * 16;
    sv = EVA_BAD_G(BUF_SG, sp, 16) ? make_uint4(0u, 0u, 0u, 0u) : ldg_stream(sp);
    av = make_uint2(0u, 0u);
    if (q == 0) {
        const __half *ap = p.al + unit * kAlphaUnitHalves + 4 * g;
        if (!EVA_BAD_G(BUF_AL, ap, 8)) av = *reinterpret_cast<const uint2 *>(ap);
    }
}

// ------------------------------------------------------------ lookup kernel
//
// Grid: Gs x Gt CTAs in clusters of Gs; CTA (ts, tt) owns K-slices [s0, s1)
// and row tiles [t0, t1); warp w owns the tiles t0 + w + kWarps i.  Per slice (and per
// codebook spanned): stage x~, build the OC image, then every warp streams
// its units: unpack an index byte into a shared-memory address with one byte
// permute, read the OC word, and feed four words per k-step into an MMA that
// sums them (the adder tree).  The Gs partial sums of a row group are combined
// inside its cluster through distributed shared memory.
//
// Before the dependency wait the kernel only touches weights: the bulk L2
// prefetch of its index range and the codebook fragments.  For one token the
// launch bounds of two CTAs per SM (128 registers; no instance spills) leave
// room for the next layer's CTA to run that prologue while this one computes,
// so the weight stream of layer l+1 overlaps the lookups of layer l; the
// token-pair variants need more registers and run one CTA per SM.

// Instances whose image rows lend their unused halves to x~, the mbarrier and
// the running sums (one token, no residual table, no rotation; not the naive
// diagnostics layout).  Their smaller footprint lets three CTAs share an SM
// (eva_lookup_kernel3, compiled for that register budget).
template <bool PAIR_T, bool RESID, bool ROT>
constexpr bool kImageGaps = !PAIR_T && !RESID && !ROT && !kNaiveOcBuild;
template <bool PAIR_T>
constexpr int kLookupMinBlocks = PAIR_T ? 1 : 2;

// The whole per-CTA program; eva_bid is the CTA's index within its layer.
template <bool PAIR_T, bool RESID, bool GROUPED, bool ROT, bool NIB>
__device__ __forceinline__ void lookup_body(const LookupParams &p, const int eva_bid) {
    // NIB: 4-bit indices (16 centroids), units of 512 bytes (16 per lane).
    constexpr uint32_t UB = NIB ? (uint32_t)kUnitBytes4 : (uint32_t)kUnitBytes;
    // Index units in flight per warp: with per-group codebooks a warp has at
    // most one tile per codebook pass, so a short ring suffices.
    constexpr int LA = GROUPED ? 2 : kLookahead;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int ts = eva_bid % p.Gs, tt = eva_bid / p.Gs;
    const int s0 = (int)((long long)p.S * ts / p.Gs), s1 = (int)((long long)p.S * (ts + 1) / p.Gs);
    const int t0 = (int)((long long)p.T * tt / p.Gt), t1 = (int)((long long)p.T * (tt + 1) / p.Gt);
    const int ntw = (t1 - t0 - warp + kWarps - 1) / kWarps;  // tiles owned by this warp

    constexpr uint32_t OC_OFF = 0;
    constexpr uint32_t HI_OFF = PAIR_T ? 128u : 0u;                      // a2/a3 column offset
    constexpr uint32_t T_OFF = PAIR_T ? (uint32_t)kOcBytes : 128u;       // residual table
    constexpr int NTOK_C = PAIR_T ? 2 : 1;
    constexpr bool NAIVE = kNaiveOcBuild && !PAIR_T && !RESID && !NIB;
    // One token, no residual table, no rotation: x~, the mbarriers and the
    // running sums live in the image rows' unused halves (kXGaps).
    constexpr bool GAPS = kImageGaps<PAIR_T, RESID, ROT>;
    constexpr uint32_t X_OFF = GAPS ? kXGaps : ((PAIR_T && RESID) ? 2u * kOcBytes : (uint32_t)kOcBytes);
    constexpr uint32_t XS_BYTES = PAIR_T ? kXStageBytes : kXStageBytes / 2;   // x~ of 1 or 2 tokens
    // mbarriers: index staging copy (+0), 8 bytes each
    constexpr uint32_t BAR_OFF = GAPS ? gap_off(247) : X_OFF + XS_BYTES;
    constexpr uint32_t ACC_OFF = GAPS ? (uint32_t)kOcBytes : BAR_OFF + 128u;   // (gaps: unused)
    // Running sums of tile tl: 128 bytes [16 rows][2 tokens] fp32.
    auto acc_off = [&](int tl) -> uint32_t {
        return GAPS ? gap_off(tl) : ACC_OFF + (uint32_t)tl * kTileRows * 2u * 4u;
    };
    // The reduction stage starts after the image (gaps) or after the sums.
    const uint32_t STAGE_OFF = GAPS ? (uint32_t)kOcBytes : ACC_OFF + (uint32_t)p.acc_tiles * kTileRows * 2u * 4u;
    // GROUPED: one codebook per tiles_per_cb row tiles (else one shared codebook).
    const int cb_first = GROUPED ? t0 / p.tiles_per_cb : 0;
    const int cb_last = GROUPED ? (t1 - 1) / p.tiles_per_cb : 0;

    // ---- prologue: weights only ----
    EVA_STAMP(0);
    pdl_launch();
    // A CTA may write a peer's shared memory only once the peer runs: arrive
    // now, wait (long satisfied) before the first remote store.
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    // The first slice's index bytes of the leading `staged` tiles: one bulk
    // copy into shared memory, completing on an mbarrier.
    const int staged = min(p.wi_staged, t1 - t0);
    const uint32_t stage_bytes_c = (uint32_t)((p.acc_tiles + p.Gs - 1) / p.Gs) * p.Gs * kTileRows * 2u * 4u;
    // Fused rotation: x~ of all this CTA's slices [ceil(S / Gs)][tokens][256]
    // fp32, then the rotation's scratch.
    const uint32_t ROT_OFF = (STAGE_OFF + stage_bytes_c + 127u) & ~127u;
    const bool rot_all = ROT && p.rot_m >= 256;   // Paley m >= 256: all slices at once
    const uint32_t xt_bytes = rot_all ? (uint32_t)((p.S + p.Gs - 1) / p.Gs) * NTOK_C * kSliceK * 4u : 0u;
    const uint32_t rot_bytes = ROT ? xt_bytes + rot_scratch_bytes(p.rot_b, p.rot_m, NTOK_C) : 0u;
    const uint32_t WIS_OFF = ROT_OFF + rot_bytes;
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(eva_smem + BAR_OFF);
    if (tid == 0 && staged > 0) {
        mbar_init(bar, 1);
        const uint8_t *src = p.wi + ((size_t)s0 * p.T + t0) * UB;
        const uint32_t bytes = (uint32_t)staged * UB;
        if (p.skip_stage_copy) {
            // Failure-detection test: nothing arrives and nothing is in flight;
            // the bounded wait below gives up and records it.
        } else if (staged > 0 && !EVA_BAD_G(BUF_WI, src, bytes) && !EVA_BAD_S(WIS_OFF) &&
            !EVA_BAD_S(WIS_OFF + bytes - 4u)) {
            mbar_arrive_expect_tx(bar, bytes);
            const uint32_t dst = (uint32_t)__cvta_generic_to_shared(eva_smem + WIS_OFF);
            for (uint32_t off = 0; off < bytes; off += 32768u)
                bulk_copy_g2s(dst + off, src + off, min(32768u, bytes - off), bar);
        } else {
            mbar_arrive(bar);
        }
    }
    if (tid < s1 - s0) {
        // Bulk L2 prefetch of this CTA's index range (the staged part excepted).
        const int skip = (tid == 0) ? staged : 0;
        const size_t u = (size_t)(s0 + tid) * p.T + t0 + skip;
        const uint32_t nt = (uint32_t)(t1 - t0 - skip);
        if (nt > 0 && !EVA_BAD_G(BUF_WI, p.wi + u * UB, nt * UB))
            prefetch_l2_bulk(p.wi + u * UB, nt * UB);
        if (RESID) {
            const size_t ur = (size_t)(s0 + tid) * p.T + t0;
            const uint32_t ntr = (uint32_t)(t1 - t0);
            if (!EVA_BAD_G(BUF_SG, p.sg + ur * kSignUnitBytes, ntr * kSignUnitBytes))
                prefetch_l2_bulk(p.sg + ur * kSignUnitBytes, ntr * kSignUnitBytes);
            if (!EVA_BAD_G(BUF_AL, p.al + ur * kAlphaUnitHalves, ntr * kAlphaUnitHalves * 2))
                prefetch_l2_bulk(p.al + ur * kAlphaUnitHalves, ntr * kAlphaUnitHalves * 2);
        }
    }
    uint32_t bfrag[4];
    int cur_cb = cb_first;   // codebook whose fragments bfrag holds
    load_codebook_frag(p, cb_first, warp, g, q, bfrag);
    // Per-group codebooks: the raw fragments of the codebook the next pass
    // uses are loaded one pass ahead (the load then overlaps a whole pass).
    uint32_t bnext[4] = {0u, 0u, 0u, 0u};
    int next_cb = -1;
    if (GROUPED && cb_last > cb_first) {
        next_cb = cb_first + 1;
        load_codebook_raw(p, next_cb, warp, g, q, bnext);
    }

    // Routing matrices of the accumulating MMA (B operand, 16 x 8, 0/1).
    // One token: column 0 sums the low half of a0/a1 and the high half of
    // a2/a3.  Token pair: column 0 sums the low halves, column 1 the high.
    const uint32_t ONE_LO = 0x00003C00u, ONE_HI = 0x3C000000u;
    uint32_t bo0, bo1;
    if (!PAIR_T) {
        bo0 = g == 0 ? ONE_LO : 0u;
        bo1 = g == 0 ? ONE_HI : 0u;
    } else {
        bo0 = bo1 = g == 0 ? ONE_LO : (g == 1 ? ONE_HI : 0u);
    }
    // Residual table routing: lanes q = 0,1 feed group 0, q = 2,3 group 1.
    uint32_t bt = 0;
    if (RESID) {
        if (!PAIR_T) bt = (g == (q >> 1)) ? ONE_LO : 0u;
        else bt = (g == 2 * (q >> 1)) ? ONE_LO : (g == 2 * (q >> 1) + 1 ? ONE_HI : 0u);
    }

    // x (unless the caller vouches it is ready) and y belong to the stream
    // order from here on.
    if (!p.independent) pdl_wait();
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    EVA_STAMP(1);

    const int npairs = PAIR_T ? (p.B + 1) / 2 : 1;
    constexpr int NTOK = PAIR_T ? 2 : 1;
    const int ctiles = t1 - t0;
    // Running sums over this CTA's slices, [ctiles][16 rows][2 tokens] (128
    // bytes per tile), and the reduction stage of the tiles this CTA owns
    // (tile tl belongs to cluster rank tl % Gs):
    // [ceil(acc_tiles / Gs) slots][Gs sources][16 rows][2 tokens].
    bool wi_ready = false;   // the staging copy has landed (waited for once)
    const float *stage = reinterpret_cast<const float *>(eva_smem + STAGE_OFF);
    const uint32_t stage_addr = (uint32_t)__cvta_generic_to_shared(eva_smem + STAGE_OFF);
    for (int pr = 0; pr < npairs; ++pr) {
        for (int s = s0; s < s1; ++s) {
            const uint32_t x_off = rot_all ? ROT_OFF + (uint32_t)((s - s0) * NTOK_C) * kSliceK * 4u : X_OFF;
            if constexpr (ROT) {
                if (!rot_all) stage_x_rot<PAIR_T>(p, s, pr, warp, lane, tid, X_OFF, ROT_OFF);
            } else {
                stage_x<PAIR_T>(p, s, pr, warp, lane, X_OFF);
            }
            for (int cb = cb_first; cb <= cb_last; ++cb) {
                // This warp's tiles that use codebook cb: the index range [i0, i1).
                int i0 = 0, i1 = ntw;
                if (GROUPED) {
                    const int lo = max(cb * p.tiles_per_cb, t0), hi = (cb + 1) * p.tiles_per_cb;
                    i0 = max(0, (lo - t0 - warp + kWarps - 1) / kWarps);
                    i1 = min(ntw, max(0, (hi - t0 - warp + kWarps - 1) / kWarps));
                    if (cb != cur_cb) {
                        if (cb == next_cb) frag_from_raw(bnext, bfrag);
                        else load_codebook_frag(p, cb, warp, g, q, bfrag);
                        cur_cb = cb;
                        // the codebook of the pass after this one
                        const int nxt = cb < cb_last ? cb + 1 : ((s + 1 < s1 || pr + 1 < npairs) ? cb_first : -1);
                        if (nxt >= 0 && nxt != cb) {
                            next_cb = nxt;
                            load_codebook_raw(p, nxt, warp, g, q, bnext);
                        }
                    }
                }
                // Tiles [i0, i_st) of the first slice read their indices from the
                // shared-memory copy; the rest stream through a lookahead ring of
                // LA units: the first ones load (from L2, where the prologue's
                // bulk prefetch put them) while the image builds, and each
                // processed tile refills the ring's tail.
                const int i_st = (s == s0) ? min(i1, max(i0, (staged - warp + kWarps - 1) / kWarps)) : i0;
                // With a residual the ring also carries each unit's signs and alpha.
                constexpr int LR = RESID ? LA : 1;
                uint4 nb[LA][2];
                uint4 ns[LR];
                uint2 na[LR];
                if constexpr (!RESID) {
                    ns[0] = make_uint4(0u, 0u, 0u, 0u);
                    na[0] = make_uint2(0u, 0u);
                }
#pragma unroll
                for (int d = 0; d < LA; ++d) {
                    nb[d][0] = nb[d][1] = make_uint4(0u, 0u, 0u, 0u);
                    if constexpr (RESID) {
                        ns[d] = make_uint4(0u, 0u, 0u, 0u);
                        na[d] = make_uint2(0u, 0u);
                    }
                    if (i_st + d < i1) {
                        const size_t unit = (size_t)s * p.T + t0 + warp + kWarps * (i_st + d);
                        load_unit<NIB>(p, p.wi + unit * UB + 16 * lane, nb[d][0], nb[d][1]);
                        if constexpr (RESID) load_resid(p, unit, lane, g, q, ns[d], na[d]);
                    }
                }
                // Paley blocks with m >= 256: x~ of every slice of this CTA at
                // once (each chunk transformed once), after the first index
                // loads are in flight; the slices then read their part of it.
                if constexpr (ROT) {
                    if (rot_all && s == s0 && cb == cb_first)
                        stage_x_rot_all<PAIR_T>(p, s0, s1, pr, warp, lane, tid, ROT_OFF, ROT_OFF + xt_bytes);
                }
                __syncthreads();  // x~ staged, accumulator cleared, previous image consumed
                EVA_STAMP(2);
                build_oc<PAIR_T, NAIVE>(p, warp, g, q, bfrag, x_off);
                if (RESID && cb == cb_first) build_sign_table<PAIR_T>(p, warp, lane, T_OFF, x_off);
                __syncthreads();
                EVA_STAMP(3);
                if (staged > 0 && !wi_ready) {
                    // Bounded: if the copy never lands the CTA records it, skips
                    // nothing else and still joins the cluster barrier below.
                    wi_ready = true;
                    if (!mbar_wait_bounded(bar, 0, p.wait_rounds) && tid == 0 && p.status) atomicOr(p.status, 1);
                }
                // One tile: 32 lookups per lane, accumulated by 8 MMAs (+ the residual).
                auto tile = [&](const int tl, const uint4 v0, const uint4 v1, const uint4 sv, const uint2 araw) {
                    const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                    // Even and odd k-steps accumulate in two chains.
                    float da[4] = {0.f, 0.f, 0.f, 0.f}, db[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int s8 = 0; s8 < 8; ++s8) {
                        const uint32_t cw = (4u * lane + 16u * s8) & 127u;   // 4 * oc_col(lane, s8)
                        uint32_t o0, o1, o2, o3;
                        if constexpr (NIB) {
                            // word s8 / 2, nibbles 4 (s8 & 1) + r: index c -> (c << 8) | cw
                            const uint32_t w = wv[s8 >> 1];
                            const int sh = 16 * (s8 & 1);
                            o0 = OC_OFF + ((((w >> sh) << 8) & 0xF00u) | cw);
                            o1 = OC_OFF + ((((w >> sh) << 4) & 0xF00u) | cw);
                            o2 = OC_OFF + HI_OFF + (((w >> sh) & 0xF00u) | cw);
                            o3 = OC_OFF + HI_OFF + (((w >> (sh + 4)) & 0xF00u) | cw);
                        } else if constexpr (NAIVE) {
                            o0 = OC_OFF + (cw << 8) + ((wv[s8] & 0xFFu) << 2);
                            o1 = OC_OFF + (cw << 8) + (((wv[s8] >> 8) & 0xFFu) << 2);
                            o2 = OC_OFF + (cw << 8) + (((wv[s8] >> 16) & 0xFFu) << 2);
                            o3 = OC_OFF + (cw << 8) + ((wv[s8] >> 24) << 2);
                        } else {
                            o0 = OC_OFF + __byte_perm(wv[s8], cw, 0x5504);
                            o1 = OC_OFF + __byte_perm(wv[s8], cw, 0x5514);
                            o2 = OC_OFF + HI_OFF + __byte_perm(wv[s8], cw, 0x5524);
                            o3 = OC_OFF + HI_OFF + __byte_perm(wv[s8], cw, 0x5534);
                        }
                        const uint32_t a0 = EVA_BAD_S(o0) ? 0u : lds32(o0);
                        const uint32_t a1 = EVA_BAD_S(o1) ? 0u : lds32(o1);
                        const uint32_t a2 = EVA_BAD_S(o2) ? 0u : lds32(o2);
                        const uint32_t a3 = EVA_BAD_S(o3) ? 0u : lds32(o3);
                        if (s8 & 1) mma_f16_k16(db, a0, a1, a2, a3, bo0, bo1);
                        else mma_f16_k16(da, a0, a1, a2, a3, bo0, bo1);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) da[e] += db[e];
                    if (RESID) {
                        const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
                        float dt[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int mi = 0; mi < 4; ++mi) {
                            const uint32_t m0 = 4u * sign_pos(lane, mi, 0), m2 = 4u * sign_pos(lane, mi, 2);
                            const uint32_t o0 = T_OFF + __byte_perm(sw[mi], m0, 0x5504);
                            const uint32_t o1 = T_OFF + __byte_perm(sw[mi], m0, 0x5514);
                            const uint32_t o2 = T_OFF + __byte_perm(sw[mi], m2, 0x5524);
                            const uint32_t o3 = T_OFF + __byte_perm(sw[mi], m2, 0x5534);
                            const uint32_t a0 = EVA_BAD_S(o0) ? 0u : lds32(o0);
                            const uint32_t a1 = EVA_BAD_S(o1) ? 0u : lds32(o1);
                            const uint32_t a2 = EVA_BAD_S(o2) ? 0u : lds32(o2);
                            const uint32_t a3 = EVA_BAD_S(o3) ? 0u : lds32(o3);
                            mma_f16_k16(dt, a0, a1, a2, a3, bt, bt);
                        }
                        float dt1[4] = {0.f, 0.f, 0.f, 0.f};
                        if (PAIR_T) {  // group 1 of a token pair sits in lane q = 1
#pragma unroll
                            for (int e = 0; e < 4; ++e) dt1[e] = __shfl_down_sync(0xffffffffu, dt[e], 1);
                        }
                        if (q == 0) {
                            const __half2 ag = *reinterpret_cast<const __half2 *>(&araw.x);   // row g: grp 0, 1
                            const __half2 ag8 = *reinterpret_cast<const __half2 *>(&araw.y);  // row g+8
                            const float a_g0 = __low2float(ag), a_g1 = __high2float(ag);
                            const float a_h0 = __low2float(ag8), a_h1 = __high2float(ag8);
                            if (!PAIR_T) {
                                da[0] += a_g0 * dt[0] + a_g1 * dt[1];
                                da[2] += a_h0 * dt[2] + a_h1 * dt[3];
                            } else {
                                da[0] += a_g0 * dt[0] + a_g1 * dt1[0];
                                da[1] += a_g0 * dt[1] + a_g1 * dt1[1];
                                da[2] += a_h0 * dt[2] + a_h1 * dt1[2];
                                da[3] += a_h0 * dt[3] + a_h1 * dt1[3];
                            }
                        }
                    }
                    // Lanes q = 0 hold column 0 (and 1): rows g and g + 8 of the tile.
                    // A tile is visited once per slice: the first visit stores.
                    if (q == 0) {
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int e = 0; e < NTOK; ++e) {
                                const uint32_t ao = acc_off(tl) + (uint32_t)((g + 8 * h) * 2 + e) * 4u;
                                if (!EVA_BAD_S(ao)) {
                                    float *ap = reinterpret_cast<float *>(eva_smem + ao);
                                    *ap = (s == s0) ? da[2 * h + e] : *ap + da[2 * h + e];
                                }
                            }
                    }
                };
                // Staged tiles first (indices from shared memory) ...
#pragma unroll 1
                for (int i = i0; i < i_st; ++i) {
                    const int tl = warp + kWarps * i;              // tile index within the CTA
                    const uint32_t wo = WIS_OFF + (uint32_t)tl * UB + 16u * lane;
                    const uint4 v0 = (EVA_BAD_S(wo) || EVA_BAD_S(wo + 12u)) ? make_uint4(0u, 0u, 0u, 0u) : lds128(wo);
                    const uint4 v1 = (NIB || EVA_BAD_S(wo + 512u) || EVA_BAD_S(wo + 524u)) ? make_uint4(0u, 0u, 0u, 0u)
                                                                                              : lds128(wo + 512u);
                    uint4 sv = make_uint4(0u, 0u, 0u, 0u);
                    uint2 av = make_uint2(0u, 0u);
                    if (RESID) load_resid(p, (size_t)s * p.T + t0 + tl, lane, g, q, sv, av);
                    tile(tl, v0, v1, sv, av);
                }
                // ... then the streamed ones, through the lookahead ring.
#pragma unroll 1
                for (int i = i_st; i < i1; ++i) {
                    const int tl = warp + kWarps * i;              // tile index within the CTA
                    const size_t unit = (size_t)s * p.T + t0 + tl;
                    const uint4 v0 = nb[0][0], v1 = nb[0][1];
                    const uint4 sv = ns[0];
                    const uint2 av = na[0];
#pragma unroll
                    for (int d = 0; d + 1 < LA; ++d) {
                        nb[d][0] = nb[d + 1][0];
                        nb[d][1] = nb[d + 1][1];
                        if constexpr (RESID) {
                            ns[d] = ns[d + 1];
                            na[d] = na[d + 1];
                        }
                    }
                    if (i + LA < i1) {
                        const size_t un = unit + (size_t)kWarps * LA;
                        load_unit<NIB>(p, p.wi + un * UB + 16 * lane, nb[LA - 1][0], nb[LA - 1][1]);
                        if (RESID) load_resid(p, un, lane, g, q, ns[LR - 1], na[LR - 1]);
                    }
                    tile(tl, v0, v1, sv, av);
                }
            }
        }

        // Epilogue of this token (pair): every CTA pushes the 128-byte sum
        // block of each of its tiles into the shared memory of the cluster CTA
        // that owns the tile (rank tl % Gs) with 16-byte remote stores; after
        // the cluster barrier each owner adds the Gs contributions of its
        // tiles in a fixed order (bitwise reproducible) and stores y.
        EVA_STAMP(4);
        __syncthreads();
        for (int i = tid; i < ctiles * 8; i += kThreads) {
            const int tl = i >> 3, chunk = i & 7;
            const uint32_t src = acc_off(tl) + (uint32_t)(chunk * 4) * 4u;
            const uint32_t dst = (uint32_t)((((tl / p.Gs) * p.Gs + ts) * 32 + chunk * 4) * 4);
            if (!EVA_BAD_S(src) && !EVA_BAD_S(src + 12u) && !EVA_BAD_S(STAGE_OFF + dst) && !EVA_BAD_S(STAGE_OFF + dst + 12u)) {
                const float4 v = *reinterpret_cast<const float4 *>(eva_smem + src);
                st_dsmem_v4(stage_addr + dst, (uint32_t)(tl % p.Gs), v);
            }
        }
        cluster_sync_all();
        EVA_STAMP(5);
        {
            // Four consecutive threads per output each add every fourth source
            // (k = part, part + 4, ...), then two shuffles combine them: a
            // fixed order, so y repeats bitwise.  The loop bound is the same
            // for every thread (every lane takes part in the shuffles).
            constexpr int SPL = 4;
            const int my_tiles = (ctiles - ts + p.Gs - 1) / p.Gs;   // tiles tl = ts + Gs * slot
            const int nout = my_tiles * kTileRows * NTOK;
            for (int base = 0; base < nout * SPL; base += kThreads) {
                const int idx = (base + tid) / SPL, part = (base + tid) % SPL;
                const int e = idx % NTOK, row = (idx / NTOK) % kTileRows, slot = idx / (NTOK * kTileRows);
                const int tl = ts + p.Gs * slot;
                const int tok = PAIR_T ? 2 * pr + e : 0;
                const int o = kTileRows * (t0 + tl) + row;
                const bool valid = idx < nout && tok < p.B && o < p.N;
                float sum = 0.f;
                if (valid) {
                    for (int k = part; k < p.Gs; k += SPL) {
                        const uint32_t si = (uint32_t)(((slot * p.Gs + k) * kTileRows + row) * 2 + e);
                        sum += EVA_BAD_S(STAGE_OFF + 4u * si) ? 0.f : stage[si];
                    }
                }
                sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                if (!valid || part != 0) continue;
                const size_t yi = (size_t)tok * p.N + o;
                if (p.out_f32) {
                    float *yp = reinterpret_cast<float *>(p.y) + yi;
                    if (!EVA_BAD_G(BUF_Y, yp, 4)) *yp = sum;
                } else {
                    __half *yp = reinterpret_cast<__half *>(p.y) + yi;
                    if (!EVA_BAD_G(BUF_Y, yp, 2)) *yp = __float2half_rn(sum);
                }
            }
        }
        // Before the next pair's sums are pushed, every owner must be done
        // reading this pair's stage (and this CTA's warps done with acc_s).
        if (pr + 1 < npairs) cluster_sync_all();
    }
    // No bulk copy may still be writing this CTA's shared memory at exit.
    if (staged > 0 && !wi_ready && !mbar_wait_bounded(bar, 0, p.wait_rounds) && tid == 0 && p.status)
        atomicOr(p.status, 2);
    // Independent calls still complete after the preceding kernel, so that
    // later calls that wait on this one see the stream order.
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

template <bool PAIR_T, bool RESID, bool GROUPED, bool ROT, bool NIB>
__global__ void __launch_bounds__(kThreads, kLookupMinBlocks<PAIR_T>) eva_lookup_kernel(const LookupParams p) {
    lookup_body<PAIR_T, RESID, GROUPED, ROT, NIB>(p, blockIdx.x);
}

// The one-token, no-residual, no-rotation program with the register budget of
// three CTAs per SM: for independent calls of layers with few tiles per CTA,
// where a third layer in flight outweighs the tighter registers.
template <bool GROUPED, bool NIB>
__global__ void __launch_bounds__(kThreads, 3) eva_lookup_kernel3(const LookupParams p) {
    lookup_body<false, false, GROUPED, false, NIB>(p, blockIdx.x);
}

// Several independent layers of one shape and format in one launch: layer
// blockIdx.x / ctas_per_layer, CTA blockIdx.x % ctas_per_layer of it (a
// cluster never spans two layers: ctas_per_layer is a multiple of Gs).
constexpr int kMaxGroup = 16;
struct LookupGroup {
    int count, ctas_per_layer;
    LookupParams p[kMaxGroup];
};

template <bool PAIR_T, bool RESID>
__global__ void __launch_bounds__(kThreads, kLookupMinBlocks<PAIR_T>) eva_lookup_group_kernel(const LookupGroup g) {
    const int li = blockIdx.x / g.ctas_per_layer;
    if (li >= g.count) return;
    lookup_body<PAIR_T, RESID, false, false, false>(g.p[li], blockIdx.x - li * g.ctas_per_layer);
}

// ----------------------------------------------------- Hadamard rotation
//
// x~ = hsign (.) (H_b x) / sqrt(b) per block of b inputs: the natural-order
// (Sylvester) fast Walsh-Hadamard transform in shared memory, fp32.
// Grid (K / b, B).
__global__ void __launch_bounds__(1024) eva_hadamard_kernel(const __half *__restrict__ x,
                                                            const int8_t *__restrict__ hs,
                                                            float *__restrict__ xt, int K, int b,
                                                            float scale, int independent) {
    float *sb = reinterpret_cast<float *>(eva_smem);
    const int blk = blockIdx.x, tok = blockIdx.y;
    pdl_launch();
    if (!independent) pdl_wait();  // x may be the output of the preceding kernel
    const unsigned short *xb =
        reinterpret_cast<const unsigned short *>(x) + (size_t)tok * K + (size_t)blk * b;
    for (int i = threadIdx.x; i < b; i += blockDim.x) sb[i] = __half2float(__ushort_as_half(__ldcg(xb + i)));
    for (int h = 1; h < b; h <<= 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < b / 2; i += blockDim.x) {
            const int lo = (i / h) * 2 * h + (i % h);
            const float a = sb[lo], c = sb[lo + h];
            sb[lo] = a + c;
            sb[lo + h] = a - c;
        }
    }
    __syncthreads();
    if (independent) pdl_wait();  // the rotated input is this handle's workspace
    for (int i = threadIdx.x; i < b; i += blockDim.x) {
        const int k = blk * b + i;
        xt[(size_t)tok * K + k] = (float)hs[k] * sb[i] * scale;
    }
}

// The Paley-block rotation of weight rows in the quantizer: grid (K / b, rows), b / 2 threads at most 1024, b floats
// of shared memory.  Stages h < m of the fast transform inside every
// m-sub-block, then out[a m + c] = sum_a' H28[a'][a] y[a' m + c] in order
// a' = 0..27, times s / sqrt(b).
__global__ void __launch_bounds__(1024) eva_paley_rows_kernel(const __half *__restrict__ x,
                                                              const int8_t *__restrict__ hs,
                                                              const int8_t *__restrict__ h28,
                                                              float *__restrict__ xt, int K, int b, int m,
                                                              float scale) {
    float *sb = reinterpret_cast<float *>(eva_smem);
    const int blk = blockIdx.x, tok = blockIdx.y;
    const unsigned short *xb =
        reinterpret_cast<const unsigned short *>(x) + (size_t)tok * K + (size_t)blk * b;
    for (int i = threadIdx.x; i < b; i += blockDim.x) sb[i] = __half2float(__ushort_as_half(__ldcg(xb + i)));
    for (int h = 1; h < m; h <<= 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < b / 2; i += blockDim.x) {
            const int lo = (i / h) * 2 * h + (i % h);
            const float a = sb[lo], c = sb[lo + h];
            sb[lo] = a + c;
            sb[lo + h] = a - c;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < b; i += blockDim.x) {
        const int a = i / m, c = i - a * m;
        float acc = 0.f;
        for (int a2 = 0; a2 < 28; ++a2) {
            const float y = sb[a2 * m + c];
            acc = h28[a2 * 28 + a] > 0 ? acc + y : acc - y;
        }
        const int k = blk * b + i;
        xt[(size_t)tok * K + k] = (float)hs[k] * acc * scale;
    }
}

// The Paley-block rotation of the input for the two-kernel routes (tcgen05
// and dequantize paths): x~ = s (.) (H28 (x) H_m) x / sqrt(b) per block of
// b = 28 m inputs.  The two Kronecker factors commute, so CTA (block, a)
// first mixes the block's 28 sub-blocks into its own one,
// z[c] = sum_a' H28[a'][a] x[a' m + c] (a' = 0..27, fp32), then runs the
// m-point fast transform on z in shared memory and writes x~[a m + c]:
// 28 CTAs per block and token and no step done twice.  Grid (28 K / b, B),
// m threads (64..1024), m floats of shared memory.
__global__ void __launch_bounds__(1024) eva_paley_x_kernel(const __half *__restrict__ x,
                                                           const int8_t *__restrict__ hs,
                                                           const int8_t *__restrict__ h28,
                                                           float *__restrict__ xt, int K, int b, int m,
                                                           float scale, int independent) {
    float *sb = reinterpret_cast<float *>(eva_smem);
    const int blk = blockIdx.x / 28, a = blockIdx.x % 28, tok = blockIdx.y;
    pdl_launch();
    if (!independent) pdl_wait();  // x may be the output of the preceding kernel
    const unsigned short *xb =
        reinterpret_cast<const unsigned short *>(x) + (size_t)tok * K + (size_t)blk * b;
    for (int c = threadIdx.x; c < m; c += blockDim.x) {
        float acc = 0.f;
#pragma unroll 4
        for (int a2 = 0; a2 < 28; ++a2) {
            const float v = __half2float(__ushort_as_half(__ldcg(xb + a2 * m + c)));
            acc = __ldg(h28 + a2 * 28 + a) > 0 ? acc + v : acc - v;
        }
        sb[c] = acc;
    }
    for (int h = 1; h < m; h <<= 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < m / 2; i += blockDim.x) {
            const int lo = (i / h) * 2 * h + (i % h);
            const float u = sb[lo], w = sb[lo + h];
            sb[lo] = u + w;
            sb[lo + h] = u - w;
        }
    }
    __syncthreads();
    if (independent) pdl_wait();  // the rotated input is this handle's workspace
    for (int c = threadIdx.x; c < m; c += blockDim.x) {
        const int k = blk * b + a * m + c;
        xt[(size_t)tok * K + k] = (float)hs[k] * sb[c] * scale;
    }
}

// ------------------------------------------------------- create-time repack

// One thread per packed byte; padding (rows >= N, sub-vectors >= J) is 0.
__global__ void eva_repack_wi_kernel(const uint8_t *__restrict__ wi, uint8_t *__restrict__ out,
                                     int N, int J, int T, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long unit = idx / kUnitBytes;
    const int b = (int)(idx % kUnitBytes);
    const int s = (int)(unit / T), t = (int)(unit % T);
    int row, jl;
    wi_unit_pos(b, row, jl);
    const int o = kTileRows * t + row, j = kSliceJ * s + jl;
    out[idx] = (o < N && j < J) ? wi[(size_t)o * J + j] : (uint8_t)0;
}

// Inverse of the repack (test hook): canonical [N][J] from the packed stream.
__global__ void eva_unpack_wi_kernel(const uint8_t *__restrict__ packed, uint8_t *__restrict__ wi,
                                     int N, int J, int T, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long unit = idx / kUnitBytes;
    const int b = (int)(idx % kUnitBytes);
    const int s = (int)(unit / T), t = (int)(unit % T);
    int row, jl;
    wi_unit_pos(b, row, jl);
    const int o = kTileRows * t + row, j = kSliceJ * s + jl;
    if (o < N && j < J) wi[(size_t)o * J + j] = packed[idx];
}

// 4-bit indices: canonical [N][J/2] (sub-vector 2t in the low nibble of byte
// t) -> units of 512 bytes; one thread per unit byte (two nibbles).
__global__ void eva_repack_wi4_kernel(const uint8_t *__restrict__ wi, uint8_t *__restrict__ out, int N, int J,
                                      int T, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long unit = idx / kUnitBytes4;
    const int b = (int)(idx % kUnitBytes4);
    const int s = (int)(unit / T), t = (int)(unit % T);
    unsigned v = 0;
    for (int h = 0; h < 2; ++h) {
        int row, jl;
        wi4_unit_pos(2 * b + h, row, jl);
        const int o = kTileRows * t + row, j = kSliceJ * s + jl;
        const unsigned c = (o < N && j < J) ? (wi[(size_t)o * (J / 2) + j / 2] >> (4 * (j & 1))) & 15u : 0u;
        v |= c << (4 * h);
    }
    out[idx] = (uint8_t)v;
}

// Inverse (test hook): one thread per canonical byte.
__global__ void eva_unpack_wi4_kernel(const uint8_t *__restrict__ packed, uint8_t *__restrict__ wi, int N, int J,
                                      int T, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int o = (int)(idx / (J / 2)), t2 = (int)(idx % (J / 2));
    unsigned v = 0;
    for (int h = 0; h < 2; ++h) {
        const int j = 2 * t2 + h, s = j / kSliceJ, jl = j % kSliceJ;
        const int n = wi4_unit_nibble(o % kTileRows, jl);
        const long long unit = (long long)s * T + o / kTileRows;
        const unsigned c = (packed[unit * kUnitBytes4 + (n >> 1)] >> (4 * (n & 1))) & 15u;
        v |= c << (4 * h);
    }
    wi[idx] = (uint8_t)v;
}

__global__ void eva_repack_signs_kernel(const uint8_t *__restrict__ sg, uint8_t *__restrict__ out,
                                        int N, int K8, int T, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long unit = idx / kSignUnitBytes;
    const int b = (int)(idx % kSignUnitBytes);
    const int s = (int)(unit / T), t = (int)(unit % T);
    int row, m;
    sign_unit_pos(b, row, m);
    const int o = kTileRows * t + row, mm = (kSliceK / 8) * s + m;
    out[idx] = (o < N && mm < K8) ? sg[(size_t)o * K8 + mm] : (uint8_t)0;
}

__global__ void eva_unpack_signs_kernel(const uint8_t *__restrict__ packed, uint8_t *__restrict__ sg,
                                        int N, int K8, int T, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long unit = idx / kSignUnitBytes;
    const int b = (int)(idx % kSignUnitBytes);
    const int s = (int)(unit / T), t = (int)(unit % T);
    int row, m;
    sign_unit_pos(b, row, m);
    const int o = kTileRows * t + row, mm = (kSliceK / 8) * s + m;
    if (o < N && mm < K8) sg[(size_t)o * K8 + mm] = packed[idx];
}

__global__ void eva_repack_alpha_kernel(const __half *__restrict__ al, __half *__restrict__ out,
                                        int N, int NG, int T, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long unit = idx / kAlphaUnitHalves;
    const int e = (int)(idx % kAlphaUnitHalves);
    const int s = (int)(unit / T), t = (int)(unit % T);
    int row, grp;
    alpha_unit_pos(e, row, grp);
    const int o = kTileRows * t + row, gq = 2 * s + grp;
    out[idx] = (o < N && gq < NG) ? al[(size_t)o * NG + gq] : __float2half(0.f);
}

}  // namespace eva
