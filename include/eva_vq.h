/*
 * eva_vq.h -- C ABI of the B200 (sm_100a) decode-phase linear layer with
 * vector-quantized weights.
 *
 * The operation (EVA: Accelerating LLM Decoding via an Efficient Vector
 * Quantization Architecture, technical summary section 2.A):
 *   - the input x of one decode step is cut into J = K/d sub-vectors x_j of
 *     length d (d = 4);
 *   - the weight codebook WC holds 2^n centroids of length d (n = 8: 256
 *     centroids and one index byte per 4 weights, 2 bits per weight; or
 *     n = 4: 16 centroids, two indices per byte, 1 bit per weight);
 *   - the output codebook OC[j][c] = <x_j, WC[c]> turns the matrix-vector
 *     product into a small matrix-matrix product;
 *   - the output is gathered through the weight-index matrix WI and summed:
 *     y[o] = sum_j OC[j][WI[o][j]].
 * The 3.125-bit variant (Replacing MatMul with SRAM lookup: a 3-bit edge
 * inference architecture, section details and its quantize() sample) adds a
 * randomized Hadamard rotation of the input and a 1-bit residual sign per
 * weight with one fp16 scale alpha per group of 128 inputs:
 *   y[o] = sum_j OC~[j][WI[o][j]] + sum_q alpha[o][q] sum_{k in q} sigma[o][k] x~[k],
 * with x~ = s (.) (H_b^T x) / sqrt(b) blockwise (s = hsign; H_b a Sylvester
 * matrix, or the Kronecker product of an order-28 Paley matrix with one).
 *
 * All entry points return a status code and never abort or trap.  No entry
 * point throws.  Device pointers must be 16-byte aligned.
 */
#ifndef EVA_VQ_H
#define EVA_VQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EVA_API __attribute__((visibility("default")))
#else
#define EVA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *eva_stream_t;

typedef enum {
    EVA_OK = 0,
    EVA_ERR_INVALID_ARG = 1,     /* bad pointer, size, alignment or handle      */
    EVA_ERR_UNSUPPORTED = 2,     /* valid but not implemented (d != 4, n not 4/8) */
    EVA_ERR_CUDA = 3,            /* a CUDA runtime call failed                   */
    EVA_ERR_OOM = 4,             /* device allocation failed in create           */
    EVA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device wait gave up                */
    EVA_ERR_NO_DEVICE = 6,       /* no sm_100 device is current                  */
    EVA_ERR_DEVICE_CHECK = 7,    /* checked build: a kernel access was out of bounds */
    EVA_ERR_SCRATCH_TOO_SMALL = 8 /* eva_vq_linear_run_noalloc: B * K * 4 > 4 MiB      */
} eva_status_t;

typedef enum { EVA_F16 = 0, EVA_F32 = 1 } eva_dtype_t;

/* Kernel family used by run(). */
typedef enum {
    EVA_PATH_AUTO = 0,        /* pick per call from B and the codebook layout   */
    EVA_PATH_OC_LOOKUP = 1,   /* output codebook in shared memory + lookups     */
    EVA_PATH_DEQUANT_MMA = 2, /* codebook gather into warp-level tensor-core
                                 operands (mma.sync; 8-bit indices; residual
                                 and rotation with one shared codebook only);
                                 AUTO takes it for B >= 3 (B >= 2 with
                                 per-group codebooks) when the layer allows it
                                 and EVA_PATH_TCGEN05 does not                  */
    EVA_PATH_TCGEN05 = 3      /* weights rebuilt from the codebook into tensor
                                 memory and multiplied by tcgen05.mma (fp32
                                 accumulation in tensor memory), residual and
                                 rotation included; 8-bit indices, K a multiple
                                 of 64, codebook_rows 0 or a multiple of 128;
                                 AUTO takes it for B > 32 on a layer with one
                                 shared codebook (residual and rotation
                                 included), for B >= 8 on a residual or rotated
                                 layer with per-group codebooks, and otherwise
                                 not.  A rotated layer runs the standalone
                                 rotation kernel first (x~ in a handle
                                 workspace of max_batch * K * 4 bytes); a
                                 handle that may take this path (forced, or
                                 AUTO with a max_batch it applies to) keeps a
                                 second copy of the indices (and signs) in
                                 128-row blocks for it.                          */
} eva_path_t;

typedef struct {
    int32_t N;               /* output features, >= 1                                   */
    int32_t K;               /* input features, multiple of d (and of 128 with residual) */
    int32_t d;               /* sub-vector length; 4 is the only supported value        */
    int32_t index_bits;      /* n: 8 (256 centroids, one byte per index) or 4 (16
                                centroids, two indices per byte: wi is [N][K/8], the even
                                sub-vector in the low nibble; K a multiple of 8; the
                                lookup path at every batch size)                         */
    int32_t codebook_rows;   /* 0: one shared codebook; R > 0: codebook g serves rows
                                [R g, R g + R); R must be a multiple of 16 dividing N    */
    int32_t residual_group;  /* 0: no sign residual; 128: signs + one alpha per 128 k   */
    int32_t hadamard_block;  /* 0: no rotation; b dividing K: a power of two in [8, 4096]
                                (Sylvester H_b), or 28 m with m a power of two in [64, 1024]
                                (H_b = H28 (x) H_m, H28 from Paley's construction over GF(27)
                                modulo t^3 + 2t + 2; b = K gives the order-K rotation)  */
    int32_t max_batch;       /* largest B passed to run(), 1..64; sizes the workspace   */
    eva_dtype_t out_dtype;   /* dtype of y                                               */
    eva_path_t path;         /* EVA_PATH_AUTO unless a test or benchmark forces one     */
} eva_vq_desc;

typedef struct eva_vq_linear *eva_vq_linear_t;

/*
 * Create a layer.  Copies and repacks the weights into library-owned device
 * memory; the copies are enqueued on `stream`, and the caller's buffers may
 * be released once `stream` has passed this call.  All pointers are device
 * pointers (16-byte aligned):
 *   wc     fp16 [G][2^n][d], G = codebook_rows ? N / codebook_rows : 1, n = index_bits
 *   wi     u8   [N][K/d], canonical row-major, WI[o][j] = centroid of row o, sub-vector j;
 *          4-bit indices: u8 [N][K/(2d)], WI[o][j] in byte j/2, bits 4 (j mod 2) .. +3
 *   signs  u8   [N][K/8], bit i of byte m is sigma[o][8m+i] (1: +1, 0: -1); NULL unless residual
 *   alpha  fp16 [N][K/residual_group]; NULL unless residual
 *   hsign  int8 [K], entries +1 or -1; NULL unless hadamard_block
 * Returns EVA_ERR_INVALID_ARG / EVA_ERR_UNSUPPORTED before touching the
 * device when the descriptor or pointers are unusable, EVA_ERR_OOM when an
 * allocation fails (nothing is leaked), EVA_ERR_CUDA on a failed launch.
 */
EVA_API eva_status_t eva_vq_linear_create(eva_vq_linear_t *out, const eva_vq_desc *desc,
                                  const void *wc, const uint8_t *wi, const uint8_t *signs,
                                  const void *alpha, const int8_t *hsign, eva_stream_t stream);

/*
 * y = layer(x) for B tokens, asynchronous on `stream`; no host sync and no
 * allocation.  x: device fp16 [B][K]; y: device [B][N] of desc.out_dtype.
 * Both are caller-owned and must not overlap.  One handle must not run on
 * two streams at once (its workspace is shared); distinct handles are
 * independent.  Kernels are launched with programmatic dependent launch: a
 * kernel of this call may start loading weights while the previous kernel
 * on the stream is finishing, but reads x only after it has completed.
 * Rejects B < 1 or B > max_batch, null or misaligned x / y.
 */
EVA_API eva_status_t eva_vq_linear_run(eva_vq_linear_t h, const void *x, int32_t B, void *y,
                               eva_stream_t stream);

/* Flags of eva_vq_linear_run_ex. */
enum {
    /* Neither x nor y is accessed by the kernel that precedes this call on
     * `stream` (for example several layers that read activations produced
     * earlier and write distinct outputs).  The layer then runs without
     * waiting for that kernel, so consecutive independent layers overlap;
     * it still completes after it, so later calls keep the stream order.
     * Passing it when x or y IS used by the preceding kernel is a race.
     * Such calls also take a grid made for overlap (fewer CTAs, each
     * covering more K-slices and row tiles; never more CTAs than the plain
     * call): y is then summed over the K-slices in another fp32 order, so
     * it matches the plain call within the rounding tolerance, not bit for
     * bit (repeated independent calls are bitwise equal to each other). */
    EVA_RUN_INDEPENDENT = 1u
};

/* eva_vq_linear_run with flags (0 gives eva_vq_linear_run). */
EVA_API eva_status_t eva_vq_linear_run_ex(eva_vq_linear_t h, const void *x, int32_t B, void *y,
                                          eva_stream_t stream, uint32_t flags);

/*
 * Several independent layers at once: layer i computes ys[i] = layer_i(xs[i])
 * for the same B (1 <= count <= 16; all handles on the current device).  No
 * layer may read another's output.  When every layer has the first one's
 * N, K and format (8-bit indices, one shared codebook, no rotation, the same
 * residual setting and output type) and takes the lookup path at this B, or
 * every layer has the first one's N, K, output type and dequantize-path plan
 * (one shared codebook each, no residual, no rotation) and takes that path,
 * the layers run as ONE launch whose CTAs the hardware schedules as slots
 * free -- e.g. the q, k and v projections of a decoder block, which share
 * their input.  Otherwise it is one eva_vq_linear_run_ex per layer.  Results
 * are bitwise those of separate calls with the same flags.  `flags` as for eva_vq_linear_run_ex,
 * for the group as a whole.  Not part of the pages' method: a launch-level
 * convenience.
 */
EVA_API eva_status_t eva_vq_linear_run_group(const eva_vq_linear_t *hs, const void *const *xs, void *const *ys,
                                             int32_t count, int32_t B, eva_stream_t stream, uint32_t flags);

/*
 * eva_vq_linear_run for callers that must not touch the device allocator.
 * No counterpart in the EVA pages or the 3-bit SRAM-lookup article: it is a
 * deployment convenience of this library.
 *
 * Who needs it: code that runs where cudaMalloc is off limits -- inside a
 * stream capture that records a whole decode step into a CUDA graph (an
 * allocation there either fails or breaks the capture), in real-time loops
 * where cudaMalloc's implicit device synchronisation is not acceptable, or
 * under an external memory manager that owns every byte of device memory.
 * This call allocates nothing and frees nothing, and neither do its kernels.
 *
 * For a layer with hadamard_block != 0 this call runs the rotation as a
 * kernel of its own (eva_vq_linear_run fuses it into the lookup kernel) and
 * the rotated input x~ goes through scratch memory: one library-wide device
 * array of 4 MiB, `static __device__` in this library, so B * K * 4 must not
 * exceed 4 MiB (EVA_ERR_SCRATCH_TOO_SMALL otherwise).  Every GPU that loads
 * the library keeps those 4 MiB until the process exits.  Layers without a
 * rotation use no scratch at all.  Results are bitwise those of
 * eva_vq_linear_run: both rotations take the same butterflies in the same
 * order.
 *
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  The device that is current must be the
 * handle's.
 *
 * Sharing: every call on a device uses the same array and it keeps the last
 * call's contents (nothing in it needs to start at zero: the rotation writes
 * all of x~ before the lookups read it).  Two calls whose kernels overlap on
 * the GPU -- on different streams, or with different handles at the same
 * time -- race on the array; serialise them (one stream is enough).
 *
 * Arguments, layouts and results are those of eva_vq_linear_run.
 */
EVA_API eva_status_t eva_vq_linear_run_noalloc(eva_vq_linear_t h, const void *x, int32_t B, void *y,
                                               eva_stream_t stream);

/*
 * The same call with HOST buffers: copies x (host fp16 [B][K]) to the
 * handle's staging buffer, runs, copies y back to y_host ([B][N] of
 * out_dtype) and waits for `stream`.  With page-locked host buffers and x of
 * at most 64 KB the kernels read x and write y in the mapped host memory
 * directly (no copy operations); larger page-locked buffers go through one
 * CUDA graph (copy in, run, copy out), captured on the first call for each B
 * and replayed with its copy addresses updated; pageable memory works, one
 * operation at a time, and is slower.  A handle keeps its graphs until it is
 * destroyed.
 */
EVA_API eva_status_t eva_vq_linear_run_host(eva_vq_linear_t h, const void *x_host, int32_t B,
                                    void *y_host, eva_stream_t stream);

/* Free the handle's device memory.  The caller must have synchronised every
 * stream the handle ran on.  NULL is accepted. */
EVA_API eva_status_t eva_vq_linear_destroy(eva_vq_linear_t h);

/*
 * Test hook: decode the handle's repacked index stream with the same
 * position functions the lookup kernels use, writing canonical WI
 * [N][K/d] u8 to device memory `wi_out`.  Bit-exact inverse of create().
 */
EVA_API eva_status_t eva_vq_unpack_indices(eva_vq_linear_t h, uint8_t *wi_out, eva_stream_t stream);

/* Synchronises the device and reports a device-side error word set by a
 * kernel (EVA_ERR_DEVICE_TIMEOUT for a bounded wait that gave up).  The word
 * belongs to the handle and stays set once a wait has given up. */
EVA_API eva_status_t eva_vq_sync_status(eva_vq_linear_t h);

/*
 * Failure-detection test hook.  The only spin-wait of the kernels is the
 * bounded wait of a waiting call (eva_vq_linear_run, or run_ex without
 * EVA_RUN_INDEPENDENT) for the bulk copy that stages its first index units
 * in shared memory; when it gives up, the CTA sets the handle's status word,
 * still joins its cluster barriers and exits, and eva_vq_sync_status returns
 * EVA_ERR_DEVICE_TIMEOUT.  After this hook the next such call on `h` that
 * stages units issues neither that copy nor its arrival (so nothing is in
 * flight and the wait cannot complete) and gives up after `rounds` try_wait
 * rounds (1 .. 2^20; the regular limit is 2^20).  One-shot; y of that call
 * is undefined.  No device fault, trap or hang is involved.
 * EVA_ERR_INVALID_ARG for a null handle or rounds out of range.
 */
EVA_API eva_status_t eva_vq_debug_inject_wait_timeout(eva_vq_linear_t h, int32_t rounds);

/*
 * Diagnostic hook of the checked build (compiled with EVA_DEVICE_CHECKS):
 * synchronises the device and copies the handle's 8-word check record to
 * host memory out8: [0] number of rejected accesses, then for the first one
 * [1] source line, [2] buffer id, [3] block, [4] thread, [5..6] byte offset
 * (low, high), [7] access size.  In the regular build the record stays zero.
 */
EVA_API eva_status_t eva_vq_device_check_record(eva_vq_linear_t h, int32_t *out8);

/*
 * Diagnostic hook of the timeline build (compiled with EVA_TIMELINE):
 * synchronises the device and copies up to max_entries %globaltimer stamps
 * (ns) of the last lookup launch to host memory `out`, 8 per CTA: start,
 * after the dependency wait, codebook image started, image built, lookups
 * done, split-K handshake done, finalisation done (0 when a CTA skipped a
 * phase).  *count receives the number copied.  The regular build returns
 * EVA_ERR_UNSUPPORTED.
 */
EVA_API eva_status_t eva_vq_debug_timeline(eva_vq_linear_t h, uint64_t *out, int32_t max_entries,
                                           int32_t *count);

/* Static string for a status code. */
EVA_API const char *eva_vq_status_string(eva_status_t s);

typedef struct {
    int64_t stream_bytes;     /* algorithmic bytes per token-batch: WI + signs + alpha + x */
    int64_t wi_bytes, sign_bytes, alpha_bytes, codebook_bytes;
    int64_t workspace_bytes;  /* device memory owned by the handle beyond the weights */
    int32_t slices;           /* K-slices of 64 sub-vectors                             */
    int32_t row_tiles;        /* row tiles of 16 outputs                                */
    int32_t grid;             /* CTAs of the lookup kernel for the last run             */
    int32_t kernels_per_run;  /* kernel launches per run() for the last run            */
    int32_t path;             /* eva_path_t used by the last run                       */
    int32_t sm_count;
    int32_t staged_units;     /* index units per CTA a waiting one-token call copies into
                                 shared memory while it waits (0: none)                */
} eva_vq_info;

/* Sizes and launch shape of a handle (host only, no device work). */
EVA_API eva_status_t eva_vq_linear_info(eva_vq_linear_t h, eva_vq_info *info);

/* ------------------------------------------------------------------------
 * Offline quantizer: the quantize() sample of the 3-bit SRAM-lookup article
 * ("section details"), run on the GPU.  Steps, in the sample's order:
 *   1. W_rot = W Q, Q = blockdiag(H_b) diag(s) / sqrt(b) -- each row gets the
 *      transform the layer applies to x (hadamard_block = 0: W_rot = W);
 *   2. blocks of d = 4 along each row;
 *   3. K-means: plain Lloyd iterations (the sample's sensitivity weighting
 *      needs calibration data the pages do not give) from starting centroids
 *      the caller chooses as blocks of W_rot; the codebook is stored in fp16
 *      and the pointers are the nearest fp16 centroids;
 *   4.-7. residual r = W_rot - codebook[pointer], its 1-bit signs packed
 *      LSB-first along k (a zero residual counts as +1) and the optimal scale
 *      per group, alpha = mean |r| (fp16).
 * The outputs are exactly what eva_vq_linear_create takes (wc, wi, signs,
 * alpha, with the same hsign and hadamard_block).
 * ---------------------------------------------------------------------- */
typedef struct {
    int32_t N;               /* rows of W (output features), >= 1                      */
    int32_t K;               /* columns of W, multiple of 4 (of 8 with a residual)     */
    int32_t d;               /* block length; 4 is the only supported value            */
    int32_t index_bits;      /* 1..8: 2^index_bits centroids per codebook              */
    int32_t codebook_rows;   /* 0: one codebook; else rows per codebook (divides N)    */
    int32_t residual_group;  /* 0: no residual; else a multiple of 8 dividing K (128)  */
    int32_t hadamard_block;  /* 0: no rotation; else as in eva_vq_desc                 */
    int32_t iters;           /* Lloyd iterations, >= 0                                 */
} eva_quant_desc;

/*
 * Quantize W (device fp16 [N][K]).  hsign: device int8 [K] in {-1, +1}
 * (required iff hadamard_block != 0).  init_index: device int32 [G][2^n]:
 * codebook g's centroid c starts as block init_index[g][c] of the codebook's
 * blocks (block m of codebook g is W_rot row g * codebook_rows + m / (K/4),
 * inputs 4 (m mod K/4) ..; G = N / codebook_rows, or 1); an index out of
 * range gives EVA_ERR_INVALID_ARG.  Outputs (device, caller-owned): wc_out fp16
 * [G][2^n][4]; wi_out u8 [N][K/4] (index_bits = 4: packed two per byte,
 * [N][K/8] with the even sub-vector in the low nibble -- the layout
 * eva_vq_linear_create takes; K a multiple of 8); signs_out u8 [N][K/8] and alpha_out fp16
 * [N][K/residual_group] (required iff residual_group != 0).  Optional:
 * wrot_out fp32 [N][K] (the rotated rows; also used as the working buffer
 * when given) and cent_out fp32 [G][2^n][4] (the centroids after the last
 * iteration, before rounding to fp16).  Work buffers are allocated on
 * `stream` (stream-ordered) and freed before return; the call synchronises
 * `stream` before it returns.
 */
EVA_API eva_status_t eva_vq_quantize(const eva_quant_desc *desc, const void *w, const int8_t *hsign,
                                     const int32_t *init_index, void *wc_out, uint8_t *wi_out,
                                     uint8_t *signs_out, void *alpha_out, float *wrot_out, float *cent_out,
                                     eva_stream_t stream);

/*
 * The K-means steps on their own (asynchronous on `stream`).  v: device fp32
 * [M][d] (16-byte aligned), d = 4; centroids: device fp32 [G][ncent][d],
 * 1 <= ncent <= 256; block m belongs to codebook m / vecs_per_cb
 * (vecs_per_cb = 0: one codebook, G = 1).
 * assign: idx_out[m] = the nearest centroid, the squared distance summed in
 * fp32 one component at a time (no fused multiply-add), the first minimum
 * winning -- bit-exact with the decision rule the oracle states.
 */
EVA_API eva_status_t eva_vq_kmeans_assign(const float *v, int64_t M, int32_t d, const float *centroids,
                                          int32_t ncent, int64_t vecs_per_cb, int32_t *idx_out,
                                          eva_stream_t stream);

/*
 * update: new_out[g][c] = mean of the blocks assigned to c (double sums,
 * one rounding to fp32); a centroid with no block keeps old[g][c].  new_out
 * may equal old.  counts_out (optional) int64 [G][ncent].  Allocates its
 * sums on `stream` (stream-ordered) and frees them before returning.
 */
EVA_API eva_status_t eva_vq_kmeans_update(const float *v, int64_t M, int32_t d, const int32_t *idx,
                                          int32_t ncent, int64_t vecs_per_cb, const float *old,
                                          float *new_out, int64_t *counts_out, eva_stream_t stream);

/*
 * residual: for wrot (device fp32 [N][K]), wc (device fp16 [G][ncent][4]) and
 * wi (device u8 [N][K/4], row o using codebook o / codebook_rows): the packed
 * signs of r = wrot - wc[wi] (fp32, bit set for r >= 0, LSB-first, device u8
 * [N][K/8]) and alpha = mean |r| per group of `group` inputs (double sum,
 * rounded to fp16, device [N][K/group]).  group: a multiple of 8 dividing K.
 */
EVA_API eva_status_t eva_vq_residual(const float *wrot, int32_t N, int32_t K, const void *wc, int32_t ncent,
                                     const uint8_t *wi, int32_t codebook_rows, int32_t group,
                                     uint8_t *signs_out, void *alpha_out, eva_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* EVA_VQ_H */
