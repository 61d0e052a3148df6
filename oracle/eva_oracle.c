/*
 * eva_oracle.c -- plain, slow, double-precision reference for the decode-phase
 * linear layer with vector-quantized weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant with the
 * CUDA library.
 *
 * What it computes, and the passages it follows:
 *
 *  - EVA: Accelerating LLM Decoding via an Efficient Vector Quantization
 *    Architecture, technical summary section 2.A: the input is cut into
 *    sub-vectors of length d, a weight codebook WC holds 2^n centroids of
 *    length d, and the weight-index matrix WI names one centroid per
 *    (output row, sub-vector).  The layer output is therefore the ordinary
 *    matrix-vector product with the dequantised weight W[o][k] =
 *    WC[WI[o][k/d]][k mod d].  The method only reorders this sum (dot products
 *    of x with the codebook first, lookups second), so the oracle is the plain
 *    definition: dequantise one row, then a dot product in ascending k.
 *    (vq_oracle_linear)
 *
 *  - The same section's two steps written out literally: the output codebook
 *    OC[j][c] = <x_j, WC[c]> followed by y[o] = sum_j OC[j][WI[o][j]].  Used
 *    only to check the identity of the two forms.  (vq_oracle_lookup_form)
 *
 *  - Replacing MatMul with SRAM lookup: a 3-bit edge inference architecture,
 *    "section details" and its quantize() sample: a randomized Hadamard
 *    rotation applied along the input dimension, a 1-bit residual sign per
 *    weight and one fp16 scale alpha per group of 128.  Reading taken: the
 *    rotated weight is approximated by WC[WI] + alpha * sign, so inference
 *    multiplies it with the rotated input x~ = Q^T x, where
 *    Q = blockdiag(H_b) diag(s) / sqrt(b) (Sylvester H_b, b = the rotation
 *    block), i.e. x~ = s (.) (H_b x) / sqrt(b) per block.  The rotation is a
 *    dense per-block matrix product here, not a fast transform.
 *    (vq_oracle_hadamard)
 *
 *  - The same sample's "optimal scale per group": for a residual r and its
 *    signs, the alpha minimising ||r - alpha*sign(r)||^2 over a group.
 *    (vq_oracle_optimal_alpha)
 *
 *  - The same sample's quantize() pipeline, offline: rotate the weight rows
 *    (W_rot = W Q, the same per-block transform as x~, row by row), cut them
 *    into blocks of d, run K-means to get the codebook and the pointers,
 *    take the residual W_rot - codebook[pointers], its 1-bit signs and the
 *    optimal scale per group, and pack the signs into bytes.  Readings taken:
 *    plain Lloyd K-means (the sample's sensitivity weights need calibration
 *    data, which the pages do not give), started from centroids the caller
 *    passes in, for a given number of iterations, an empty cluster keeping
 *    its centroid; the nearest-centroid decision is made in fp32 (the
 *    precision the GPU kernel decides in), distances summed in component
 *    order, ties to the lower index; centroid means in double.
 *    (vq_oracle_kmeans_assign, vq_oracle_kmeans_update, vq_oracle_residual)
 *
 * Layouts are the canonical ones of the input generator:
 *   wc [G][2^n][d] fp16, wi [N][K/d] u8, signs [N][K/8] u8 LSB-first
 *   (bit set -> +1, clear -> -1), alpha [N][K/rg] fp16, hsign [K] int8,
 *   x [B][K] fp16.  fp16 values are decoded exactly into double.
 *
 * Every entry point returns 0 on success and a negative value on a bad
 * argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* IEEE binary16 -> double, exact (every binary16 value is a double). */
double vq_oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)mant, -24);                 /* subnormal: m * 2^-24 */
    else if (expo == 0x1f)
        v = mant ? NAN : INFINITY;
    else
        v = ldexp((double)(mant | 0x400), expo - 25); /* (1024+m) * 2^(e-25) */
    return sign ? -v : v;
}

void vq_oracle_f16_array_to_f64(const uint16_t *h, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = vq_oracle_f16_to_f64(h[i]);
}

static int popcount_u32(uint32_t v)
{
    int c = 0;
    while (v) { c += (int)(v & 1u); v >>= 1; }
    return c;
}

/* Sylvester Hadamard entry: (-1)^popcount(p & q). */
static double sylvester(int p, int q)
{
    return (popcount_u32((uint32_t)(p & q)) & 1) ? -1.0 : 1.0;
}

/*
 * Paley construction I of a Hadamard matrix of order 28 = 27 + 1, q = 27 = 3^3
 * (q = 3 mod 4).  Reading taken (the pages give none): GF(27) is GF(3)[t]
 * modulo t^3 + 2t + 2, element e = c0 + 3 c1 + 9 c2 is c0 + c1 t + c2 t^2;
 * chi is the quadratic character (chi(a) = a^13, chi(0) = 0); the Jacobsthal
 * matrix is Q[i][j] = chi(e_i - e_j); H28 = I + S with S = [0, 1^T; -1, Q].
 */
static int gf27_sub(int a, int b)
{
    int r = 0, w = 1;
    for (int i = 0; i < 3; ++i) {
        int d = ((a % 3) - (b % 3) + 3) % 3;
        r += d * w;
        w *= 3;
        a /= 3;
        b /= 3;
    }
    return r;
}

static int gf27_mul(int a, int b)
{
    int x[3], y[3], z[5] = {0, 0, 0, 0, 0};
    for (int i = 0; i < 3; ++i) { x[i] = a % 3; a /= 3; y[i] = b % 3; b /= 3; }
    for (int i = 0; i < 3; ++i)
        for (int j = 0; j < 3; ++j) z[i + j] = (z[i + j] + x[i] * y[j]) % 3;
    /* t^3 = t + 1 and t^4 = t^2 + t (mod 3, modulo t^3 + 2t + 2) */
    z[1] = (z[1] + z[3]) % 3; z[0] = (z[0] + z[3]) % 3;
    z[2] = (z[2] + z[4]) % 3; z[1] = (z[1] + z[4]) % 3;
    return z[0] + 3 * z[1] + 9 * z[2];
}

static int gf27_chi(int a)
{
    if (a == 0) return 0;
    int r = 1;
    for (int i = 0; i < 13; ++i) r = gf27_mul(r, a);
    return r == 1 ? 1 : -1;   /* a^13 is 1 or -1 (= element 2) */
}

static double paley28_entry(int i, int j)
{
    if (i == 0) return 1.0;
    if (j == 0) return -1.0;
    if (i == j) return 1.0;
    return (double)gf27_chi(gf27_sub(i - 1, j - 1));
}

/* The 784 entries, computed once (the character is slow to evaluate). */
static double paley28(int i, int j)
{
    static double tab[28][28];
    static int ready = 0;
    if (!ready) {
#ifdef _OPENMP
#pragma omp critical(vq_oracle_paley)
#endif
        {
            if (!ready) {
                for (int a = 0; a < 28; ++a)
                    for (int b = 0; b < 28; ++b) tab[a][b] = paley28_entry(a, b);
                ready = 1;
            }
        }
    }
    return tab[i][j];
}

static int is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

/* Rotation blocks: a power of two b (Sylvester H_b), or b = 28 m with m a
 * power of two (H_b = H28 (x) H_m, Kronecker, the order-28 factor outside). */
static int valid_block(int b) { return is_pow2(b) || (b % 28 == 0 && is_pow2(b / 28)); }

static double block_entry(int b, int p, int q)
{
    if (is_pow2(b)) return sylvester(p, q);
    const int m = b / 28;
    return paley28(p / m, q / m) * sylvester(p % m, q % m);
}

/*
 * x~ = s (.) (H_b^T x) / sqrt(b), block by block, for one token (H_b^T = H_b
 * for Sylvester blocks).  With Q = blockdiag(H_b) diag(s) / sqrt(b) this is
 * x~ = Q^T x, the partner of W_rot = W Q.  xin and xout are K doubles; b must
 * divide K (b = 0 copies x).
 */
static void rotate_token(const double *xin, const int8_t *hsign, int K, int b, double *xout)
{
    if (b <= 0) {
        memcpy(xout, xin, sizeof(double) * (size_t)K);
        return;
    }
    double inv = 1.0 / sqrt((double)b);
    for (int blk = 0; blk < K / b; ++blk) {
        const double *xb = xin + (size_t)blk * b;
        for (int p = 0; p < b; ++p) {
            double acc = 0.0;
            for (int q = 0; q < b; ++q)
                acc += block_entry(b, q, p) * xb[q];
            int k = blk * b + p;
            xout[k] = (double)hsign[k] * acc * inv;
        }
    }
}

/* The rotated input for B tokens.  x is fp16 [B][K], out double [B][K].
 * b = 0 returns x decoded unchanged. */
int vq_oracle_hadamard(const uint16_t *x, const int8_t *hsign, int B, int K, int b, double *out)
{
    if (!x || !out || B < 0 || K <= 0) return -1;
    if (b > 0 && (!hsign || K % b != 0 || !valid_block(b))) return -2;
    double *row = (double *)malloc(sizeof(double) * (size_t)K);
    if (!row) return -3;
    for (int t = 0; t < B; ++t) {
        vq_oracle_f16_array_to_f64(x + (size_t)t * K, K, row);
        rotate_token(row, hsign, K, b, out + (size_t)t * K);
    }
    free(row);
    return 0;
}

typedef struct {
    int N, K, d, ncent;          /* ncent <= 2^n centroids per codebook */
    int index_bits;              /* n: 8 (one byte per index) or 4 (two per byte) */
    int codebook_rows;           /* 0: one codebook; else rows per codebook */
    int residual_group;          /* 0: no residual */
    int hadamard_block;          /* 0: no rotation */
} vq_oracle_desc;

static int check_desc(const vq_oracle_desc *d)
{
    if (!d || d->N <= 0 || d->K <= 0 || d->d <= 0 || d->K % d->d) return -1;
    if (d->index_bits != 8 && d->index_bits != 4) return -1;
    if (d->ncent <= 0 || d->ncent > (1 << d->index_bits)) return -1;
    if (d->index_bits == 4 && (d->K / d->d) % 2) return -1;
    if (d->codebook_rows < 0 || (d->codebook_rows && d->N % d->codebook_rows)) return -1;
    if (d->residual_group < 0 || (d->residual_group && (d->K % d->residual_group || d->K % 8)))
        return -1;
    if (d->hadamard_block < 0 || (d->hadamard_block && d->K % d->hadamard_block)) return -1;
    return 0;
}

/* Index WI[o][j].  n = 8: byte j of row o ([N][K/d]).  n = 4: the indices are
 * packed two per byte ([N][K/(2d)]), sub-vector j in byte j/2, the even one in
 * the low nibble (LSB first, like the sign bits). */
static int index_of(const vq_oracle_desc *d, const uint8_t *wi, int o, int j)
{
    const int J = d->K / d->d;
    if (d->index_bits == 8) return wi[(size_t)o * (size_t)J + (size_t)j];
    const uint8_t byte = wi[(size_t)o * (size_t)(J / 2) + (size_t)(j / 2)];
    return (byte >> (4 * (j & 1))) & 15;
}

/* Codebook index of output row o. */
static int group_of_row(const vq_oracle_desc *d, int o)
{
    return d->codebook_rows ? o / d->codebook_rows : 0;
}

/* Residual sign of weight (o, k): bit k%8 of byte k/8 of row o, LSB-first. */
static double sign_of(const vq_oracle_desc *d, const uint8_t *signs, int o, int k)
{
    uint8_t byte = signs[(size_t)o * (size_t)(d->K / 8) + (size_t)(k / 8)];
    return ((byte >> (k % 8)) & 1) ? 1.0 : -1.0;
}

/* Dequantised row o of the weight, in double: WC[g][WI[o][k/d]][k mod d]
 * plus alpha[o][k/rg] * sigma[o][k] when the residual is present. */
static void dequant_row(const vq_oracle_desc *d, const uint16_t *wc, const uint8_t *wi,
                        const uint8_t *signs, const uint16_t *alpha, int o, double *wrow)
{
    int J = d->K / d->d;
    int g = group_of_row(d, o);
    const uint16_t *cb = wc + (size_t)g * (size_t)d->ncent * (size_t)d->d;
    for (int k = 0; k < d->K; ++k) {
        int c = index_of(d, wi, o, k / d->d);
        wrow[k] = vq_oracle_f16_to_f64(cb[(size_t)c * (size_t)d->d + (size_t)(k % d->d)]);
    }
    if (d->residual_group) {
        int ngroups = d->K / d->residual_group;
        for (int k = 0; k < d->K; ++k) {
            double a = vq_oracle_f16_to_f64(
                alpha[(size_t)o * (size_t)ngroups + (size_t)(k / d->residual_group)]);
            wrow[k] += a * sign_of(d, signs, o, k);
        }
    }
}

static int check_indices(const vq_oracle_desc *d, const uint8_t *wi)
{
    for (int o = 0; o < d->N; ++o)
        for (int j = 0; j < d->K / d->d; ++j)
            if (index_of(d, wi, o, j) >= d->ncent) return -4;
    return 0;
}

/*
 * y[B][N] (double) = dequantised W times the (rotated) input, row by row,
 * ascending k.  nthreads <= 0 means one thread; the threads split the output
 * rows and each row's sum is the same sequential loop, so the result does not
 * depend on the thread count.
 */
int vq_oracle_linear(const vq_oracle_desc *desc, const uint16_t *wc, const uint8_t *wi,
                     const uint8_t *signs, const uint16_t *alpha, const int8_t *hsign,
                     const uint16_t *x, int B, double *y, int nthreads)
{
    if (check_desc(desc) || !wc || !wi || !x || !y || B < 0) return -1;
    if (desc->residual_group && (!signs || !alpha)) return -2;
    if (desc->hadamard_block && !hsign) return -2;
    if (check_indices(desc, wi)) return -4;
    const int N = desc->N, K = desc->K;

    double *xt = (double *)malloc(sizeof(double) * (size_t)B * (size_t)K + 1);
    if (!xt) return -3;
    int rc = vq_oracle_hadamard(x, hsign, B, K, desc->hadamard_block, xt);
    if (rc) { free(xt); return rc; }

    int nt = nthreads > 0 ? nthreads : 1;
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(nt) reduction(|:failed)
#endif
    {
        double *wrow = (double *)malloc(sizeof(double) * (size_t)K);
        if (!wrow) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
            for (int o = 0; o < N; ++o) {
                dequant_row(desc, wc, wi, signs, alpha, o, wrow);
                for (int t = 0; t < B; ++t) {
                    const double *xv = xt + (size_t)t * K;
                    double acc = 0.0;
                    for (int k = 0; k < K; ++k)
                        acc += wrow[k] * xv[k];
                    y[(size_t)t * N + o] = acc;
                }
            }
            free(wrow);
        }
    }
    (void)nt;
    free(xt);
    return failed ? -3 : 0;
}

/*
 * The two-step form, written out: OC[g][t][j][c] = sum_{u<d} x~[t][d*j+u] *
 * WC[g][c][u], then y[t][o] = sum_j OC[g(o)][t][j][WI[o][j]] plus the sign
 * residual sum_q alpha[o][q] * sum_{k in group q} sigma[o][k] x~[t][k].
 * Also returns sum_k |W[o][k] x~[t][k]| per output in absy (may be NULL),
 * the scale for the identity check.  Small problems only: OC is G*B*J*2^n.
 */
int vq_oracle_lookup_form(const vq_oracle_desc *desc, const uint16_t *wc, const uint8_t *wi,
                          const uint8_t *signs, const uint16_t *alpha, const int8_t *hsign,
                          const uint16_t *x, int B, double *y, double *absy)
{
    if (check_desc(desc) || !wc || !wi || !x || !y || B < 0) return -1;
    if (desc->residual_group && (!signs || !alpha)) return -2;
    if (desc->hadamard_block && !hsign) return -2;
    if (check_indices(desc, wi)) return -4;
    const int N = desc->N, K = desc->K, dd = desc->d, nc = desc->ncent;
    const int J = K / dd;
    const int G = desc->codebook_rows ? N / desc->codebook_rows : 1;

    double *xt = (double *)malloc(sizeof(double) * (size_t)B * (size_t)K + 1);
    double *oc = (double *)malloc(sizeof(double) * (size_t)G * (size_t)B * (size_t)J * (size_t)nc + 1);
    double *wrow = (double *)malloc(sizeof(double) * (size_t)K + 1);
    if (!xt || !oc || !wrow) { free(xt); free(oc); free(wrow); return -3; }
    int rc = vq_oracle_hadamard(x, hsign, B, K, desc->hadamard_block, xt);
    if (rc) { free(xt); free(oc); free(wrow); return rc; }

    /* Step 1: output codebook, the dot product of every sub-vector with
     * every centroid. */
    for (int g = 0; g < G; ++g)
        for (int t = 0; t < B; ++t)
            for (int j = 0; j < J; ++j)
                for (int c = 0; c < nc; ++c) {
                    double acc = 0.0;
                    for (int u = 0; u < dd; ++u)
                        acc += xt[(size_t)t * K + (size_t)j * dd + u] *
                               vq_oracle_f16_to_f64(wc[((size_t)g * nc + c) * dd + u]);
                    oc[(((size_t)g * B + t) * J + j) * nc + c] = acc;
                }

    /* Step 2: gather through WI and accumulate over j. */
    for (int o = 0; o < N; ++o) {
        int g = desc->codebook_rows ? o / desc->codebook_rows : 0;
        if (absy) dequant_row(desc, wc, wi, signs, alpha, o, wrow);
        for (int t = 0; t < B; ++t) {
            double acc = 0.0;
            for (int j = 0; j < J; ++j) {
                int c = index_of(desc, wi, o, j);
                acc += oc[(((size_t)g * B + t) * J + j) * nc + c];
            }
            if (desc->residual_group) {
                int rg = desc->residual_group;
                for (int q = 0; q < K / rg; ++q) {
                    double s = 0.0;
                    for (int k = q * rg; k < (q + 1) * rg; ++k)
                        s += sign_of(desc, signs, o, k) * xt[(size_t)t * K + k];
                    acc += vq_oracle_f16_to_f64(alpha[(size_t)o * (K / rg) + q]) * s;
                }
            }
            y[(size_t)t * N + o] = acc;
            if (absy) {
                double a = 0.0;
                for (int k = 0; k < K; ++k)
                    a += fabs(wrow[k] * xt[(size_t)t * K + k]);
                absy[(size_t)t * N + o] = a;
            }
        }
    }
    free(xt); free(oc); free(wrow);
    return 0;
}

/*
 * Optimal residual scale per group: for each row and each group of `group`
 * consecutive entries of r, the alpha minimising sum (r - alpha * s)^2 with
 * s = sign(r) (zero mapped to +1).  Setting the derivative to zero gives
 * alpha = sum(r*s) / sum(s*s) = mean |r| over the group.
 * r is double [rows][cols], alpha_out double [rows][cols/group].
 */
int vq_oracle_optimal_alpha(const double *r, int rows, int cols, int group, double *alpha_out)
{
    if (!r || !alpha_out || rows <= 0 || cols <= 0 || group <= 0 || cols % group) return -1;
    for (int i = 0; i < rows; ++i)
        for (int q = 0; q < cols / group; ++q) {
            double num = 0.0, den = 0.0;
            for (int k = q * group; k < (q + 1) * group; ++k) {
                double v = r[(size_t)i * cols + k];
                double s = v >= 0.0 ? 1.0 : -1.0;
                num += v * s;
                den += s * s;
            }
            alpha_out[(size_t)i * (cols / group) + q] = num / den;
        }
    return 0;
}

/*
 * K-means assignment: for each of the M vectors of length d (fp32, [M][d]),
 * the index of the nearest of the ncent centroids of its codebook (fp32,
 * [G][ncent][d]); vector m uses codebook m / vecs_per_cb (0: one codebook).
 * The squared distance is accumulated in float, one component at a time in
 * order (each difference, square and sum rounded to float); the first
 * minimum wins.  Compiled without floating-point contraction.
 */
int vq_oracle_kmeans_assign(const float *v, int64_t M, int d, const float *cent, int ncent,
                            int64_t vecs_per_cb, int32_t *idx_out)
{
    if (!v || !cent || !idx_out || M < 0 || d <= 0 || ncent <= 0 || vecs_per_cb < 0) return -1;
    for (int64_t m = 0; m < M; ++m) {
        const int64_t g = vecs_per_cb ? m / vecs_per_cb : 0;
        const float *cb = cent + (size_t)g * ncent * d;
        int best = 0;
        float best_d = 0.f;
        for (int c = 0; c < ncent; ++c) {
            float dist = 0.f;
            for (int t = 0; t < d; ++t) {
                const float diff = v[(size_t)m * d + t] - cb[(size_t)c * d + t];
                const float sq = diff * diff;
                dist = dist + sq;
            }
            if (c == 0 || dist < best_d) {
                best = c;
                best_d = dist;
            }
        }
        idx_out[m] = best;
    }
    return 0;
}

/*
 * K-means update: centroid c of codebook g becomes the mean (in double,
 * rounded once to float) of the vectors assigned to it; a centroid with no
 * vector keeps its old value.  counts_out[g][c] (optional) receives the
 * cluster sizes.
 */
int vq_oracle_kmeans_update(const float *v, int64_t M, int d, const int32_t *idx, int ncent,
                            int64_t vecs_per_cb, const float *old_cent, float *new_cent,
                            int64_t *counts_out)
{
    if (!v || !idx || !old_cent || !new_cent || M < 0 || d <= 0 || ncent <= 0 || vecs_per_cb < 0)
        return -1;
    const int64_t G = vecs_per_cb ? (M + vecs_per_cb - 1) / vecs_per_cb : 1;
    double *sum = calloc((size_t)G * ncent * d, sizeof(double));
    int64_t *cnt = calloc((size_t)G * ncent, sizeof(int64_t));
    if (!sum || !cnt) { free(sum); free(cnt); return -2; }
    for (int64_t m = 0; m < M; ++m) {
        const int64_t g = vecs_per_cb ? m / vecs_per_cb : 0;
        const int c = idx[m];
        if (c < 0 || c >= ncent) { free(sum); free(cnt); return -1; }
        cnt[g * ncent + c] += 1;
        for (int t = 0; t < d; ++t) sum[((size_t)g * ncent + c) * d + t] += (double)v[(size_t)m * d + t];
    }
    for (int64_t gc = 0; gc < G * ncent; ++gc) {
        for (int t = 0; t < d; ++t)
            new_cent[(size_t)gc * d + t] = cnt[gc] ? (float)(sum[(size_t)gc * d + t] / (double)cnt[gc])
                                                   : old_cent[(size_t)gc * d + t];
        if (counts_out) counts_out[gc] = cnt[gc];
    }
    free(sum); free(cnt);
    return 0;
}

/*
 * Residual, signs and scales of a quantized rotated weight.  wrot: fp32
 * [N][K]; wc: fp16 [G][ncent][d]; wi: u8 [N][K/d]; row o uses codebook
 * o / codebook_rows (0: one codebook).  The residual is
 * r = wrot - codebook[pointer] evaluated in float (one rounding); its sign
 * bit is set for r >= 0 (a zero residual counts as +1) and stored LSB-first
 * along k (bit i of byte m is k = 8m + i, signs_out [N][K/8]).  alpha_out
 * [N][K/group] (double) is the optimal scale of each group of `group`
 * consecutive k: mean |r|, summed in double.
 */
int vq_oracle_residual(const float *wrot, int N, int K, int d, const uint16_t *wc, int ncent,
                       const uint8_t *wi, int codebook_rows, int group, uint8_t *signs_out,
                       double *alpha_out)
{
    if (!wrot || !wc || !wi || !signs_out || !alpha_out || N <= 0 || K <= 0 || d <= 0 || K % d ||
        K % 8 || group <= 0 || K % group || (codebook_rows && N % codebook_rows))
        return -1;
    const int J = K / d;
    memset(signs_out, 0, (size_t)N * (K / 8));
    for (int o = 0; o < N; ++o) {
        const int g = codebook_rows ? o / codebook_rows : 0;
        for (int q = 0; q < K / group; ++q) {
            double acc = 0.0;
            for (int k = q * group; k < (q + 1) * group; ++k) {
                const int c = wi[(size_t)o * J + k / d];
                if (c >= ncent) return -1;
                const float cv = (float)vq_oracle_f16_to_f64(wc[((size_t)g * ncent + c) * d + k % d]);
                const float r = wrot[(size_t)o * K + k] - cv;
                if (r >= 0.f) signs_out[(size_t)o * (K / 8) + k / 8] |= (uint8_t)(1u << (k % 8));
                acc += fabs((double)r);
            }
            alpha_out[(size_t)o * (K / group) + q] = acc / (double)group;
        }
    }
    return 0;
}

int vq_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
