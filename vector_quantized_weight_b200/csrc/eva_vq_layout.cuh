// eva_vq_layout.cuh -- data layout of the repacked weights and the shared-memory
// output-codebook image, shared by the create-time repack, the unpack test hook
// and the lookup kernels; at the end, the dequantize kernel's lane order of
// sub-vectors and residual sign units.
//
// Work unit: one tile of 16 output rows (the M of one tensor-core MMA) times one
// K-slice of 64 sub-vectors (256 inputs).  A unit holds 1024 index bytes.
//
// Output-codebook (OC) image in shared memory: 256 centroid rows of 256 bytes
// (64 32-bit words).  The bank of a word depends only on its column, never on
// the centroid, so 32 lanes reading 32 distinct columns never collide whatever
// indices they look up -- the conflict-free lookup of the EVA summary, section
// 2.A ("rows derived from different input vectors map to different banks").
//   one token  (j-paired):   word(c, w) = half2(OC[w][c], OC[w+32][c]), w < 32
//   two tokens (token-paired): word(c, j) = half2(OC_a[j][c], OC_b[j][c]), j < 64
//
// The lookup for lane L = 4g + q (g = L/4, q = L%4) at k-step s8 reads column
// w = (L + 4 s8) mod 32.  Per k-step the lane supplies the four A registers of
// an m16n8k16 MMA: a0 -> row g, a1 -> row g+8 (sub-vector w), a2 -> row g,
// a3 -> row g+8 (sub-vector w + 32).  Over the 8 k-steps row g sees each of
// the 64 sub-vectors exactly once.
#pragma once
#include <stdint.h>

namespace eva {

constexpr int kD = 4;             // sub-vector length d
constexpr int kCent = 256;        // 2^n centroids, n = 8
constexpr int kSliceJ = 64;       // sub-vectors per K-slice
constexpr int kSliceK = kSliceJ * kD;   // 256 inputs per K-slice
constexpr int kTileRows = 16;     // output rows per unit
constexpr int kUnitBytes = kSliceJ * kTileRows;      // 1024 index bytes
constexpr int kSignUnitBytes = kTileRows * kSliceK / 8;  // 512 sign bytes
constexpr int kAlphaUnitHalves = kTileRows * 2;     // 2 groups of 128 per slice
constexpr int kOcRowBytes = 256;
constexpr int kOcBytes = kCent * kOcRowBytes;       // 64 KB image

// OC column read by lane `lane` at k-step `s8`.
__host__ __device__ __forceinline__ int oc_col(int lane, int s8) { return (lane + 4 * s8) & 31; }

// Index byte `b` of a unit (0..1023) -> (row in tile, sub-vector in slice).
// Byte b = 512*h + 16*lane + 4*(s8 - 4h) + r: the first 16 bytes of all 32
// lanes (k-steps 0..3) come first, then the second 16 (k-steps 4..7), so each
// 128-bit load of a warp reads 512 contiguous bytes (coalesced in global
// memory, bank-conflict-free in shared memory).  r selects the A register a_r.
__host__ __device__ __forceinline__ void wi_unit_pos(int b, int &row, int &jl) {
    const int h = b >> 9, lane = (b >> 4) & 31, s8 = 4 * h + ((b >> 2) & 3), r = b & 3;
    row = (lane >> 2) + ((r & 1) ? 8 : 0);
    jl = oc_col(lane, s8) + ((r & 2) ? 32 : 0);
}

// 4-bit indices (16 centroids): a unit is 512 bytes, 16 per lane; lane L's
// word u (0..3) holds k-steps 2u and 2u + 1, nibble 4 (s8 & 1) + r of the
// word being register r of k-step s8.  Nibble n = 32 L + 8 u + e of the unit
// -> (row in tile, sub-vector in slice), with the same (lane, s8, r) meaning
// as the byte layout.
constexpr int kUnitBytes4 = kUnitBytes / 2;

__host__ __device__ __forceinline__ void wi4_unit_pos(int n, int &row, int &jl) {
    const int lane = n >> 5, u = (n >> 3) & 3, e = n & 7;
    const int s8 = 2 * u + (e >> 2), r = e & 3;
    row = (lane >> 2) + ((r & 1) ? 8 : 0);
    jl = oc_col(lane, s8) + ((r & 2) ? 32 : 0);
}

// Inverse of wi4_unit_pos: the nibble of (row in tile, sub-vector in slice).
__host__ __device__ __forceinline__ int wi4_unit_nibble(int row, int jl) {
    const int r = ((row >= 8) ? 1 : 0) | ((jl >= 32) ? 2 : 0);
    const int g = row & 7, w = jl & 31, q = w & 3;
    const int s8 = (((w - q) >> 2) - g) & 7;
    const int lane = 4 * g + q;
    return 32 * lane + 8 * (s8 >> 1) + 4 * (s8 & 1) + r;
}

// Sign position read by lane (g, q) in residual MMA i (0..3), register r.
// Lanes q = 0,1 cover the first 128-input group of the slice (positions
// 0..15), lanes q = 2,3 the second (16..31); per register the 32 lanes read
// 32 distinct positions, i.e. 32 distinct banks.
__host__ __device__ __forceinline__ int sign_pos(int lane, int i, int r) {
    const int g = lane >> 2, q = lane & 3;
    const int st = 2 * i + (r >> 1);
    return 16 * (q >> 1) + ((2 * g + (q & 1) + 2 * st) & 15);
}

// Sign byte `b` of a unit (0..511) -> (row in tile, sign-byte position in slice).
// Byte b = 16*lane + 4*i + r.
__host__ __device__ __forceinline__ void sign_unit_pos(int b, int &row, int &m) {
    const int lane = b >> 4, i = (b >> 2) & 3, r = b & 3;
    row = (lane >> 2) + ((r & 1) ? 8 : 0);
    m = sign_pos(lane, i, r);
}

// Alpha half `e` of a unit (0..31) -> (row in tile, group in slice).
// Lane g (q = 0) reads halves 4g..4g+3: (row g: grp 0, 1), (row g+8: grp 0, 1).
__host__ __device__ __forceinline__ void alpha_unit_pos(int e, int &row, int &grp) {
    const int g = e >> 2;
    row = g + (((e >> 1) & 1) ? 8 : 0);
    grp = e & 1;
}

// ------------------------------------------------ dequantize-path layouts
//
// Sub-vector (within the slice) that lane quarter q reads in MMA block beta of
// the dequantize kernel (16 inputs = 4 sub-vectors per block).
__host__ __device__ __forceinline__ int dq_subvec(int beta, int q) {
    return beta < 8 ? 4 * beta + q : 4 * (beta - 8) + q + 32;
}

// Sign units of the residual on the dequantize path (one per slice and row
// tile, like the index units): 512 bytes, 16 per lane, so that one 128-bit
// read gives lane (g, q) every sign bit it multiplies.  Word w of lane
// L = 4 g + q: row g + 8 (w >> 1) of the tile; nibble n of the word: MMA block
// beta = 8 (w & 1) + n, whose bit e is the sign of slice input
// 4 dq_subvec(beta, q) + e (set: + alpha).
constexpr int kDqSignUnitBytes = 512;
constexpr int kDqResidUnitBytes = kDqSignUnitBytes + kAlphaUnitHalves * 2;   // + the lookup's alpha unit

// Bit t of sign byte b of a unit -> (row in tile, slice input).
__host__ __device__ __forceinline__ void dq_sign_pos(int b, int t, int &row, int &kin) {
    const int lane = b >> 4, w = (b >> 2) & 3, n = 2 * (b & 3) + (t >> 2);
    const int g = lane >> 2, q = lane & 3, beta = 8 * (w & 1) + n;
    row = g + 8 * (w >> 1);
    kin = 4 * dq_subvec(beta, q) + (t & 3);
}

}  // namespace eva
