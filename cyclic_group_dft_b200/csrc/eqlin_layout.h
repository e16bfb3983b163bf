// eqlin_layout.h -- data layout of the frequency-domain weights shared by the
// weight pre-transform kernel (writer) and the fused forward kernels (readers).
//
// Frequency components ("planes") of a real length-G signal, G even:
//   plane 0 = Re X_0,  plane 1 = Re X_{G/2},  plane 2k = Re X_k,  plane 2k+1 = Im X_k
// for 0 < k < G/2, with X_k = sum_m v_m exp(-2 pi i m k / G).  The stored weight
// planes carry the inverse-DFT scale: 1/G on planes 0 and 1, 2/G on the complex
// planes (the conjugate partner k' = G-k is folded into the factor 2).
//
// fp32 planes (always built; used by the fp32 path and for inspection):
//   w_f32[p][i][o], p < G, i < Cin, o < Cout  (output channel fastest)
//
// bf16 tensor-core image (bf16 I/O only): the exact shared-memory image the UMMA
// A operand reads, so a plain bulk copy stages it:
//   [oc][c][p][r][32]  with oc < n_oc (128-row output chunks), c < nK (32-channel
//   chunks of Cin, zero padded), p < G, r < rows (output rows of the chunk, zero
//   padded), 32 bf16 = one 64-byte row, K-major, SWIZZLE_64B: the 16-byte piece j
//   of row r is stored at piece j ^ ((r >> 1) & 3).
#pragma once

#include <cstddef>
#include <cstdint>

namespace eqlin {

constexpr int kChunkK = 32;          // input channels per K chunk
constexpr int kPlaneRowBytes = 64;   // one K chunk of one row in bf16
constexpr int kMmaM = 128;           // UMMA M (output rows per chunk)

// device status word values (mirrors EQLIN_ERR_TIMEOUT in eqlin.h)
constexpr int kDeviceErrTimeout = -6;

// byte offset of element (row r, column col) of sub-block `sub` (each sub-block
// holds `rows` rows of 64 bytes)
__host__ __device__ inline size_t image_offset(size_t sub, int rows, int r, int col) {
    const int piece = (col >> 3) ^ ((r >> 1) & 3);
    return sub * static_cast<size_t>(rows) * kPlaneRowBytes + static_cast<size_t>(r) * kPlaneRowBytes +
           static_cast<size_t>(piece) * 16 + static_cast<size_t>(col & 7) * 2;
}

// Slot layout of an MMA operand that pairs the products of a complex frequency.  The
// slots are: plane 0, plane 1, then for each complex frequency k the three slots
// [-Im V_k, Re V_k, Im V_k].  They are stored back to back, so [Re V_k; Im V_k] and
// [-Im V_k; Re V_k] are each one operand of twice the slot's rows, and a complex product
// (a + ib)(c + id) takes two MMAs that write the Re and Im planes of D side by side:
//   [D_re | D_im] += a [c; d],   [D_re | D_im] += b [-d; c].
// The tokens-on-N kernels use it for X^.
__host__ __device__ constexpr int pair_slots(int G) { return 2 + 3 * (G / 2 - 1); }
// first slot of complex frequency k (0 < k < G/2): the -Im slot
__host__ __device__ constexpr int pair_first_slot(int k) { return 2 + 3 * (k - 1); }
// frequency plane held by slot s, and its sign
__host__ __device__ inline int pair_slot_plane(int s, float* sign) {
    *sign = 1.0f;
    if (s < 2) return s;
    const int k = (s - 2) / 3 + 1, j = (s - 2) % 3;
    if (j == 0) *sign = -1.0f;
    return j == 1 ? 2 * k : 2 * k + 1;
}

// Tokens-on-M kernel variant: 16-channel K chunks, rows of 32 bytes, SWIZZLE_32B
// (16-byte piece j of row r stored at piece j ^ ((r >> 2) & 1)).  Image layout
// [oc][c][s][r < rows][16] over the weight slots s:
//  - G <= 8: the G planes of W^ in plane order (Re and Im of a complex frequency adjacent,
//    so [Re W_k | Im W_k] is one operand of twice the rows; the -Im W_k factor of a
//    complex product comes from the MMA's negate-B bit, one more MMA per frequency);
//  - G = 16: the pair slots above, so each complex product is two MMAs.
// B200: p8 C64 19.3 us with plane order (a fourth ring stage fits) against 19.6 us;
// C16 C32 112.5 us with plane order against 110.6 us.
__host__ __device__ constexpr bool tm_pair_slots(int G) { return G > 8; }
__host__ __device__ constexpr int tm_weight_slots(int G) { return tm_pair_slots(G) ? pair_slots(G) : G; }
constexpr int kChunkK16 = 16;
constexpr int kRowBytes32 = 32;
__host__ __device__ inline size_t image_offset_k16(size_t sub, int rows, int r, int col) {
    const int piece = (col >> 3) ^ ((r >> 2) & 1);
    return sub * static_cast<size_t>(rows) * kRowBytes32 + static_cast<size_t>(r) * kRowBytes32 +
           static_cast<size_t>(piece) * 16 + static_cast<size_t>(col & 7) * 2;
}

}  // namespace eqlin
