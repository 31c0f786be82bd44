// The chunk record: everything the state scan needs about one chunk of one
// (segment, head) that does not depend on the state, written by the chunk
// preparation kernel and read by the scan with two bulk copies.
//
// Page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit
// festem Zustand": prefill evaluates a chunk's tokens in parallel and hands a
// state from chunk to chunk.  Over a chunk of C = 64 tokens with cumulative
// gate Gamma_i = sum_{s<=i} g'_s (per key channel, g' = max(g, -5)), with y_q,
// y_k the short-conv outputs of q and k before normalisation, r^q_t, r^k_t the
// reciprocal norms (q_hat = r^q y_q, k_hat = r^k y_k) and Dq, Dk the diagonal
// matrices of those reciprocals, the step of the recurrence S_t = Diag(alpha_t)
// S_{t-1} + k_t u_t^T, u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t) sums to
//     m_ij = sum_c y^k_ic y^k_jc e^{Gamma_ic - Gamma_jc} (i > j),  p_ij likewise with y^q_i (j <= i)
//     T    = (I + diag(beta) Dk m Dk)^-1 diag(beta)
//     U'   = Dk U = (Dk T) V - W' S,     W' = (Dk T Dk) (e^Gamma * Y_k)
//     O    = Dq ((e^Gamma * Y_q) S + p U')
//     S   <- diag(e^{Gamma_C}) S + (e^{Gamma_C - Gamma} * Y_k)^T U'
// so that the normalisations act on 64-element vectors and 64 x 64 matrices
// only.  (With r = 1 and the normalised q_hat, k_hat in place of y_q, y_k the
// same record holds the plainly normalised form.)
//
// Layout (REC_BYTES per chunk-head; all tiles fp32 values rounded to tf32,
// K-major, 128-byte swizzled, see kda_tc.cuh), p = the chunk's index within
// its segment mod 2:
//   RA [128][128 k]  -W' and Q~' = e^Gamma y_q stacked by rows: -W' in rows
//                    0..63 when p == 0, Q~' there when p == 1, so that one
//                    N = 128 product writes U'^T next to the output buffer of
//                    the chunk's parity
//   TS [64 t][64 s]  Dk T strictly below the diagonal
//   B2 [192][64 s]   p strictly below the diagonal (64 rows) and
//                    K-bar'^T = (e^{Gamma_C - Gamma} y_k)^T (128 rows, key k),
//                    P first when p == 0, K-bar'^T first when p == 1, so that
//                    one N = 192 product adds U'^T p^T to the output buffer and
//                    U'^T K-bar' to the next state buffer
//   SC fp32 b[64] = r^k_t beta_t (the diagonal of Dk T), d[64] = p_tt (the
//      diagonal of p, exact fp32), r[64] = r^q_t, gamma[128] = e^{Gamma_C}
// The diagonal terms b_t v_t and d_t u'_t carry the largest single-token
// contributions and are applied in fp32 by the scan.
#pragma once
#include <stdint.h>

namespace kda {

constexpr int CH = 64;  // chunk length
// raw input tiles of one head: 3 halo rows + 64 chunk rows of 128 bf16 (256 B)
constexpr int RAW_ROWS = CH + 3;
constexpr uint32_t RAW_BYTES = RAW_ROWS * 128 * 2;  // 17152

constexpr uint32_t REC_RA = 0;          // 4 slabs x (128 rows x 128 B)
constexpr uint32_t REC_TS = 65536;      // 2 slabs x (64 rows x 128 B)
constexpr uint32_t REC_B2 = 81920;      // 2 slabs x (192 rows x 128 B)
constexpr uint32_t REC_SC = 131072;     // 320 floats
constexpr uint32_t REC_BYTES = 132352;  // a multiple of 128: records start on cache lines
constexpr uint32_t REC_PIECE_A = REC_B2;              // RA + TS: read by the first product group
constexpr uint32_t REC_PIECE_B = REC_BYTES - REC_B2;  // B2 + SC: the second product group, scalars
constexpr int SC_B = 0, SC_D = 64, SC_R = 128, SC_G = 192;
constexpr int B2_ROWS = 192;
static_assert(REC_BYTES % 128 == 0 && REC_PIECE_A % 1024 == 0 && REC_PIECE_B % 16 == 0, "record layout");

// first row of each block by chunk parity
__host__ __device__ constexpr int ra_w_row(int parity) { return parity ? 64 : 0; }
__host__ __device__ constexpr int ra_q_row(int parity) { return parity ? 0 : 64; }
__host__ __device__ constexpr int b2_p_row(int parity) { return parity ? 128 : 0; }
__host__ __device__ constexpr int b2_k_row(int parity) { return parity ? 0 : 64; }

}  // namespace kda
