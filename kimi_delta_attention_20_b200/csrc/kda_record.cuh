// Layout of the per-(chunk, head) record that pass 1 of the two-pass chunk
// forward writes and pass 2 (and the chunked backward) read.
#pragma once

#include <stdint.h>

namespace kda {
namespace tp {

// ---- record of one (chunk, head), bytes; every tile is a shared-memory image
// with the 128-byte swizzle (16-byte chunk index XOR row % 8, rows of 128 B)
// Pass 2 reads [Qtil^T | -W^T] as one N = 128 operand and [Khat^T ; A_qk] as one
// N = 192 operand, so those tiles are adjacent.
constexpr uint32_t R_QT = 0;        // Qtil^T [128 c][64 r]: B of S^T Qtil^T, N = r contiguous (MN-major)
constexpr uint32_t R_WT = 16384;    // -W^T   [128 c][64 r]: B of S^T (-W^T), MN-major
constexpr uint32_t R_KH = 32768;    // Khat^T [128 c][64 s]: B of D~^T Khat, K = s contiguous (K-major)
constexpr uint32_t R_AQK = 49152;   // A_qk (raw rows) [64 r][64 s], K-major B
constexpr uint32_t R_TPU = 57344;   // T' = T diag(beta) [64 r][64 s], K-major B
static_assert(R_WT - R_QT == 16384 && R_AQK == R_KH + 16384, "operand groups of pass 2 are adjacent");
constexpr uint32_t R_MISC = 65536;  // f32: e^{G_last}[128], 1/|q_r|[64], 1/|k_s|[64]
constexpr uint32_t R_GAM = R_MISC, R_INVQ = R_MISC + 512, R_INVK = R_MISC + 768;
constexpr uint32_t REC_BYTES = R_MISC + 1024;
static_assert(REC_BYTES % 1024 == 0, "records stay 1024-byte aligned");

// ---- backward record of one (chunk, head), bytes: what the chunked backward keeps
// from the forward's state pass and from its own cotangent pass, as the bf16 tile
// images (128-byte swizzle, 64-column halves) those passes build for their products.
constexpr uint32_t BR_S0 = 0;       // S^T entering the chunk [128 v][128 k]
constexpr uint32_t BR_DL = 32768;   // D~^T = (diag(1/|k_s|) D)^T [128 v][64 s], D = U - W S
constexpr uint32_t BR_DS = 49152;   // dS^T, the cotangent of the state leaving the chunk [128 v][128 k]
constexpr uint32_t BR_DD = 81920;   // dD^T, the cotangent of D [128 v][64 s]
constexpr uint32_t BR_BYTES = 98304;

}  // namespace tp
}  // namespace kda
