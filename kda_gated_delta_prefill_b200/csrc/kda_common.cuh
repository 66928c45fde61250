// kda_common.cuh -- sizes shared by the KDA kernels.
#pragma once

namespace kda {

constexpr int CH = 64;   // chunk length (tokens); the page's golden chunk size
constexpr int DK = 128;  // key / query head dim
constexpr int DV = 128;  // value head dim

// Per-(chunk, value head) block handed from the intra-chunk kernel to the
// carry kernel, laid out exactly as the carry kernel's shared-memory stage.
// "SW128" = rows of 128 bytes in 1024-byte atoms of 8 rows whose 16-byte
// chunks are XOR-swizzled by row % 8; a 128-column fp16 matrix is two such
// 64-column halves 8192 bytes apart.
constexpr int ITEM_WN = 0;        // fp16 [64 tok][128 key] SW128: -W (B operand, K-major)
constexpr int ITEM_QG = 16384;    // fp16 [64 tok][128 key] SW128: K^-0.5 q exp(G) (B operand, K-major)
constexpr int ITEM_KG = 32768;    // fp16 [64 tok][128 key] SW128: k exp(G_last - G) (B operand, MN-major)
constexpr int ITEM_AQK = 49152;   // fp16 [64 i][64 j] SW128: causal Aqk (B operand, K-major)
constexpr int ITEM_U = 57344;     // fp16 [128 value][64 tok] SW128: U^T = (A v)^T
constexpr int ITEM_GL = 73728;    // fp32 [128]: exp(G_last)
constexpr int ITEM_BYTES = 74240;

}  // namespace kda
