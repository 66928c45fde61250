// kda_common.cuh -- sizes shared by the KDA kernels.
#pragma once

namespace kda {

constexpr int CH = 64;   // chunk length (tokens); the page's golden chunk size
constexpr int DK = 128;  // key / query head dim
constexpr int DV = 128;  // value head dim

// Per-(chunk, value head) block handed from the intra-chunk kernel to the
// carry kernel, laid out exactly as the carry kernel's shared-memory stage.
constexpr int ITEM_WN = 0;        // fp16 [64 tok][128 key]: -W, rows of 256 bytes, 16-byte chunks swizzled
constexpr int ITEM_QG = 16384;    // fp16 [64][128]: K^-0.5 q exp(G), same layout
constexpr int ITEM_KG = 32768;    // fp16 [64][128]: k exp(G_last - G), same layout
constexpr int ITEM_AQK = 49152;   // fp16 [64][64]: causal Aqk, rows of 128 bytes, swizzled
constexpr int ITEM_U = 57344;     // fp16 [4 column quarters][64 tok][32]: U = A v, plain rows
constexpr int ITEM_GL = 73728;    // fp32 [128]: exp(G_last)
constexpr int ITEM_BYTES = 74240;

}  // namespace kda
