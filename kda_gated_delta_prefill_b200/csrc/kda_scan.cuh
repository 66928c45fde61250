// kda_scan.cuh -- composition of per-segment affine state maps for the
// segmented carry ("KDA Chunk Prefill on Ascend A3", section "Mathematical
// definition", last formula: the chunk update of S is affine in S, so a run
// of chunks maps its start state S to M S + B).
//
// With M_p the linear map of segment p (the carry from the identity with U
// taken as zero) and B_p its image of zero, the start states follow
//   S_{p+1} = M_p S_p + B_p,   p = 1 .. seg_count - 2,
// given S_1 (the end of segment 0, carried from the real initial state).
// Every state is fp32 [K][V]; the V columns are independent, so a CTA owns
// 16 columns of one (sequence, value head) unit and walks the segments.
#pragma once
#include "kda_common.cuh"

namespace kda {

constexpr int kScanCols = 16;                // V columns per CTA
constexpr int kScanCtasPerUnit = DV / kScanCols;

// grid: units * kScanCtasPerUnit, block: 256 threads (thread = row r, 8-column half)
__global__ void __launch_bounds__(256) kda_seg_scan_kernel(float *seg_S, const float *seg_M, const float *seg_B,
                                                           int seg_count)
{
    __shared__ float cur[DK][kScanCols];
    const int unit = blockIdx.x / kScanCtasPerUnit, col0 = (blockIdx.x % kScanCtasPerUnit) * kScanCols;
    const int r = threadIdx.x >> 1, c0 = (threadIdx.x & 1) * 8;
    const int64_t unit_off = static_cast<int64_t>(unit) * seg_count * DK * DV;

    // S_1
    const float *s1 = seg_S + unit_off + static_cast<int64_t>(1) * DK * DV + r * DV + col0 + c0;
#pragma unroll
    for (int c = 0; c < 8; ++c) cur[r][c0 + c] = s1[c];
    __syncthreads();

    for (int sp = 1; sp + 1 < seg_count; ++sp) {
        const int64_t off = unit_off + static_cast<int64_t>(sp) * DK * DV;
        const float *m = seg_M + off + r * DK;                   // row r of M_p
        const float *b = seg_B + off + r * DV + col0 + c0;       // B_p[r][cols]
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = b[c];
        for (int k4 = 0; k4 < DK; k4 += 4) {
            const float4 mv = *reinterpret_cast<const float4 *>(m + k4);
            const float mk[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = __fmaf_rn(mk[kk], cur[k4 + kk][c0 + c], acc[c]);
        }
        __syncthreads();  // every thread has read cur
        float *dst = seg_S + off + static_cast<int64_t>(DK) * DV + r * DV + col0 + c0;  // S_{p+1}
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            cur[r][c0 + c] = acc[c];
            dst[c] = acc[c];
        }
        __syncthreads();
    }
}

}  // namespace kda
