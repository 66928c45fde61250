// kda_norm.cuh -- exact-rounding L2 normalisation of Q/K rows to bf16.
//
// "KDA Chunk Prefill on Ascend A3", section "Mathematical definition":
// xf = float32(x); xn = bfloat16(xf / sqrt(sum(xf*xf) + 1e-6)).
// Each product xf*xf is rounded to float32 before it is added (no fused
// multiply-add), the epsilon is the float32 constant 1e-6 added inside the
// square root, the root is IEEE sqrt and the quotient is the correctly
// rounded float32 quotient, rounded once more to bf16 (nearest-even).  The
// order of the 128 additions is a butterfly over the warp; every lane ends
// with the same bits because float addition is commutative.
//
// The correctly rounded quotient uses Markstein's correction (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): with r = RN(1/d) and
// q0 = RN(x*r), the residual e = x - q0*d is exact in one fma, and
// RN(q0 + e*r) equals RN(x/d).  It costs one multiply and two fmas per
// element instead of a full division, since d is shared by the whole row.
#pragma once
#include "ptx.cuh"

namespace kda {

__device__ __forceinline__ float div_rn_with_rcp(float x, float d, float r)
{
    const float q0 = __fmul_rn(x, r);
    const float e = __fmaf_rn(-q0, d, x);
    return __fmaf_rn(e, r, q0);
}

// The row's denominator sqrt(sum x^2 + 1e-6) when a warp holds a row of 128
// bf16 values, lane l holding elements 4l..4l+3 as two packed bf16 pairs.
__device__ __forceinline__ float l2norm_den128_warp(uint2 raw)
{
    const float x0 = bf16lo(raw.x), x1 = bf16hi(raw.x), x2 = bf16lo(raw.y), x3 = bf16hi(raw.y);
    float ss = __fmul_rn(x0, x0);
    ss = __fadd_rn(ss, __fmul_rn(x1, x1));
    ss = __fadd_rn(ss, __fmul_rn(x2, x2));
    ss = __fadd_rn(ss, __fmul_rn(x3, x3));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
    return __fsqrt_rn(__fadd_rn(ss, 1e-6f));
}

// The normalised values of lane l's four elements given the row's denominator.
__device__ __forceinline__ uint2 l2norm_apply128(uint2 raw, float den)
{
    const float x0 = bf16lo(raw.x), x1 = bf16hi(raw.x), x2 = bf16lo(raw.y), x3 = bf16hi(raw.y);
    const float r = __frcp_rn(den);
    uint2 out;
    out.x = pack_bf16(div_rn_with_rcp(x0, den, r), div_rn_with_rcp(x1, den, r));
    out.y = pack_bf16(div_rn_with_rcp(x2, den, r), div_rn_with_rcp(x3, den, r));
    return out;
}

// One warp normalises one row of 128 bf16 values; lane l holds elements
// 4l..4l+3 as two packed bf16 pairs (lo, hi).  Returns the packed result.
__device__ __forceinline__ uint2 l2norm_row128_warp(uint2 raw) { return l2norm_apply128(raw, l2norm_den128_warp(raw)); }

// Standalone pass: rows of 128 bf16, one warp per row, grid-stride.
__global__ void __launch_bounds__(256) l2norm_bf16_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                          __nv_bfloat16 *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(x + r * 128 + lane * 4);
        const uint2 res = l2norm_row128_warp(raw);
        *reinterpret_cast<uint2 *>(out + r * 128 + lane * 4) = res;
    }
}

}  // namespace kda
