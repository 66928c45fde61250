// kda_norm.cuh -- exact-rounding L2 normalisation of Q/K rows to bf16.
//
// "KDA Chunk Prefill on Ascend A3", section "Mathematical definition":
// xf = float32(x); xn = bfloat16(xf / sqrt(sum(xf*xf) + 1e-6)).
// Each product xf*xf is rounded to float32 before it is added (no fused
// multiply-add), the epsilon is the float32 constant 1e-6 added inside the
// square root, the root is IEEE sqrt and the quotient is the correctly
// rounded float32 quotient, rounded once more to bf16 (nearest-even).  The
// order of the 128 additions is fixed by l2norm_half_row below (the page
// leaves it open); both lanes of a row end with the same bits.
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

// One row of 128 bf16 values held by two adjacent lanes of a warp (lanes 2m and 2m+1): each holds 64
// consecutive elements of the row as eight 16-byte words (any order of the words; the element order inside a
// word is (lo, hi) pairs).  This is the only normalisation routine: the forward's intra-chunk prologue and the
// standalone kda_l2norm_bf16 kernel both call it, so the arithmetic the forward runs is the arithmetic the
// standalone kernel's tests check.
// Sum of squares: a thread keeps two float32 partial sums, one over the low and one over the high elements of
// its packed pairs, taking its words in index order and each pair's squares rounded before they are added
// (packed f32x2 multiply, then packed add); then low + high, then + the partner lane's sum (xor-1 shuffle),
// which both lanes form in the same order.  The words are overwritten with the normalised row.
__device__ __forceinline__ void l2norm_half_row(uint4 (&raw)[8])
{
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 x = unpack_bf16(w[j]);
            acc = add2(acc, mul2(x, x));
        }
    }
    float ss = __fadd_rn(acc.x, acc.y);
    ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, 1));
    const float den = __fsqrt_rn(__fadd_rn(ss, 1e-6f));
    const float rr = __frcp_rn(den);
    const float2 r2 = make_float2(rr, rr), nd2 = make_float2(-den, -den);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // Markstein's correction, packed: q0 = x r, e = x - q0 d (exact), RN(q0 + e r) = RN(x / d)
            const float2 x = unpack_bf16(w[j]);
            const float2 q0 = mul2(x, r2);
            const float2 e = fma2(q0, nd2, x);
            const float2 y = fma2(e, r2, q0);
            w[j] = pack_bf16(y.x, y.y);
        }
        raw[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// A whole warp on one row (the decode step and the backward's recomputation, whose threads hold other
// slices): lane l holds elements 4l..4l+3 as two packed bf16 pairs; the sum of squares is the lane's four
// products added left to right, then a butterfly over the warp.  Within one bf16 unit of the exact quotient
// like l2norm_half_row, but not necessarily bit-equal to it.
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

__device__ __forceinline__ uint2 l2norm_row128_warp(uint2 raw) { return l2norm_apply128(raw, l2norm_den128_warp(raw)); }

// Standalone pass: rows of 128 bf16, two lanes per row (64 elements each), grid-stride over groups of 16 rows
// per warp.
__global__ void __launch_bounds__(256) l2norm_bf16_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                          __nv_bfloat16 *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t r0 = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 16; r0 < rows;
         r0 += warps * 16) {
        const int64_t r = r0 + (lane >> 1);
        const bool live = r < rows;  // both lanes of a row agree; the shuffle partner is always in the warp
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (live ? r : r0) * 128 + (lane & 1) * 64);
        uint4 raw[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) raw[c] = src[c];
        l2norm_half_row(raw);
        if (live) {
            uint4 *dst = reinterpret_cast<uint4 *>(out + r * 128 + (lane & 1) * 64);
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = raw[c];
        }
    }
}

}  // namespace kda
