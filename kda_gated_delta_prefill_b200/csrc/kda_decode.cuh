// kda_decode.cuh -- one recurrent decode step on a bf16 state pool.
//
// The recurrence of "KDA Chunk Prefill on Ascend A3" (section "Mathematical
// definition") for a single token, with the state kept in a caller-owned
// bf16 pool as on the "flashinfer.kda_decode.packed_kda_decode" page: row b
// reads and updates pool slot state_indices[b] in place, and a row whose index
// is -1 writes zeros to its output and touches no state.  For value head h and
// its query/key head hq = h / (HV/H):
//   qn, kn = exact-rounding L2 normalisation of q[b,hq], k[b,hq]   (bf16)
//   S'  = diag(exp(g[b,h])) S                                       (S = float(slot))
//   r   = v[b,h] - kn^T S'
//   S'' = S' + beta[b,h] kn r^T         -> slot = bf16(S'') (nearest even)
//   o   = K^-0.5 qn^T S'' = K^-0.5 (qn^T S' + beta (qn . kn) r)
// The last identity lets one pass over S' give both dot products.
//
// One CTA of 512 threads per (row, value head): thread t owns value columns
// 4 (t % 32) .. +3 and key rows 8 (t / 32) .. +7 of the 128x128 slot, i.e.
// 32 values in registers; every warp reads and writes whole 256-byte rows.
#pragma once
#include "kda_common.cuh"
#include "kda_norm.cuh"
#include "ptx.cuh"

namespace kda {

struct DecodeParams {
    const __nv_bfloat16 *q, *k, *v;  // rows of H*K / H*K / HV*V bf16, row strides below (elements)
    int64_t q_stride, k_stride, v_stride;
    const float *g;                  // [B, HV, K]
    const float *beta;               // [B, HV]
    __nv_bfloat16 *state;            // pool: slot s at state + s * slot_stride, [HV][K][V] inside
    int64_t slot_stride;
    const int32_t *state_indices;    // [B]
    __nv_bfloat16 *o;                // [B, HV, V]
    int H, HV;
};

constexpr int kDecodeThreads = 512, kDecodeRows = DK / (kDecodeThreads / 32);

__global__ void __launch_bounds__(kDecodeThreads) kda_decode_kernel(const DecodeParams p)
{
    constexpr int NW = kDecodeThreads / 32, R = kDecodeRows;
    __shared__ float qn[DK], kn[DK], ex[DK], rr[DV];
    __shared__ __align__(16) float red[NW][2][DV];
    __shared__ float qk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x / p.HV, h = blockIdx.x % p.HV, hq = h / (p.HV / p.H);
    const int slot = p.state_indices[b];
    __nv_bfloat16 *ob = p.o + (static_cast<int64_t>(b) * p.HV + h) * DV;
    if (slot < 0) {  // padding row
        if (tid < DV / 2) reinterpret_cast<uint32_t *>(ob)[tid] = 0u;
        return;
    }
    // this thread's 8 rows x 4 columns of the slot, requested before anything else so that the load overlaps
    // the normalisation below
    const int v0 = 4 * lane, k0 = R * warp;
    __nv_bfloat16 *sp = p.state + static_cast<int64_t>(slot) * p.slot_stride + static_cast<int64_t>(h) * DK * DV;
    uint2 raw[R];
#pragma unroll
    for (int i = 0; i < R; ++i) raw[i] = *reinterpret_cast<const uint2 *>(sp + (k0 + i) * DV + v0);
    // normalised q and k (warps 0 and 1), exp(g) (warps 2-5), as float32
    if (warp < 2) {
        const __nv_bfloat16 *src = warp == 0 ? p.q + b * p.q_stride + hq * DK : p.k + b * p.k_stride + hq * DK;
        const uint2 res = l2norm_row128_warp(*reinterpret_cast<const uint2 *>(src + lane * 4));
        float *dst = warp == 0 ? qn : kn;
        dst[4 * lane] = bf16lo(res.x);
        dst[4 * lane + 1] = bf16hi(res.x);
        dst[4 * lane + 2] = bf16lo(res.y);
        dst[4 * lane + 3] = bf16hi(res.y);
    } else if (warp < 6) {
        const int kk = 32 * (warp - 2) + lane;
        ex[kk] = ex2(p.g[(static_cast<int64_t>(b) * p.HV + h) * DK + kk] * 1.4426950408889634f);
    }
    __syncthreads();
    if (warp == 0) {  // qn . kn
        float s = __fmul_rn(qn[4 * lane], kn[4 * lane]);
#pragma unroll
        for (int j = 1; j < 4; ++j) s = __fmaf_rn(qn[4 * lane + j], kn[4 * lane + j], s);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
        if (lane == 0) qk = s;
    }

    // S' = diag(exp(g)) S for this thread's rows and columns, and its partial dot products
    float s[R][4];
    float a[4] = {}, bq[4] = {};
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const float e = ex[k0 + i], kv = kn[k0 + i], qv = qn[k0 + i];
        s[i][0] = __fmul_rn(bf16lo(raw[i].x), e);
        s[i][1] = __fmul_rn(bf16hi(raw[i].x), e);
        s[i][2] = __fmul_rn(bf16lo(raw[i].y), e);
        s[i][3] = __fmul_rn(bf16hi(raw[i].y), e);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            a[c] = __fmaf_rn(kv, s[i][c], a[c]);
            bq[c] = __fmaf_rn(qv, s[i][c], bq[c]);
        }
    }
    *reinterpret_cast<float4 *>(&red[warp][0][v0]) = make_float4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<float4 *>(&red[warp][1][v0]) = make_float4(bq[0], bq[1], bq[2], bq[3]);
    __syncthreads();
    const float be = p.beta[static_cast<int64_t>(b) * p.HV + h];
    if (tid < DV) {  // column v = tid: r = v - kn^T S', o = K^-0.5 (qn^T S' + beta (qn . kn) r)
        float ka = red[0][0][tid], qa = red[0][1][tid];
#pragma unroll
        for (int w = 1; w < NW; ++w) {
            ka = __fadd_rn(ka, red[w][0][tid]);
            qa = __fadd_rn(qa, red[w][1][tid]);
        }
        const float vv = __bfloat162float(p.v[b * p.v_stride + h * DV + tid]);
        const float r = __fsub_rn(vv, ka);
        rr[tid] = r;
        const float ov = __fmul_rn(0.08838834764831845f, __fmaf_rn(__fmul_rn(be, qk), r, qa));
        ob[tid] = __float2bfloat16_rn(ov);
    }
    __syncthreads();
    // S'' = S' + beta kn r^T, stored as bf16
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const float bk = __fmul_rn(be, kn[k0 + i]);
        float u[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) u[c] = __fmaf_rn(bk, rr[v0 + c], s[i][c]);
        *reinterpret_cast<uint2 *>(sp + (k0 + i) * DV + v0) = make_uint2(pack_bf16(u[0], u[1]), pack_bf16(u[2], u[3]));
    }
}

}  // namespace kda
