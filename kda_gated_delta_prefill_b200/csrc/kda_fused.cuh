// kda_fused.cuh -- fused KDA chunk-prefill forward (one CTA per
// (sequence, value head, value-column slice)).
//
// Math: "KDA Chunk Prefill on Ascend A3", section "Mathematical definition"
// (chunk construction).  For each 64-token chunk the CTA
//   1. stages q, k (Q/K head h / (HV/H)), g, beta and its v columns in shared
//      memory (cp.async, zero-filled past the sequence end, which reproduces
//      the page's zero padding of a partial chunk),
//   2. L2-normalises q/k in place (exact rounding order),
//   3. forms the gate factors from e_u = exp(g_u): inside each 16-token block
//      the inclusive running product base_i = prod_{u<=i} e_u and the
//      exclusive suffix product b_j = prod_{u>j} e_u, so that for i >= j
//      exp(G_i - G_j) = (base_i c) (b_j) with a per-channel factor c built
//      from whole-block products.  Every factor except the diagonal-block
//      c = 1/P_I is <= 1, so nothing overflows for gates in the stated
//      domain, and only one exponential per gate element is evaluated,
//   4. builds L (beta_i-scaled, strictly lower) and Aqk (K^-0.5-scaled,
//      causal) with bf16 tensor-core MMAs over 16x16 block pairs,
//   5. solves A = (I+L)^-1 diag(beta): exact float32 forward substitution
//      inside the four 16x16 diagonal blocks, tf32 MMAs for the off-diagonal
//      blocks (block forward substitution),
//   6. forms -W = -A (exp(G) k) (shared) and U = A v (per warp, registers),
//   7. carries the state: every warp owns 16 value columns and keeps S^T for
//      them in MMA accumulator registers (fp32); Vnew = U - W S,
//      O = Qg S + Aqk Vnew, S^T <- diag-scaled S^T + Vnew^T Kg.
// The loads of chunk c+1 are issued before the carry of chunk c.
#pragma once
#include "kda_norm.cuh"
#include "ptx.cuh"

namespace kda {

constexpr int CH = 64;   // chunk length (tokens)
constexpr int DK = 128;  // key / query head dim
constexpr int DV = 128;  // value head dim

struct FwdParams {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    const float *g;
    const float *beta;
    const float *s0;     // [N,HV,K,V] or null
    const int32_t *cu;   // [N+1] or null
    const int32_t *order;  // [N] longest-first sequence order, or null
    __nv_bfloat16 *o;
    float *sN;
    int B, T, H, HV, N;
    int nslices;         // value-column slices per (sequence, head)
};

// Shared-memory map (byte offsets).  NW warps, VS = 16*NW value columns.
template <int NW>
struct Smem {
    static constexpr int VS = 16 * NW;
    static constexpr int Q = 0;                      // bf16 [64][128], swizzled, normalised in place
    static constexpr int K = Q + CH * DK * 2;        // bf16 [64][128]
    static constexpr int G = K + CH * DK * 2;        // fp32 [64][128]: g -> e -> base
    static constexpr int V = G + CH * DK * 4;        // bf16 [64][VS]
    static constexpr int BETA = V + CH * VS * 2;     // fp32 [64]
    static constexpr int KB = BETA + 256;            // bf16 [64][128]: k*b, later k*exp(G)
    static constexpr int QG = KB + CH * DK * 2;      // bf16 [64][128]: K^-0.5 q exp(G)
    static constexpr int KG = QG + CH * DK * 2;      // bf16 [64][128]: k exp(G_last - G)
    static constexpr int WN = KG + CH * DK * 2;      // bf16 [64][128]: -W
    static constexpr int L = WN + CH * DK * 2;       // fp32 [64][64]
    static constexpr int A = L + CH * CH * 4;        // bf16 [64][64]
    static constexpr int AQK = A + CH * CH * 2;      // bf16 [64][64]
    static constexpr int FC = AQK + CH * CH * 2;     // fp32 [10][128] block-pair factors
    static constexpr int FE = FC + 10 * DK * 4;      // fp32 [4][128] exp(G at block start - 1)
    static constexpr int FGL = FE + 4 * DK * 4;      // fp32 [128] exp(G_last)
    static constexpr int UNI = FGL + DK * 4;         // union: per-warp Vnew | X fp32[64][64] + T scratch
    static constexpr int VN_STRIDE = 48;             // bytes per Vnew row (16 bf16 + pad)
    static constexpr int VN_BYTES = NW * CH * VN_STRIDE;
    static constexpr int X_BYTES = CH * CH * 4;
    static constexpr int TS_STRIDE = 24;             // floats per row of a 16x16 T scratch
    static constexpr int TS_BYTES = 16 * TS_STRIDE * 4;
    static constexpr int UNI_BYTES = (VN_BYTES > X_BYTES + 4 * TS_BYTES) ? VN_BYTES : X_BYTES + 4 * TS_BYTES;
    static constexpr int TOTAL = UNI + UNI_BYTES;
};

// Block pair p = I*(I+1)/2 + J of the lower block triangle, J <= I.
__device__ __forceinline__ void pair_of(int p, int &I, int &J)
{
    I = (p >= 6) ? 3 : (p >= 3) ? 2 : (p >= 1) ? 1 : 0;
    J = p - I * (I + 1) / 2;
}

template <int NW>
__device__ __forceinline__ void load_chunk(uint32_t sbase, const FwdParams &p, int64_t row0, int nvalid, int h,
                                           int hq, int v0)
{
    using S = Smem<NW>;
    constexpr int NT = NW * 32;
    const int tid = threadIdx.x;
    for (int idx = tid; idx < CH * 16; idx += NT) {
        const int r = idx >> 4, ch = idx & 15;
        const bool ok = r < nvalid;
        const int64_t gr = row0 + (ok ? r : 0);
        const uint32_t off = swz(r, ch * 16, 256);
        cp_async16(sbase + S::Q + off, p.q + (gr * p.H + hq) * DK + ch * 8, ok ? 16u : 0u);
        cp_async16(sbase + S::K + off, p.k + (gr * p.H + hq) * DK + ch * 8, ok ? 16u : 0u);
    }
    for (int idx = tid; idx < CH * 32; idx += NT) {
        const int r = idx >> 5, ch = idx & 31;
        const bool ok = r < nvalid;
        const int64_t gr = row0 + (ok ? r : 0);
        cp_async16(sbase + S::G + swz(r, ch * 16, 512), p.g + (gr * p.HV + h) * DK + ch * 4, ok ? 16u : 0u);
    }
    constexpr int VCH = S::VS / 8;
    for (int idx = tid; idx < CH * VCH; idx += NT) {
        const int r = idx / VCH, ch = idx % VCH;
        const bool ok = r < nvalid;
        const int64_t gr = row0 + (ok ? r : 0);
        cp_async16(sbase + S::V + swz(r, ch * 16, S::VS * 2), p.v + (gr * p.HV + h) * DV + v0 + ch * 8,
                   ok ? 16u : 0u);
    }
    if (tid < CH) {
        const bool ok = tid < nvalid;
        const int64_t gr = row0 + (ok ? tid : 0);
        cp_async4(sbase + S::BETA + tid * 4, p.beta + gr * p.HV + h, ok ? 4u : 0u);
    }
    cp_async_commit();
}

// Off-diagonal block of X = (I+L)^-1: X_IJ = -D_I * sum_{M=J}^{I-1} L_IM X_MJ  (one warp, tf32 MMAs).
constexpr int TS = 24;  // row stride (floats) of the per-warp 16x16 scratch; conflict-free column reads

__device__ __forceinline__ void solve_block(uint8_t *sm_L, uint8_t *sm_X, float *ts, int I, int J, int lane)
{
    const int g = lane >> 2, t = lane & 3;
    auto Lat = [&](int r, int c) { return *reinterpret_cast<const float *>(sm_L + swz(r, c * 4, 256)); };
    auto Xat = [&](int r, int c) { return *reinterpret_cast<const float *>(sm_X + swz(r, c * 4, 256)); };
    float acc[2][4] = {};
    for (int M = J; M < I; ++M) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t a[4];
            a[0] = to_tf32(Lat(16 * I + g, 16 * M + 8 * ks + t));
            a[1] = to_tf32(Lat(16 * I + g + 8, 16 * M + 8 * ks + t));
            a[2] = to_tf32(Lat(16 * I + g, 16 * M + 8 * ks + t + 4));
            a[3] = to_tf32(Lat(16 * I + g + 8, 16 * M + 8 * ks + t + 4));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const uint32_t b0 = to_tf32(Xat(16 * M + 8 * ks + t, 16 * J + 8 * nt + g));
                const uint32_t b1 = to_tf32(Xat(16 * M + 8 * ks + t + 4, 16 * J + 8 * nt + g));
                mma_tf32(acc[nt], a, b0, b1);
            }
        }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        ts[g * TS + 8 * nt + 2 * t] = acc[nt][0];
        ts[g * TS + 8 * nt + 2 * t + 1] = acc[nt][1];
        ts[(g + 8) * TS + 8 * nt + 2 * t] = acc[nt][2];
        ts[(g + 8) * TS + 8 * nt + 2 * t + 1] = acc[nt][3];
    }
    __syncwarp();
    float x[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[4];
        a[0] = to_tf32(Xat(16 * I + g, 16 * I + 8 * ks + t));
        a[1] = to_tf32(Xat(16 * I + g + 8, 16 * I + 8 * ks + t));
        a[2] = to_tf32(Xat(16 * I + g, 16 * I + 8 * ks + t + 4));
        a[3] = to_tf32(Xat(16 * I + g + 8, 16 * I + 8 * ks + t + 4));
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = to_tf32(ts[(8 * ks + t) * TS + 8 * nt + g]);
            const uint32_t b1 = to_tf32(ts[(8 * ks + t + 4) * TS + 8 * nt + g]);
            mma_tf32(x[nt], a, b0, b1);
        }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int c = 16 * J + 8 * nt + 2 * t;
        *reinterpret_cast<float2 *>(sm_X + swz(16 * I + g, c * 4, 256)) = make_float2(-x[nt][0], -x[nt][1]);
        *reinterpret_cast<float2 *>(sm_X + swz(16 * I + g + 8, c * 4, 256)) = make_float2(-x[nt][2], -x[nt][3]);
    }
    __syncwarp();
}

template <int NW>
__global__ void __launch_bounds__(NW * 32, 1) kda_fused_fwd_kernel(const FwdParams p)
{
    using S = Smem<NW>;
    constexpr int VS = S::VS;
    constexpr int NT = NW * 32;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;

    // ---- work unit ----
    const int slice = blockIdx.x % p.nslices;
    const int rest = blockIdx.x / p.nslices;
    const int h = rest % p.HV;
    const int r_idx = rest / p.HV;
    const int n = p.order ? p.order[r_idx] : r_idx;
    const int hq = h / (p.HV / p.H);
    const int v0 = slice * VS;
    int64_t bt0;
    int len;
    if (p.cu) {
        bt0 = p.cu[n];
        len = p.cu[n + 1] - p.cu[n];
    } else {
        bt0 = static_cast<int64_t>(n) * p.T;
        len = p.T;
    }
    if (len < 0) len = 0;
    const int nchunks = (len + CH - 1) / CH;
    const float scale = 0.08838834764831845f;  // 128^-0.5 rounded to float32

    // ---- state: S^T for this warp's 16 value columns, as MMA accumulators ----
    // sT[nt][e]: value column vl = g8 + 8*(e>>1), key channel kd = 8*nt + 2*t4 + (e&1)
    float sT[16][4];
    {
        const int vcol = v0 + 16 * warp + g8;
        const float *s0 = p.s0 ? p.s0 + (static_cast<int64_t>(n) * p.HV + h) * DK * DV : nullptr;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int kd = 8 * nt + 2 * t4 + (e & 1);
                const int vc = vcol + 8 * (e >> 1);
                sT[nt][e] = s0 ? s0[kd * DV + vc] : 0.f;
            }
    }

    if (nchunks > 0) load_chunk<NW>(sbase, p, bt0, len < CH ? len : CH, h, hq, v0);

    for (int c = 0; c < nchunks; ++c) {
        const int64_t row0 = bt0 + static_cast<int64_t>(c) * CH;
        const int nvalid = (len - c * CH) < CH ? (len - c * CH) : CH;
        cp_async_wait_all();
        __syncthreads();

        // ---- (2) normalise q and k in place ----
        for (int rr = warp; rr < 2 * CH; rr += NW) {
            uint8_t *tile = sm + (rr < CH ? S::Q : S::K);
            const uint32_t off = swz(rr & (CH - 1), lane * 8, 256);
            uint2 raw = *reinterpret_cast<uint2 *>(tile + off);
            *reinterpret_cast<uint2 *>(tile + off) = l2norm_row128_warp(raw);
        }
        __syncthreads();

        // ---- (3) gate factors: thread d owns key channel d ----
        if (tid < DK) {
            const int d = tid;
            float P[4];
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                float pr = 1.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    float *gp = reinterpret_cast<float *>(sm + S::G + swz(16 * J + u, d * 4, 512));
                    const float e = ex2(*gp * 1.4426950408889634f);
                    *gp = e;
                    pr *= e;
                }
                P[J] = pr;
            }
            const float E[4] = {1.f, P[0], P[0] * P[1], P[0] * P[1] * P[2]};
            const float F[4] = {P[1] * P[2] * P[3], P[2] * P[3], P[3], 1.f};
            float *fc = reinterpret_cast<float *>(sm + S::FC);
            float rp[4];
#pragma unroll
            for (int J = 0; J < 4; ++J) rp[J] = __frcp_rn(fmaxf(P[J], 1e-37f));
            fc[0 * DK + d] = rp[0];
            fc[1 * DK + d] = 1.f;
            fc[2 * DK + d] = rp[1];
            fc[3 * DK + d] = P[1];
            fc[4 * DK + d] = 1.f;
            fc[5 * DK + d] = rp[2];
            fc[6 * DK + d] = P[1] * P[2];
            fc[7 * DK + d] = P[2];
            fc[8 * DK + d] = 1.f;
            fc[9 * DK + d] = rp[3];
            float *fe = reinterpret_cast<float *>(sm + S::FE);
#pragma unroll
            for (int J = 0; J < 4; ++J) fe[J * DK + d] = E[J];
            reinterpret_cast<float *>(sm + S::FGL)[d] = E[3] * P[3];
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                float e[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    e[u] = *reinterpret_cast<float *>(sm + S::G + swz(16 * J + u, d * 4, 512));
                float b[16];
                b[15] = 1.f;
#pragma unroll
                for (int u = 14; u >= 0; --u) b[u] = b[u + 1] * e[u + 1];
                float bs = 1.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = 16 * J + u;
                    bs *= e[u];
                    *reinterpret_cast<float *>(sm + S::G + swz(i, d * 4, 512)) = bs;
                    const uint32_t o2 = swz(i, d * 2, 256);
                    const float kv = __bfloat162float(*reinterpret_cast<__nv_bfloat16 *>(sm + S::K + o2));
                    const float qv = __bfloat162float(*reinterpret_cast<__nv_bfloat16 *>(sm + S::Q + o2));
                    *reinterpret_cast<__nv_bfloat16 *>(sm + S::KB + o2) = __float2bfloat16_rn(kv * b[u]);
                    *reinterpret_cast<__nv_bfloat16 *>(sm + S::KG + o2) = __float2bfloat16_rn(kv * b[u] * F[J]);
                    *reinterpret_cast<__nv_bfloat16 *>(sm + S::QG + o2) =
                        __float2bfloat16_rn(scale * qv * bs * E[J]);
                }
            }
        }
        __syncthreads();

        // ---- (4) L and Aqk over the 10 lower block pairs ----
        for (int pidx = warp; pidx < 10; pidx += NW) {
            int I, J;
            pair_of(pidx, I, J);
            float accL[2][4] = {}, accQ[2][4] = {};
            const float *fc = reinterpret_cast<const float *>(sm + S::FC) + pidx * DK;
#pragma unroll 2
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t ak[4], aq[4];
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {      // column half: +0 / +8
                    const int col = 16 * ks + 2 * t4 + 8 * hc;
                    const float2 cc = *reinterpret_cast<const float2 *>(fc + col);
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {  // row half: +0 / +8
                        const int row = 16 * I + g8 + 8 * hr;
                        const float2 bs = *reinterpret_cast<const float2 *>(sm + S::G + swz(row, col * 4, 512));
                        const uint32_t o2 = swz(row, col * 2, 256);
                        const uint32_t kx = *reinterpret_cast<const uint32_t *>(sm + S::K + o2);
                        const uint32_t qx = *reinterpret_cast<const uint32_t *>(sm + S::Q + o2);
                        const float s0 = bs.x * cc.x, s1 = bs.y * cc.y;
                        ak[hr + 2 * hc] = pack_bf16(bf16lo(kx) * s0, bf16hi(kx) * s1);
                        aq[hr + 2 * hc] = pack_bf16(bf16lo(qx) * s0, bf16hi(qx) * s1);
                    }
                }
                uint32_t b[4];
                {
                    const int mi = lane >> 3;
                    const int j = 16 * J + (mi >> 1) * 8 + (lane & 7);
                    const int d = 16 * ks + (mi & 1) * 8;
                    ldsm_x4(sbase + S::KB + swz(j, d * 2, 256), b[0], b[1], b[2], b[3]);
                }
                mma_bf16(accL[0], ak, b[0], b[1]);
                mma_bf16(accL[1], ak, b[2], b[3]);
                mma_bf16(accQ[0], aq, b[0], b[1]);
                mma_bf16(accQ[1], aq, b[2], b[3]);
            }
            const float *sbeta = reinterpret_cast<const float *>(sm + S::BETA);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int i = 16 * I + g8 + 8 * hr;
                    const int j = 16 * J + 8 * nt + 2 * t4;
                    const float bi = sbeta[i];
                    const float l0 = (j < i) ? bi * accL[nt][2 * hr] : 0.f;
                    const float l1 = (j + 1 < i) ? bi * accL[nt][2 * hr + 1] : 0.f;
                    const float q0 = (j <= i) ? scale * accQ[nt][2 * hr] : 0.f;
                    const float q1 = (j + 1 <= i) ? scale * accQ[nt][2 * hr + 1] : 0.f;
                    *reinterpret_cast<float2 *>(sm + S::L + swz(i, j * 4, 256)) = make_float2(l0, l1);
                    *reinterpret_cast<uint32_t *>(sm + S::AQK + swz(i, j * 2, 128)) = pack_bf16(q0, q1);
                }
        }
        __syncthreads();

        // ---- (5) A = (I+L)^-1 diag(beta) ----
        uint8_t *sX = sm + S::UNI;
        if (warp < 4 && lane < 16) {  // diagonal blocks: exact fp32 forward substitution, lane = column
            const int I = warp, cidx = lane;
            float dcol[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float acc = (j == cidx) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < j; ++m)
                    acc = __fmaf_rn(-*reinterpret_cast<const float *>(sm + S::L + swz(16 * I + j, (16 * I + m) * 4, 256)),
                                    dcol[m], acc);
                dcol[j] = acc;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j)
                *reinterpret_cast<float *>(sX + swz(16 * I + j, (16 * I + cidx) * 4, 256)) = dcol[j];
        }
        __syncthreads();
        {
            float *ts = reinterpret_cast<float *>(sm + S::UNI + S::X_BYTES) + warp * 16 * S::TS_STRIDE;
            // level 1: (1,0) (2,1) (3,2)
            if (warp < 3) solve_block(sm + S::L, sX, ts, warp + 1, warp, lane);
            __syncthreads();
            if (warp < 2) solve_block(sm + S::L, sX, ts, warp + 2, warp, lane);
            __syncthreads();
            if (warp < 1) solve_block(sm + S::L, sX, ts, 3, 0, lane);
            __syncthreads();
        }
        {
            // A (bf16) = X diag(beta), zero above the diagonal; k*exp(G) into the KB buffer.
            const float *sbeta = reinterpret_cast<const float *>(sm + S::BETA);
            for (int idx = tid; idx < CH * CH / 2; idx += NT) {
                const int i = idx >> 5, j = (idx & 31) * 2;
                const float2 x = *reinterpret_cast<const float2 *>(sX + swz(i, j * 4, 256));
                const float a0 = (j <= i) ? x.x * sbeta[j] : 0.f;
                const float a1 = (j + 1 <= i) ? x.y * sbeta[j + 1] : 0.f;
                *reinterpret_cast<uint32_t *>(sm + S::A + swz(i, j * 2, 128)) = pack_bf16(a0, a1);
            }
            const float *fe = reinterpret_cast<const float *>(sm + S::FE);
            for (int idx = tid; idx < CH * DK / 2; idx += NT) {
                const int i = idx >> 6, d = (idx & 63) * 2;
                const float2 bs = *reinterpret_cast<const float2 *>(sm + S::G + swz(i, d * 4, 512));
                const float2 ee = *reinterpret_cast<const float2 *>(fe + (i >> 4) * DK + d);
                const uint32_t o2 = swz(i, d * 2, 256);
                const uint32_t kx = *reinterpret_cast<const uint32_t *>(sm + S::K + o2);
                *reinterpret_cast<uint32_t *>(sm + S::KB + o2) =
                    pack_bf16(bf16lo(kx) * bs.x * ee.x, bf16hi(kx) * bs.y * ee.y);
            }
        }
        __syncthreads();

        // ---- (6) -W = -A (exp(G) k) into WN (split over warps by key columns); U = A v in registers ----
        float acc[4][2][4];  // [m-tile][value n-tile][4]: U, then Vnew
        {
            constexpr int WNT = 16 / NW;  // n-tiles (8 key columns) per warp
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                float w[WNT][4] = {};
                for (int ks = 0; ks <= mt; ++ks) {
                    uint32_t a[4];
                    {
                        const int mi = lane >> 3;
                        const int r = 16 * mt + (mi & 1) * 8 + (lane & 7);
                        const int cc = 16 * ks + (mi >> 1) * 8;
                        ldsm_x4(sbase + S::A + swz(r, cc * 2, 128), a[0], a[1], a[2], a[3]);
                    }
#pragma unroll
                    for (int np = 0; np < WNT; np += 2) {
                        const int n0 = (warp * WNT + np) * 8;
                        const int mi = lane >> 3;
                        const int tok = 16 * ks + (mi & 1) * 8 + (lane & 7);
                        const int kd = n0 + (mi >> 1) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(sbase + S::KB + swz(tok, kd * 2, 256), b0, b1, b2, b3);
                        mma_bf16(w[np], a, b0, b1);
                        mma_bf16(w[np + 1], a, b2, b3);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < WNT; ++nt) {
                    const int kd = (warp * WNT + nt) * 8 + 2 * t4;
                    const int r = 16 * mt + g8;
                    *reinterpret_cast<uint32_t *>(sm + S::WN + swz(r, kd * 2, 256)) = pack_bf16(-w[nt][0], -w[nt][1]);
                    *reinterpret_cast<uint32_t *>(sm + S::WN + swz(r + 8, kd * 2, 256)) =
                        pack_bf16(-w[nt][2], -w[nt][3]);
                }
                // U for this warp's 16 value columns
                acc[mt][0][0] = acc[mt][0][1] = acc[mt][0][2] = acc[mt][0][3] = 0.f;
                acc[mt][1][0] = acc[mt][1][1] = acc[mt][1][2] = acc[mt][1][3] = 0.f;
                for (int ks = 0; ks <= mt; ++ks) {
                    uint32_t a[4];
                    {
                        const int mi = lane >> 3;
                        const int r = 16 * mt + (mi & 1) * 8 + (lane & 7);
                        const int cc = 16 * ks + (mi >> 1) * 8;
                        ldsm_x4(sbase + S::A + swz(r, cc * 2, 128), a[0], a[1], a[2], a[3]);
                    }
                    const int mi = lane >> 3;
                    const int tok = 16 * ks + (mi & 1) * 8 + (lane & 7);
                    const int vc = 16 * warp + (mi >> 1) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(sbase + S::V + swz(tok, vc * 2, VS * 2), b0, b1, b2, b3);
                    mma_bf16(acc[mt][0], a, b0, b1);
                    mma_bf16(acc[mt][1], a, b2, b3);
                }
            }
        }
        __syncthreads();

        // raw buffers are free: prefetch chunk c+1 while the carry runs
        if (c + 1 < nchunks) {
            const int nv1 = (len - (c + 1) * CH) < CH ? (len - (c + 1) * CH) : CH;
            load_chunk<NW>(sbase, p, row0 + CH, nv1, h, hq, v0);
        }

        // ---- (7) state carry (warp-local) ----
        float oacc[4][2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t bs[2][2];
#pragma unroll
            for (int nv = 0; nv < 2; ++nv) {
                bs[nv][0] = pack_bf16(sT[2 * ks][2 * nv], sT[2 * ks][2 * nv + 1]);
                bs[nv][1] = pack_bf16(sT[2 * ks + 1][2 * nv], sT[2 * ks + 1][2 * nv + 1]);
            }
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                const int mi = lane >> 3;
                const int r = 16 * mt + (mi & 1) * 8 + (lane & 7);
                const int cc = 16 * ks + (mi >> 1) * 8;
                uint32_t aw[4], aqg[4];
                ldsm_x4(sbase + S::WN + swz(r, cc * 2, 256), aw[0], aw[1], aw[2], aw[3]);
                ldsm_x4(sbase + S::QG + swz(r, cc * 2, 256), aqg[0], aqg[1], aqg[2], aqg[3]);
#pragma unroll
                for (int nv = 0; nv < 2; ++nv) {
                    mma_bf16(acc[mt][nv], aw, bs[nv][0], bs[nv][1]);
                    mma_bf16(oacc[mt][nv], aqg, bs[nv][0], bs[nv][1]);
                }
            }
        }
        // Vnew -> bf16 -> per-warp buffer [64 tok][16 v]
        uint8_t *vn = sm + S::UNI + warp * CH * S::VN_STRIDE;
        const uint32_t vn_s = smem_u32(vn);
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int nv = 0; nv < 2; ++nv) {
                const int r = 16 * mt + g8;
                const int vc = 8 * nv + 2 * t4;
                *reinterpret_cast<uint32_t *>(vn + r * S::VN_STRIDE + vc * 2) = pack_bf16(acc[mt][nv][0], acc[mt][nv][1]);
                *reinterpret_cast<uint32_t *>(vn + (r + 8) * S::VN_STRIDE + vc * 2) =
                    pack_bf16(acc[mt][nv][2], acc[mt][nv][3]);
            }
        __syncwarp();
        // O += Aqk Vnew
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            for (int ks = 0; ks <= mt; ++ks) {
                const int mi = lane >> 3;
                uint32_t a[4];
                {
                    const int r = 16 * mt + (mi & 1) * 8 + (lane & 7);
                    const int cc = 16 * ks + (mi >> 1) * 8;
                    ldsm_x4(sbase + S::AQK + swz(r, cc * 2, 128), a[0], a[1], a[2], a[3]);
                }
                const int tok = 16 * ks + (mi & 1) * 8 + (lane & 7);
                const int vc = (mi >> 1) * 8;
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vn_s + tok * S::VN_STRIDE + vc * 2, b0, b1, b2, b3);
                mma_bf16(oacc[mt][0], a, b0, b1);
                mma_bf16(oacc[mt][1], a, b2, b3);
            }
        }
        // store o rows of valid tokens
        {
            __nv_bfloat16 *obase = p.o + (row0 * p.HV + h) * DV + v0 + 16 * warp;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int tok = 16 * mt + g8 + 8 * hr;
                    if (tok < nvalid) {
#pragma unroll
                        for (int nv = 0; nv < 2; ++nv)
                            *reinterpret_cast<uint32_t *>(obase + static_cast<int64_t>(tok) * p.HV * DV + 8 * nv + 2 * t4) =
                                pack_bf16(oacc[mt][nv][2 * hr], oacc[mt][nv][2 * hr + 1]);
                    }
                }
        }
        // S^T <- S^T diag(exp(G_last)) + Vnew^T Kg
        {
            const float *gl = reinterpret_cast<const float *>(sm + S::FGL);
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                const float2 f = *reinterpret_cast<const float2 *>(gl + 8 * nt + 2 * t4);
                sT[nt][0] *= f.x;
                sT[nt][1] *= f.y;
                sT[nt][2] *= f.x;
                sT[nt][3] *= f.y;
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int mi = lane >> 3;
                uint32_t a[4];
                {
                    const int tok = 16 * ks + (mi >> 1) * 8 + (lane & 7);
                    const int vc = (mi & 1) * 8;
                    ldsm_x4_t(vn_s + tok * S::VN_STRIDE + vc * 2, a[0], a[1], a[2], a[3]);
                }
#pragma unroll
                for (int np = 0; np < 16; np += 2) {
                    const int tok = 16 * ks + (mi & 1) * 8 + (lane & 7);
                    const int kd = 8 * np + (mi >> 1) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(sbase + S::KG + swz(tok, kd * 2, 256), b0, b1, b2, b3);
                    mma_bf16(sT[np], a, b0, b1);
                    mma_bf16(sT[np + 1], a, b2, b3);
                }
            }
        }
    }

    // ---- final state ----
    {
        float *sN = p.sN + (static_cast<int64_t>(n) * p.HV + h) * DK * DV;
        const int vcol = v0 + 16 * warp + g8;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int kd = 8 * nt + 2 * t4 + (e & 1);
                sN[kd * DV + vcol + 8 * (e >> 1)] = sT[nt][e];
            }
    }
}

// Longest-first order of packed sequences: order[rank] = n, ranks by
// descending length, ties by index.  One thread per sequence.
__global__ void __launch_bounds__(256) seq_order_kernel(const int32_t *__restrict__ cu, int N, int32_t *__restrict__ order)
{
    __shared__ int32_t len_tile[1024];
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int my = (n < N) ? cu[n + 1] - cu[n] : 0;
    int rank = 0;
    for (int base = 0; base < N; base += 1024) {
        __syncthreads();
        for (int i = threadIdx.x; i < 1024; i += blockDim.x)
            len_tile[i] = (base + i < N) ? cu[base + i + 1] - cu[base + i] : -1;
        __syncthreads();
        const int lim = (N - base) < 1024 ? (N - base) : 1024;
        for (int i = 0; i < lim; ++i) {
            const int l = len_tile[i];
            rank += (l > my) || (l == my && base + i < n);
        }
    }
    if (n < N) order[rank] = n;
}

}  // namespace kda
