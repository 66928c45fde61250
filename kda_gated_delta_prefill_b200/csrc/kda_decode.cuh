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
// Persistent CTAs walk the (row, value head) units u = blockIdx.x,
// blockIdx.x + gridDim.x, ...  The 32 KB [K][V] block of a unit is contiguous
// in the pool, so it moves through a ring of STAGES shared-memory stages by
// one bulk copy each way: thread 0 requests the block of the next unit while
// the CTA updates the current one in place, and a bulk store writes it back.
// The small operands of the next unit (q, k, g, v, beta rows) are loaded into
// registers one unit ahead and the pool indices two units ahead, so that no
// global-memory latency sits on a unit's own critical path.  Thread t owns
// value columns 4 (t % 32) .. +3 and key rows R (t / 32) .. +R-1 of the block.
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
    unsigned *err;                   // device error word (ERR_TMA_WAIT when a copy never lands)
    int B, H, HV;
};

constexpr int kDecodeBlockBytes = DK * DV * 2;

template <int THREADS, int STAGES>
struct DecodeSmem {
    static constexpr int NW = THREADS / 32;
    static constexpr int RING = 0;                                       // STAGES x [K][V] bf16
    static constexpr int ROWC = STAGES * kDecodeBlockBytes;              // float4 [K]: exp(g), kn, qn, -
    static constexpr int RR = ROWC + DK * 16;                            // float [V]: r
    static constexpr int RED = RR + DV * 4;                              // float [NW][2][V]
    static constexpr int QK = RED + NW * 2 * DV * 4;                     // float [2]: qn . kn, beta
    static constexpr int FLAG = QK + 8;                                  // int
    static constexpr int BAR = QK + 16;                                  // mbarriers [STAGES]
    static constexpr int TOTAL = BAR + 8 * STAGES;
};

// Launch shape of the decode step: 256 threads, a two-stage ring, three CTAs on an SM.
constexpr int kDecodeThreads = 256, kDecodeStages = 2, kDecodeCtasPerSm = 3;

template <int THREADS, int STAGES>
__global__ void __launch_bounds__(THREADS) kda_decode_kernel(const DecodeParams p)
{
    static_assert(STAGES == 2 || STAGES == 3, "ring shape");
    static_assert(THREADS >= 6 * 32 && THREADS >= DV, "warps 0-5 stage the operands, threads 0..V-1 finish columns");
    using S = DecodeSmem<THREADS, STAGES>;
    constexpr int NW = S::NW, R = DK / NW;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    float4 *rowc = reinterpret_cast<float4 *>(sm + S::ROWC);
    float *rr = reinterpret_cast<float *>(sm + S::RR);
    float(*red)[2][DV] = reinterpret_cast<float(*)[2][DV]>(sm + S::RED);
    float *qk = reinterpret_cast<float *>(sm + S::QK);
    volatile int *flag = reinterpret_cast<volatile int *>(sm + S::FLAG);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int units = p.B * p.HV, G = gridDim.x;
    const int v0 = 4 * lane, k0 = R * warp;

    auto slot_of = [&](int u) -> int { return u < units ? p.state_indices[u / p.HV] : -1; };
    auto block_of = [&](int u, int slot) -> __nv_bfloat16 * {
        return p.state + static_cast<int64_t>(slot) * p.slot_stride + static_cast<int64_t>(u % p.HV) * DK * DV;
    };
    // this thread's share of unit u's small operands: a q or k quad (warps 0, 1), one exp(g) input
    // (warps 2-5), one v element and beta (threads 0..V-1)
    struct Ops {
        uint2 x;
        float gv, vv, be;
    };
    auto fetch = [&](int u, Ops &o) {
        if (u >= units) return;
        const int b = u / p.HV, h = u - b * p.HV, hq = h / (p.HV / p.H);
        if (warp < 2)
            o.x = *reinterpret_cast<const uint2 *>((warp == 0 ? p.q + b * p.q_stride : p.k + b * p.k_stride) +
                                                   hq * DK + lane * 4);
        else if (warp < 6)
            o.gv = p.g[(static_cast<int64_t>(b) * p.HV + h) * DK + 32 * (warp - 2) + lane];
        if (tid < DV) {
            o.vv = __bfloat162float(p.v[b * p.v_stride + h * DV + tid]);
            o.be = p.beta[static_cast<int64_t>(b) * p.HV + h];
        }
    };
    // thread 0: request unit u's block (slot >= 0) into stage st
    auto request = [&](int u, int slot, int st) {
        mbar_expect_tx(sb + S::BAR + 8 * st, kDecodeBlockBytes);
        bulk_load(sb + S::RING + st * kDecodeBlockBytes, block_of(u, slot), kDecodeBlockBytes, sb + S::BAR + 8 * st);
    };

    int u = blockIdx.x;
    int slot_cur = slot_of(u), slot_nxt = slot_of(u + G);
    Ops cur{}, nxt{};
    fetch(u, cur);
    // thread 0 bookkeeping: `stored` = the previous unit committed a bulk store; bit st of `pend` = a copy
    // into stage st is in flight and not yet waited for; bit st of `phases` = parity of its next completion
    bool stored = false;
    uint32_t pend = 0, phases = 0;
    if (tid == 0) {
        for (int st = 0; st < STAGES; ++st) mbar_init(sb + S::BAR + 8 * st, 1);
        fence_mbar_init();
        if (u < units && slot_cur >= 0) {
            request(u, slot_cur, 0);
            pend = 1;
        }
    }
    __syncthreads();

    bool ok = true;
    for (int i = 0; u < units; u += G, ++i) {
        const int st = i % STAGES;
        const int b = u / p.HV, h = u - b * p.HV;
        __nv_bfloat16 *ob = p.o + (static_cast<int64_t>(b) * p.HV + h) * DV;
        const int slot_far = slot_of(u + 2 * G);
        fetch(u + G, nxt);
        if (tid == 0 && u + G < units && slot_nxt >= 0) {
            // the next stage last held the unit STAGES steps back; with three stages the previous unit's store
            // may still be reading its own stage
            if (STAGES == 3 && stored) bulk_wait_read_allow<1>();
            else bulk_wait_read();
            const int sn = (i + 1) % STAGES;
            request(u + G, slot_nxt, sn);
            pend |= 1u << sn;
        }
        if (tid == 0) stored = false;
        if (slot_cur < 0) {  // padding row
            if (tid < DV / 2) reinterpret_cast<uint32_t *>(ob)[tid] = 0u;
        } else {
            // per key row: exp(g) (warps 2-5), normalised k (warp 1) and q (warp 0), as float32
            if (warp < 2) {
                const uint2 res = l2norm_row128_warp(cur.x);
                float *d = reinterpret_cast<float *>(rowc) + (warp == 0 ? 2 : 1);
                d[16 * lane] = bf16lo(res.x);
                d[16 * lane + 4] = bf16hi(res.x);
                d[16 * lane + 8] = bf16lo(res.y);
                d[16 * lane + 12] = bf16hi(res.y);
            } else if (warp < 6) {
                rowc[32 * (warp - 2) + lane].x = ex2(cur.gv * 1.4426950408889634f);
            }
            if (tid == 0) {
                const bool landed = mbar_wait(sb + S::BAR + 8 * st, (phases >> st) & 1);
                flag[0] = landed;
                if (landed) {
                    phases ^= 1u << st;
                    pend &= ~(1u << st);
                }
            }
            __syncthreads();
            if (!flag[0]) {
                ok = false;
                break;
            }
            if (warp == 0) {  // qn . kn
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 c = rowc[4 * lane + j];
                    s = j == 0 ? __fmul_rn(c.z, c.y) : __fmaf_rn(c.z, c.y, s);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
                if (lane == 0) qk[0] = s;
            }
            // partial kn^T S' and qn^T S' over this thread's rows, S' = diag(exp(g)) S
            uint8_t *blk = sm + S::RING + st * kDecodeBlockBytes;
            // (column pairs in packed f32x2 arithmetic; every lane rounds as the scalar form would)
            float2 a01 = make_float2(0.f, 0.f), a23 = a01, q01 = a01, q23 = a01;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint2 raw = *reinterpret_cast<const uint2 *>(blk + ((k0 + r) * DV + v0) * 2);
                const float4 c = rowc[k0 + r];
                const float2 e2 = make_float2(c.x, c.x), k2 = make_float2(c.y, c.y), q2 = make_float2(c.z, c.z);
                const float2 s01 = mul2(unpack_bf16(raw.x), e2), s23 = mul2(unpack_bf16(raw.y), e2);
                a01 = fma2(k2, s01, a01);
                a23 = fma2(k2, s23, a23);
                q01 = fma2(q2, s01, q01);
                q23 = fma2(q2, s23, q23);
            }
            *reinterpret_cast<float4 *>(&red[warp][0][v0]) = make_float4(a01.x, a01.y, a23.x, a23.y);
            *reinterpret_cast<float4 *>(&red[warp][1][v0]) = make_float4(q01.x, q01.y, q23.x, q23.y);
            __syncthreads();
            if (tid < DV) {  // column v = tid: r = v - kn^T S', o = K^-0.5 (qn^T S' + beta (qn . kn) r)
                float ka = red[0][0][tid], qa = red[0][1][tid];
#pragma unroll
                for (int w = 1; w < NW; ++w) {
                    ka = __fadd_rn(ka, red[w][0][tid]);
                    qa = __fadd_rn(qa, red[w][1][tid]);
                }
                const float r = __fsub_rn(cur.vv, ka);
                rr[tid] = r;
                const float ov = __fmul_rn(0.08838834764831845f, __fmaf_rn(__fmul_rn(cur.be, qk[0]), r, qa));
                ob[tid] = __float2bfloat16_rn(ov);
                if (tid == 0) qk[1] = cur.be;
            }
            __syncthreads();
            // S'' = S' + beta kn r^T as bf16, in place in the stage (S' recomputed from the same bf16 values)
            const float be = qk[1];
            const float4 r4 = *reinterpret_cast<const float4 *>(rr + v0);
            const float2 r01 = make_float2(r4.x, r4.y), r23 = make_float2(r4.z, r4.w);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                uint2 *pw = reinterpret_cast<uint2 *>(blk + ((k0 + r) * DV + v0) * 2);
                const uint2 raw = *pw;
                const float4 c = rowc[k0 + r];
                const float2 e2 = make_float2(c.x, c.x);
                const float bk = __fmul_rn(be, c.y);
                const float2 b2 = make_float2(bk, bk);
                const float2 w01 = fma2(b2, r01, mul2(unpack_bf16(raw.x), e2));
                const float2 w23 = fma2(b2, r23, mul2(unpack_bf16(raw.y), e2));
                *pw = make_uint2(pack_bf16(w01.x, w01.y), pack_bf16(w23.x, w23.y));
            }
            fence_proxy_async();
            __syncthreads();
            if (tid == 0) {
                bulk_store(block_of(u, slot_cur), sb + S::RING + st * kDecodeBlockBytes, kDecodeBlockBytes);
                bulk_commit();
                stored = true;
            }
        }
        cur = nxt;
        slot_cur = slot_nxt;
        slot_nxt = slot_far;
    }
    if (tid == 0) {
        if (!ok) {
            atomicOr(p.err, ERR_TMA_WAIT);
            // the look-ahead copy may still land: wait for it (bounded) before the CTA leaves
            for (int st = 0; st < STAGES; ++st)
                if (pend >> st & 1) mbar_wait(sb + S::BAR + 8 * st, (phases >> st) & 1);
        }
        bulk_wait_read();  // the stages must outlive the stores' reads
    }
    __syncthreads();
}

}  // namespace kda
