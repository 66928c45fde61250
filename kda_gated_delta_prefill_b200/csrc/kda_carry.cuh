// kda_carry.cuh -- inter-chunk state carry ("KDA Chunk Prefill on Ascend A3",
// section "Mathematical definition", last three formulas):
//   Vnew  = U - W S_in
//   O     = Qg S_in + Aqk Vnew
//   S_out = exp(G_last)[:,None] * S_in + Kg^T Vnew
// One CTA per (sequence, value head, slice of 16*NW value columns); the
// columns of S evolve independently, so slicing is exact.  Every consumer
// warp owns 16 value columns and keeps S^T for them in MMA accumulator
// registers (float32) for the whole sequence.  A producer warp streams the
// per-chunk blocks written by the intra-chunk kernel through a three-stage
// shared-memory ring with bulk copies and mbarriers.
#pragma once
#include "kda_common.cuh"
#include "ptx.cuh"

namespace kda {

template <int NW>
struct CarrySmem {
    static constexpr int VS = 16 * NW;
    static constexpr int U_BYTES = VS * CH * 2;                         // fp16 U columns of this slice
    static constexpr int U_OFF = ITEM_U;                                // stage image follows the item layout
    static constexpr int GL_OFF = ITEM_U + U_BYTES;
    static constexpr int STAGE = ((GL_OFF + 512) + 1023) / 1024 * 1024;
    static constexpr int NST = 3;
    static constexpr int VN_STRIDE = 48;                                // bytes per Vnew row (16 fp16 + pad)
    static constexpr int VN = NST * STAGE;
    static constexpr int BAR = VN + NW * CH * VN_STRIDE;
    static constexpr int TOTAL = BAR + 2 * NST * 8;
    static constexpr uint32_t TX = ITEM_U + U_BYTES + 512;
};

struct CarryParams {
    const uint8_t *items;
    const float *s0;           // [N,HV,K,V] or null
    const int32_t *cu;         // [N+1] or null
    const int32_t *chunk_off;  // [N+1] or null
    const int32_t *order;      // [N] longest-first, or null
    __nv_bfloat16 *o;
    float *sN;
    unsigned *err;
    int T, HV, N;
    int chunks_per_seq;
    int nslices;
};

template <int NW>
__global__ void __launch_bounds__((NW + 1) * 32, 1) kda_carry_kernel(const CarryParams p)
{
    using S = CarrySmem<NW>;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;

    const int slice = blockIdx.x % p.nslices;
    const int rest = blockIdx.x / p.nslices;
    const int h = rest % p.HV;
    const int r_idx = rest / p.HV;
    const int n = p.order ? p.order[r_idx] : r_idx;
    int64_t c_begin, tok0;
    int nck, len;
    if (p.cu) {
        c_begin = p.chunk_off[n];
        nck = p.chunk_off[n + 1] - p.chunk_off[n];
        tok0 = p.cu[n];
        len = p.cu[n + 1] - p.cu[n];
    } else {
        c_begin = static_cast<int64_t>(n) * p.chunks_per_seq;
        nck = p.chunks_per_seq;
        tok0 = static_cast<int64_t>(n) * p.T;
        len = p.T;
    }
    const int v0 = slice * S::VS;

    const uint32_t full0 = sb + S::BAR, empty0 = sb + S::BAR + S::NST * 8;
    if (tid == 0) {
        for (int s = 0; s < S::NST; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, NW);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == NW) {  // ---- producer ----
        if (lane == 0) {
            for (int c = 0; c < nck; ++c) {
                const int s = c % S::NST;
                if (c >= S::NST && !mbar_wait(empty0 + 8 * s, ((c / S::NST) - 1) & 1)) {
                    atomicOr(p.err, ERR_PIPE_EMPTY_WAIT);
                    return;
                }
                const uint8_t *item = p.items + ((c_begin + c) * p.HV + h) * ITEM_BYTES;
                const uint32_t dst = sb + s * S::STAGE;
                mbar_expect_tx(full0 + 8 * s, S::TX);
                bulk_load(dst, item, ITEM_U, full0 + 8 * s);
                bulk_load(dst + S::U_OFF, item + ITEM_U + slice * S::U_BYTES, S::U_BYTES, full0 + 8 * s);
                bulk_load(dst + S::GL_OFF, item + ITEM_GL, 512, full0 + 8 * s);
            }
        }
        return;
    }

    // ---- consumers: S^T for value columns vl = g8 + 8*(e>>1) of this warp, key kd = 8*nt + 2*t4 + (e&1) ----
    float sT[16][4];
    {
        const int vcol = v0 + 16 * warp + g8;
        const float *s0 = p.s0 ? p.s0 + (static_cast<int64_t>(n) * p.HV + h) * DK * DV : nullptr;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int kd = 8 * nt + 2 * t4 + (e & 1);
                sT[nt][e] = s0 ? s0[kd * DV + vcol + 8 * (e >> 1)] : 0.f;
            }
    }
    uint8_t *vn = sm + S::VN + warp * CH * S::VN_STRIDE;
    const uint32_t vn_s = smem_u32(vn);
    const int mi = lane >> 3;

    for (int c = 0; c < nck; ++c) {
        const int s = c % S::NST;
        if (!mbar_wait(full0 + 8 * s, (c / S::NST) & 1)) {
            atomicOr(p.err, ERR_PIPE_FULL_WAIT);
            return;
        }
        const uint8_t *st = sm + s * S::STAGE;
        const uint32_t st_s = sb + s * S::STAGE;
        const int nvalid = min(CH, len - c * CH);

        // U -> accumulators (becomes Vnew)
        float acc[4][2][4];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int nv = 0; nv < 2; ++nv)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int tok = 16 * mt + g8 + 8 * hr;
                    const int col = (warp & 1) * 16 + 8 * nv + 2 * t4;
                    const float2 u = unpack_f16(
                        *reinterpret_cast<const uint32_t *>(st + S::U_OFF + (warp >> 1) * 4096 + tok * 64 + col * 2));
                    acc[mt][nv][2 * hr] = u.x;
                    acc[mt][nv][2 * hr + 1] = u.y;
                }
        float oacc[4][2][4] = {};
        // Vnew = U + (-W) S ;  O = Qg S
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t bs[2][2];
#pragma unroll
            for (int nv = 0; nv < 2; ++nv) {
                bs[nv][0] = pack_f16(sT[2 * ks][2 * nv], sT[2 * ks][2 * nv + 1]);
                bs[nv][1] = pack_f16(sT[2 * ks + 1][2 * nv], sT[2 * ks + 1][2 * nv + 1]);
            }
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                const int r = 16 * mt + (mi & 1) * 8 + (lane & 7);
                const int cc = 16 * ks + (mi >> 1) * 8;
                uint32_t aw[4], aq[4];
                ldsm_x4(st_s + ITEM_WN + swz(r, cc * 2, 256), aw[0], aw[1], aw[2], aw[3]);
                ldsm_x4(st_s + ITEM_QG + swz(r, cc * 2, 256), aq[0], aq[1], aq[2], aq[3]);
#pragma unroll
                for (int nv = 0; nv < 2; ++nv) {
                    mma_f16(acc[mt][nv], aw, bs[nv][0], bs[nv][1]);
                    mma_f16(oacc[mt][nv], aq, bs[nv][0], bs[nv][1]);
                }
            }
        }
        // Vnew -> fp16 -> per-warp buffer [64 tok][16 v]
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int nv = 0; nv < 2; ++nv) {
                const int r = 16 * mt + g8;
                const int vc = 8 * nv + 2 * t4;
                *reinterpret_cast<uint32_t *>(vn + r * S::VN_STRIDE + vc * 2) = pack_f16(acc[mt][nv][0], acc[mt][nv][1]);
                *reinterpret_cast<uint32_t *>(vn + (r + 8) * S::VN_STRIDE + vc * 2) =
                    pack_f16(acc[mt][nv][2], acc[mt][nv][3]);
            }
        __syncwarp();
        // O += Aqk Vnew (causal: key blocks ks <= mt)
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            for (int ks = 0; ks <= mt; ++ks) {
                uint32_t a[4];
                ldsm_x4(st_s + ITEM_AQK + swz(16 * mt + (mi & 1) * 8 + (lane & 7), (16 * ks + (mi >> 1) * 8) * 2, 128),
                        a[0], a[1], a[2], a[3]);
                const int tok = 16 * ks + (mi & 1) * 8 + (lane & 7);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vn_s + tok * S::VN_STRIDE + (mi >> 1) * 16, b0, b1, b2, b3);
                mma_f16(oacc[mt][0], a, b0, b1);
                mma_f16(oacc[mt][1], a, b2, b3);
            }
        }
        // o rows of valid tokens (bf16)
        {
            __nv_bfloat16 *ob = p.o + ((tok0 + static_cast<int64_t>(c) * CH) * p.HV + h) * DV + v0 + 16 * warp;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int tok = 16 * mt + g8 + 8 * hr;
                    if (tok < nvalid) {
#pragma unroll
                        for (int nv = 0; nv < 2; ++nv)
                            *reinterpret_cast<uint32_t *>(ob + static_cast<int64_t>(tok) * p.HV * DV + 8 * nv + 2 * t4) =
                                pack_bf16(oacc[mt][nv][2 * hr], oacc[mt][nv][2 * hr + 1]);
                    }
                }
        }
        // S^T <- S^T diag(exp(G_last)) + Vnew^T Kg
        {
            const float *gl = reinterpret_cast<const float *>(st + S::GL_OFF);
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
                uint32_t a[4];
                ldsm_x4_t(vn_s + (16 * ks + (mi >> 1) * 8 + (lane & 7)) * S::VN_STRIDE + (mi & 1) * 16, a[0], a[1], a[2],
                          a[3]);
#pragma unroll
                for (int np = 0; np < 16; np += 2) {
                    const int tok = 16 * ks + (mi & 1) * 8 + (lane & 7);
                    const int kd = 8 * np + (mi >> 1) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(st_s + ITEM_KG + swz(tok, kd * 2, 256), b0, b1, b2, b3);
                    mma_f16(sT[np], a, b0, b1);
                    mma_f16(sT[np + 1], a, b2, b3);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
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

}  // namespace kda
