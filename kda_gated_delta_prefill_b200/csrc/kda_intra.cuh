// kda_intra.cuh -- intra-chunk kernel: everything of the chunk construction
// that does not depend on the carried state, for one (chunk, value head)
// item per CTA, fully parallel over items.
//
// "KDA Chunk Prefill on Ascend A3", section "Mathematical definition": for a
// chunk of 64 tokens with inclusive per-channel cumulative gate G,
//   L_ij   = beta_i sum_d k_id k_jd exp(G_id - G_jd)   (j < i)
//   Aqk_ij = K^-0.5 sum_d q_id k_jd exp(G_id - G_jd)   (j <= i)
//   A = (I + L)^-1 diag(beta),  W = A (exp(G) k),  U = A v,
//   Qg = K^-0.5 q exp(G),  Kg = k exp(G_last - G),  and exp(G_last).
// The item's results -- -W, Qg, Kg, Aqk, U^T (fp16) and exp(G_last) (fp32) --
// are written as one contiguous block in the 128-byte-swizzled operand
// layouts the carry kernel's tensor-core descriptors read, so the carry
// kernel copies it into shared memory with one bulk copy.
//
// Steps inside the CTA (256 threads):
//   1. TMA tile loads of q, k (Q/K head h / (HV/H)), v, g; beta by plain
//      loads.  Rows past the end of the sequence are zeroed (the page's zero
//      padding of a partial chunk).
//   2. L2 normalisation of q and k in place (exact rounding order).
//   3. Gate factors from e_u = exp(g_u), one exponential per gate element:
//      within each 16-token block the inclusive running product base_i and
//      the exclusive suffix product b_j, block products P_J, and
//      per-channel factors built from them, so that for i >= j
//      exp(G_i - G_j) = base_i * (c_IJ * b_j) with every factor <= 1 except the
//      diagonal-block c_II = 1/P_I (then c_II * b_j = 1/base_j <= e^75).
//   4. L and Aqk: bf16 tensor-core MMAs over the ten lower 16x16 block pairs
//      (bf16 keeps the range of the gate-rescaled operands).
//   5. A: exact float32 forward substitution in the 16x16 diagonal blocks,
//      tf32 MMAs for the blocks next to them and then for the lower-left
//      32x32 block as -X_B (L_C X_A).
//   6. W and U^T: fp16 tensor-core MMAs.
// Results go straight from registers to the item block in global memory
// (coalesced rows), so the CTA needs about 105 KB of shared memory and two
// CTAs share an SM.
#pragma once
#include "kda_common.cuh"
#include "kda_norm.cuh"
#include "ptx.cuh"

namespace kda {

struct IntraSmem {
    static constexpr int Q = 0;          // bf16 [64][128] (two SW128 halves): q -> normalised -> K^-0.5 q*base; X (step 5)
    static constexpr int K = 16384;      // bf16: k -> normalised -> k*base; A fp16 [64][64] (step 5)
    static constexpr int V = 32768;      // bf16 v -> fp16 v
    static constexpr int G = 49152;      // fp32 [64][128] g; then KEXP fp16 (first half) and KBB bf16 (second half)
    static constexpr int KEXP = G;
    static constexpr int KBB = G + 16384;
    static constexpr int L = 81920;      // fp32 [64][64]
    static constexpr int X = Q;          // fp32 [64][64], once q*base is no longer needed
    static constexpr int A = K;          // fp16 [64][64], once k*base is no longer needed
    static constexpr int WST = Q;        // fp16 -W staging (step 6), once X is no longer needed
    static constexpr int UST = L;        // fp16 U^T staging (step 6), once L is no longer needed
    static constexpr int BETA = 98304;   // fp32 [64]
    static constexpr int CF = 98560;     // bf16x2 [10][64] block-pair factors
    static constexpr int PS = 101120;    // float2 [4][64] block products; later float [32][40] (over PS and TS)
    static constexpr int TS = 103168;    // fp32 8 x [16][8] solve scratch
    static constexpr int BAR = 107776;   // mbarriers: q/k/g tiles, v tile
    static constexpr int TOTAL = 107848;
};

struct IntraParams {
    const float *beta;
    const int32_t *cu;         // [N+1] or null
    const int32_t *chunk_off;  // [N+1] chunk offsets of the packed sequences, or null
    uint8_t *items;            // [num_chunks][HV] item blocks
    unsigned *err;
    int B, T, H, HV, N;
    int chunks_per_seq;        // ceil(T/64) when cu is null
    int chunk_begin;           // cu null: this launch covers chunks [chunk_begin, chunk_begin + chunk_count)
    int chunk_count;           //   of every sequence (cu given: all chunks, chunk_begin = 0)
    int prefetch_stride;       // CTAs resident at once (L2 prefetch distance), 0 = no prefetch
    // cu given, optional: this launch covers one chunk window, chunks [win_begin, ...) of every sequence, with
    // win_off[n] = the window's chunks in the sequences before n and win_off[N] = its total
    const int32_t *win_off;
    int win_begin;
    // optional: only value heads [h_begin, h_begin + h_count) (h_count 0: all)
    int h_begin, h_count;
};

// Off-diagonal block of X = (I+L)^-1, columns 16J+8nt .. +7:
//   X_IJ = -D_I * sum_{M=J}^{I-1} L_IM X_MJ   (D_I = X_II; one warp, tf32 MMAs),
// written as fp32 X (for later blocks) and as fp16 A = X diag(beta) (for W and U).
// ts: this warp's [16][8] float scratch for the intermediate sum.
__device__ __forceinline__ void solve_block(const uint8_t *sL, uint8_t *sX, uint8_t *sA, const float *beta, float *ts, int I,
                                            int J, int nt, int lane)
{
    const int g = lane >> 2, t = lane & 3;
    auto Lat = [&](int r, int c) { return *reinterpret_cast<const float *>(sL + swz(r, c * 4, 256)); };
    auto Xat = [&](int r, int c) { return *reinterpret_cast<const float *>(sX + swz(r, c * 4, 256)); };
    const int cn = 16 * J + 8 * nt + g;  // this lane's column of the B fragments
    float acc[4] = {};
    for (int M = J; M < I; ++M) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t a[4];
            a[0] = to_tf32(Lat(16 * I + g, 16 * M + 8 * ks + t));
            a[1] = to_tf32(Lat(16 * I + g + 8, 16 * M + 8 * ks + t));
            a[2] = to_tf32(Lat(16 * I + g, 16 * M + 8 * ks + t + 4));
            a[3] = to_tf32(Lat(16 * I + g + 8, 16 * M + 8 * ks + t + 4));
            mma_tf32(acc, a, to_tf32(Xat(16 * M + 8 * ks + t, cn)), to_tf32(Xat(16 * M + 8 * ks + t + 4, cn)));
        }
    }
    ts[g * 8 + 2 * t] = acc[0];
    ts[g * 8 + 2 * t + 1] = acc[1];
    ts[(g + 8) * 8 + 2 * t] = acc[2];
    ts[(g + 8) * 8 + 2 * t + 1] = acc[3];
    __syncwarp();
    float x[4] = {};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[4];
        a[0] = to_tf32(Xat(16 * I + g, 16 * I + 8 * ks + t));
        a[1] = to_tf32(Xat(16 * I + g + 8, 16 * I + 8 * ks + t));
        a[2] = to_tf32(Xat(16 * I + g, 16 * I + 8 * ks + t + 4));
        a[3] = to_tf32(Xat(16 * I + g + 8, 16 * I + 8 * ks + t + 4));
        mma_tf32(x, a, to_tf32(ts[(8 * ks + t) * 8 + g]), to_tf32(ts[(8 * ks + t + 4) * 8 + g]));
    }
    const int c = 16 * J + 8 * nt + 2 * t;
    *reinterpret_cast<float2 *>(sX + swz(16 * I + g, c * 4, 256)) = make_float2(-x[0], -x[1]);
    *reinterpret_cast<float2 *>(sX + swz(16 * I + g + 8, c * 4, 256)) = make_float2(-x[2], -x[3]);
    // A = X diag(beta) in fp16 for step 6
    const float b0 = beta[c], b1 = beta[c + 1];
    *reinterpret_cast<uint32_t *>(sA + swz(16 * I + g, c * 2, 128)) = pack_f16(-x[0] * b0, -x[1] * b1);
    *reinterpret_cast<uint32_t *>(sA + swz(16 * I + g + 8, c * 2, 128)) = pack_f16(-x[2] * b0, -x[3] * b1);
    __syncwarp();
}

constexpr int kIntraCtasPerSm = 2;  // the shared-memory footprint and register cap let two CTAs share an SM

__global__ void __launch_bounds__(256, kIntraCtasPerSm)
    kda_intra_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tg,
                     const IntraParams p)
{
    using S = IntraSmem;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;

    // ---- launch-local chunk -> (item chunk index, row of the chunk start, valid rows); false past the end ----
    const int32_t *offs = p.cu ? (p.win_off ? p.win_off : p.chunk_off) : nullptr;
    const int nchunks = p.cu ? offs[p.N] : p.B * p.chunk_count;
    auto locate = [&](int local, int &ci, int64_t &row0, int &nvalid) {
        if (local >= nchunks) return false;
        if (p.cu) {
            int lo = 0, hi = p.N - 1;  // last n with offs[n] <= local: the sequence that holds it
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (offs[mid] <= local) lo = mid; else hi = mid - 1;
            }
            const int c = (p.win_off ? p.win_begin : 0) + local - offs[lo];
            ci = p.chunk_off[lo] + c;
            const int len = p.cu[lo + 1] - p.cu[lo];
            row0 = p.cu[lo] + static_cast<int64_t>(c) * CH;
            nvalid = min(CH, len - c * CH);
        } else {
            const int b = local / p.chunk_count, c = p.chunk_begin + local % p.chunk_count;
            ci = b * p.chunks_per_seq + c;
            row0 = static_cast<int64_t>(b) * p.T + static_cast<int64_t>(c) * CH;
            nvalid = min(CH, p.T - c * CH);
        }
        return true;
    };
    const int nh = p.h_count ? p.h_count : p.HV;  // value heads this launch covers, from h_begin
    const int h = p.h_begin + static_cast<int>(blockIdx.x % nh);
    int ci;
    int64_t row0;
    int nvalid;
    if (!locate(blockIdx.x / nh, ci, row0, nvalid)) return;
    const int hq = h / (p.HV / p.H);
    uint8_t *out = p.items + (static_cast<int64_t>(ci) * p.HV + h) * ITEM_BYTES;  // item block (global)

    // ---- 1. loads ----
    const uint32_t bar = sb + S::BAR;
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 8, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_expect_tx(bar, 2 * 16384 + 32768);
        mbar_expect_tx(bar + 8, 16384);
        const int z = static_cast<int>(row0);
        tma_load_3d(sb + S::Q, &tq, 0, hq, z, bar);
        tma_load_3d(sb + S::Q + 8192, &tq, 64, hq, z, bar);
        tma_load_3d(sb + S::K, &tk, 0, hq, z, bar);
        tma_load_3d(sb + S::K + 8192, &tk, 64, hq, z, bar);
        tma_load_3d(sb + S::V, &tv, 0, h, z, bar + 8);
        tma_load_3d(sb + S::V + 8192, &tv, 64, h, z, bar + 8);
        tma_load_3d(sb + S::G, &tg, 0, h, z, bar);
        // The CTA that takes this slot after the current wave of resident CTAs will want item
        // blockIdx.x + prefetch_stride: pull its inputs into L2 now, so that its loads overlap the compute
        // of this wave instead of waiting on DRAM.
        const int pi = blockIdx.x + p.prefetch_stride;
        int pci, pvalid;
        int64_t prow;
        if (p.prefetch_stride > 0 && pi < static_cast<int>(gridDim.x) && locate(pi / nh, pci, prow, pvalid)) {
            const int ph = p.h_begin + pi % nh, pz = static_cast<int>(prow), phq = ph / (p.HV / p.H);
            tma_prefetch_3d(&tq, 0, phq, pz);
            tma_prefetch_3d(&tq, 64, phq, pz);
            tma_prefetch_3d(&tk, 0, phq, pz);
            tma_prefetch_3d(&tk, 64, phq, pz);
            tma_prefetch_3d(&tv, 0, ph, pz);
            tma_prefetch_3d(&tv, 64, ph, pz);
            tma_prefetch_3d(&tg, 0, ph, pz);
        }
    }
    float *sbeta = reinterpret_cast<float *>(sm + S::BETA);
    if (tid < CH) sbeta[tid] = (tid < nvalid) ? p.beta[(row0 + tid) * p.HV + h] : 0.f;
    if (!mbar_wait(bar, 0)) {
        atomicOr(p.err, ERR_TMA_WAIT);
        return;
    }
    if (nvalid < CH) {  // zero the padding rows of a partial chunk (q, k, g; v once it has arrived)
        for (int idx = tid; idx < (CH - nvalid) * 48; idx += 256) {
            const int r = nvalid + idx / 48, w = idx % 48;  // 16-byte words: q 16, k 16, g 32 (two per step)
            uint4 *dst;
            if (w < 32) {
                const int buf = w / 16, c16 = w % 16;  // q, k: two halves of 8 chunks
                dst = reinterpret_cast<uint4 *>(sm + buf * 16384 + (c16 >> 3) * 8192 + r * 128 + ((c16 & 7) << 4));
            } else {
                dst = reinterpret_cast<uint4 *>(sm + S::G + r * 512 + (w - 32) * 16);
                dst[16] = make_uint4(0, 0, 0, 0);
            }
            *dst = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();

    // ---- 2. normalise q and k (thread = row half) ----
    {
        const int r = tid >> 1, half = tid & 1;
        uint8_t *tile = sm + (r < CH ? S::Q : S::K) + half * 8192 + (r & 63) * 128;
        const int rs = r & 7;
        uint4 raw[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) raw[c] = *reinterpret_cast<const uint4 *>(tile + ((c ^ rs) << 4));
        l2norm_half_row(raw);  // the routine the standalone kda_l2norm_bf16 kernel runs
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(tile + ((c ^ rs) << 4)) = raw[c];
    }
    __syncthreads();

    // ---- 3. gate factors and operands: warp = (block J, channel half), lane = channel pair ----
    {
        const int J = warp & 3, dp = 32 * (warp >> 2) + lane, d0 = 2 * dp;
        float2 e[16], bb[16];
        const float2 l2e = make_float2(1.4426950408889634f, 1.4426950408889634f);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const float2 gv = *reinterpret_cast<const float2 *>(sm + S::G + (16 * J + u) * 512 + d0 * 4);
            const float2 y = mul2(gv, l2e);
            e[u] = make_float2(ex2_ftz(y.x), ex2_ftz(y.y));
        }
        bb[15] = make_float2(1.f, 1.f);
#pragma unroll
        for (int u = 14; u >= 0; --u) bb[u] = mul2(bb[u + 1], e[u + 1]);
#pragma unroll
        for (int u = 1; u < 16; ++u) e[u] = mul2(e[u - 1], e[u]);  // e -> inclusive running product (base)
        float2 *ps = reinterpret_cast<float2 *>(sm + S::PS);
        ps[J * 64 + dp] = e[15];  // block product P_J of this channel pair
        __syncthreads();          // every g read is done (the G region becomes KEXP / KBB); P visible
        float2 P[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) P[j] = ps[j * 64 + dp];
        // E_J = prod_{J'<J} P_J' (gate from the chunk start to the block start), F_J = prod_{J'>J} P_J'
        const float2 one2 = make_float2(1.f, 1.f);
        const float2 P01 = mul2(P[0], P[1]), P23 = mul2(P[2], P[3]);
        const float2 myE = (J == 0) ? one2 : (J == 1) ? P[0] : (J == 2) ? P01 : mul2(P01, P[2]);
        const float2 myF = (J == 3) ? one2 : (J == 2) ? P[3] : (J == 1) ? P23 : mul2(P[1], P23);
        const float scale = 0.08838834764831845f;  // 128^-0.5 in float32
        const float2 s2 = make_float2(scale, scale);
        if (J == 0) {
            // per-channel factors of the ten block pairs, as bf16 pairs; c_II = 1/P_I
            uint32_t *cf = reinterpret_cast<uint32_t *>(sm + S::CF);
            auto rcp2 = [](float2 a) {
                return make_float2(__frcp_rn(fmaxf(a.x, 1e-37f)), __frcp_rn(fmaxf(a.y, 1e-37f)));
            };
            const float2 cv[10] = {rcp2(P[0]), one2, rcp2(P[1]), P[1], one2, rcp2(P[2]), mul2(P[1], P[2]), P[2], one2,
                                   rcp2(P[3])};
#pragma unroll
            for (int pi = 0; pi < 10; ++pi) cf[pi * 64 + dp] = pack_bf16(cv[pi].x, cv[pi].y);
            *reinterpret_cast<float2 *>(out + ITEM_GL + d0 * 4) = mul2(P01, P23);
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int i = 16 * J + u;
            const uint32_t a16 = lh(i, d0);
            const float2 xk = unpack_bf16(*reinterpret_cast<const uint32_t *>(sm + S::K + a16));
            const float2 xq = unpack_bf16(*reinterpret_cast<const uint32_t *>(sm + S::Q + a16));
            const float2 kb = mul2(xk, e[u]);
            const float2 qb = mul2(xq, mul2(e[u], s2));
            const float2 kx = mul2(kb, myE);
            const float2 qg = mul2(qb, myE);
            const float2 kbb = mul2(xk, bb[u]);
            const float2 kg = mul2(kbb, myF);
            *reinterpret_cast<uint32_t *>(sm + S::K + a16) = pack_bf16(kb.x, kb.y);
            *reinterpret_cast<uint32_t *>(sm + S::Q + a16) = pack_bf16(qb.x, qb.y);
            *reinterpret_cast<uint32_t *>(sm + S::KEXP + a16) = pack_f16(kx.x, kx.y);
            *reinterpret_cast<uint32_t *>(sm + S::KBB + a16) = pack_bf16(kbb.x, kbb.y);
            *reinterpret_cast<uint32_t *>(out + ITEM_QG + a16) = pack_f16(qg.x, qg.y);
            *reinterpret_cast<uint32_t *>(out + ITEM_KG + a16) = pack_f16(kg.x, kg.y);
        }
    }
    __syncthreads();

    // ---- 4. L and Aqk over the ten lower block pairs x two 8-column tiles (bf16 MMAs).  A warp takes the
    //         tiles of one row block I and a run of column blocks J, loading its q and k fragments once per
    //         k-step for all of them; the 20 tiles split 2-2-2-2-3-3-3-3 over the warps:
    //         warps 0-3: I = 3, J in {0,1} / {2,3};  warps 4-5: I = 2, J in {0,1,2};
    //         warps 6-7: I = 1, J in {0,1}, then I = 0, J = 0.  nt = warp & 1. ----
    {
        const int nt = warp & 1;
        const int mi = lane >> 3;
        auto tiles = [&](int I, int J0, int nJ) {
            const uint32_t *cf = reinterpret_cast<const uint32_t *>(sm + S::CF) + (I * (I + 1) / 2 + J0) * 64;
            float accL[3][4] = {}, accQ[3][4] = {};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t ak[4], aq[4];
                const int ar = 16 * I + (mi & 1) * 8 + (lane & 7), ac = 16 * ks + (mi >> 1) * 8;
                ldsm_x4(sb + S::K + lh(ar, ac), ak[0], ak[1], ak[2], ak[3]);
                ldsm_x4(sb + S::Q + lh(ar, ac), aq[0], aq[1], aq[2], aq[3]);
#pragma unroll
                for (int jj = 0; jj < 3; ++jj) {
                    if (jj >= nJ) continue;
                    uint32_t b0, b1;
                    ldsm_x2(sb + S::KBB + lh(16 * (J0 + jj) + 8 * nt + (lane & 7), 16 * ks + (mi & 1) * 8), b0, b1);
                    // the pair's per-channel factor scales the key side: b0 holds channels 2t,2t+1, b1 2t+8,2t+9
                    b0 = hmul2_bf16(b0, cf[jj * 64 + 8 * ks + t4]);
                    b1 = hmul2_bf16(b1, cf[jj * 64 + 8 * ks + 4 + t4]);
                    mma_bf16(accL[jj], ak, b0, b1);
                    mma_bf16(accQ[jj], aq, b0, b1);
                }
            }
#pragma unroll
            for (int jj = 0; jj < 3; ++jj) {
                if (jj >= nJ) continue;
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int i = 16 * I + g8 + 8 * hr;
                    const int j = 16 * (J0 + jj) + 8 * nt + 2 * t4;
                    const float bi = sbeta[i];
                    const float l0 = (j < i) ? bi * accL[jj][2 * hr] : 0.f;
                    const float l1 = (j + 1 < i) ? bi * accL[jj][2 * hr + 1] : 0.f;
                    const float q0 = (j <= i) ? accQ[jj][2 * hr] : 0.f;
                    const float q1 = (j + 1 <= i) ? accQ[jj][2 * hr + 1] : 0.f;
                    *reinterpret_cast<float2 *>(sm + S::L + swz(i, j * 4, 256)) = make_float2(l0, l1);
                    *reinterpret_cast<uint32_t *>(out + ITEM_AQK + swz(i, j * 2, 128)) = pack_f16(q0, q1);
                }
            }
        };
        if (warp < 4) {
            tiles(3, 2 * (warp >> 1), 2);
        } else if (warp < 6) {
            tiles(2, 0, 3);
        } else {
            tiles(1, 0, 2);
            tiles(0, 0, 1);
        }
    }
    // The carry kernel multiplies the whole 64x64 Aqk tile: its six upper 16x16 blocks must be zeros.
    for (int idx = tid; idx < 6 * 16 * 8; idx += 256) {
        const int blk = idx >> 7, r = (idx >> 3) & 15, w = idx & 7;  // block, row in block, 4-byte word in block row
        const int I = (blk < 3) ? 0 : (blk < 5) ? 1 : 2;
        const int J = (blk < 3) ? blk + 1 : (blk < 5) ? blk - 1 : 3;
        const int i = 16 * I + r, j = 16 * J + 2 * w;
        *reinterpret_cast<uint32_t *>(out + ITEM_AQK + swz(i, j * 2, 128)) = 0u;
    }
    __syncthreads();

    // ---- 5. A = (I+L)^-1 diag(beta) ----
    uint8_t *sX = sm + S::X;  // overlays q*base, dead after step 4
    {  // diagonal blocks: exact float32 forward substitution on all 256 threads.  Thread = (block I, column c,
       // row group r4 owning rows r4, r4+4, r4+8, r4+12); the four threads of a column are adjacent lanes.
       // Right-looking: row m, once final, is broadcast to the column's lanes and updates every later row,
       // each row accumulating its terms in the order m = 0, 1, ...
        const int I = tid >> 6, c = (tid >> 2) & 15, r4 = tid & 3;
        const uint8_t *sLb = sm + S::L;
        float x[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) x[q] = (4 * q + r4 == c) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < 15; ++m) {
            const float xm = __shfl_sync(0xffffffffu, x[m >> 2], (lane & ~3) | (m & 3));
#pragma unroll
            for (int q = m >> 2; q < 4; ++q) {
                const int j = 4 * q + r4;
                const float l = *reinterpret_cast<const float *>(sLb + swz(16 * I + j, (16 * I + m) * 4, 256));
                if (j > m) x[q] = __fmaf_rn(-l, xm, x[q]);
            }
        }
        const float bc = sbeta[16 * I + c];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int j = 4 * q + r4;
            *reinterpret_cast<float *>(sX + swz(16 * I + j, (16 * I + c) * 4, 256)) = x[q];
            // A = X diag(beta) in fp16, zero above the diagonal (step 6 multiplies whole diagonal blocks)
            *reinterpret_cast<__half *>(sm + S::A + swz(16 * I + j, (16 * I + c) * 2, 128)) =
                __float2half_rn(j >= c ? x[q] * bc : 0.f);
        }
    }
    __syncthreads();
    {  // blocks next to the diagonal (X_10, X_21, X_32); one warp per (block, 8-column tile)
        float *ts = reinterpret_cast<float *>(sm + S::TS) + warp * 128;
        if (warp < 6) solve_block(sm + S::L, sX, sm + S::A, sbeta, ts, (warp >> 1) + 1, warp >> 1, warp & 1, lane);
        __syncthreads();
    }
    {  // the rest as 32x32 blocks: with X_A = X[0..31][0..31] and X_B = X[32..63][32..63] now complete,
       // X[32..63][0..31] = -X_B (L[32..63][0..31] X_A).  Warp = 16x8 output tile, tf32 MMAs; the 16x16
       // blocks above the diagonal of X_A and X_B are zero and skipped.
        const int mt = warp >> 2, nt = warp & 3;
        float *sT = reinterpret_cast<float *>(sm + S::PS);  // [32][40] floats over PS and TS
        auto Lat = [&](int r, int cc) { return *reinterpret_cast<const float *>(sm + S::L + swz(r, cc * 4, 256)); };
        auto Xat = [&](int r, int cc) { return *reinterpret_cast<const float *>(sX + swz(r, cc * 4, 256)); };
        float d[4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            if (nt >= 2 && ks < 2) continue;  // X_A[0..15][16..31] = 0
            uint32_t a[4];
            a[0] = to_tf32(Lat(32 + 16 * mt + g8, 8 * ks + t4));
            a[1] = to_tf32(Lat(32 + 16 * mt + g8 + 8, 8 * ks + t4));
            a[2] = to_tf32(Lat(32 + 16 * mt + g8, 8 * ks + t4 + 4));
            a[3] = to_tf32(Lat(32 + 16 * mt + g8 + 8, 8 * ks + t4 + 4));
            mma_tf32(d, a, to_tf32(Xat(8 * ks + t4, 8 * nt + g8)), to_tf32(Xat(8 * ks + t4 + 4, 8 * nt + g8)));
        }
        *reinterpret_cast<float2 *>(sT + (16 * mt + g8) * 40 + 8 * nt + 2 * t4) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2 *>(sT + (16 * mt + g8 + 8) * 40 + 8 * nt + 2 * t4) = make_float2(d[2], d[3]);
        __syncthreads();
        float e[4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            if (mt == 0 && ks >= 2) continue;  // X_B[0..15][16..31] = 0
            uint32_t a[4];
            a[0] = to_tf32(Xat(32 + 16 * mt + g8, 32 + 8 * ks + t4));
            a[1] = to_tf32(Xat(32 + 16 * mt + g8 + 8, 32 + 8 * ks + t4));
            a[2] = to_tf32(Xat(32 + 16 * mt + g8, 32 + 8 * ks + t4 + 4));
            a[3] = to_tf32(Xat(32 + 16 * mt + g8 + 8, 32 + 8 * ks + t4 + 4));
            mma_tf32(e, a, to_tf32(sT[(8 * ks + t4) * 40 + 8 * nt + g8]), to_tf32(sT[(8 * ks + t4 + 4) * 40 + 8 * nt + g8]));
        }
        // only A = X diag(beta) is needed from here on
        const int cc = 8 * nt + 2 * t4;
        const float b0 = sbeta[cc], b1 = sbeta[cc + 1];
        *reinterpret_cast<uint32_t *>(sm + S::A + swz(32 + 16 * mt + g8, cc * 2, 128)) = pack_f16(-e[0] * b0, -e[1] * b1);
        *reinterpret_cast<uint32_t *>(sm + S::A + swz(32 + 16 * mt + g8 + 8, cc * 2, 128)) = pack_f16(-e[2] * b0, -e[3] * b1);
    }
    __syncthreads();

    // ---- v tile (its copy overlapped steps 2-5): zero padding rows, bf16 -> fp16 in place ----
    if (!mbar_wait(bar + 8, 0)) {
        atomicOr(p.err, ERR_TMA_WAIT);
        return;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int idx = tid + 256 * k;  // 16-byte chunk: half (idx >> 9), row ((idx >> 3) & 63)
        uint4 *pv = reinterpret_cast<uint4 *>(sm + S::V) + idx;
        uint4 u = *pv;
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
        const bool pad = ((idx >> 3) & 63) >= nvalid;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 x = unpack_bf16(w[j]);
            w[j] = pad ? 0u : pack_f16(x.x, x.y);
        }
        *pv = make_uint4(w[0], w[1], w[2], w[3]);
    }
    __syncthreads();

    // ---- 6. -W = -A (exp(G) k) (warp = 16 key columns) and U^T = v^T A^T (warp = 16 value rows); fp16 MMAs.
    //         Each 16x16 tile of A is loaded once: as the A operand of W, and, with its fragment registers
    //         reordered, as the two B fragments (8 rows of A each) of U^T. ----
    {
        const int mi = lane >> 3;
        // U^T A operand: v^T rows 16*warp .. +15 for the four 16-token K steps (ldmatrix.trans of v)
        uint32_t av[4][4];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const int tok = 16 * ks + (mi >> 1) * 8 + (lane & 7), col = 16 * warp + (mi & 1) * 8;
            ldsm_x4_t(sb + S::V + lh(tok, col), av[ks][0], av[ks][1], av[ks][2], av[ks][3]);
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            float w[2][4] = {}, u[2][4] = {};
            for (int ks = 0; ks <= mt; ++ks) {
                uint32_t a[4];  // A rows 16mt + (g, g+8), columns 16ks + (2t, 2t+8)
                ldsm_x4(sb + S::A + swz(16 * mt + (mi & 1) * 8 + (lane & 7), (16 * ks + (mi >> 1) * 8) * 2, 128), a[0], a[1],
                        a[2], a[3]);
                const int tok = 16 * ks + (mi & 1) * 8 + (lane & 7), col = 16 * warp + (mi >> 1) * 8;
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(sb + S::KEXP + lh(tok, col), b0, b1, b2, b3);
                mma_f16(w[0], a, b0, b1);
                mma_f16(w[1], a, b2, b3);
                // U^T[v][i] += v^T[v][j] A[i][j]: B fragment of rows i = 16mt + g is (a0, a2), of i + 8 is (a1, a3)
                mma_f16(u[0], av[ks], a[0], a[2]);
                mma_f16(u[1], av[ks], a[1], a[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int r = 16 * mt + g8 + 8 * hr;
                    const int c = 16 * warp + 8 * nt + 2 * t4;
                    *reinterpret_cast<uint32_t *>(sm + S::WST + lh(r, c)) = pack_f16(-w[nt][2 * hr], -w[nt][2 * hr + 1]);
                    const int vr = 16 * warp + g8 + 8 * hr;  // value row
                    const int tk = 16 * mt + 8 * nt + 2 * t4;  // token column
                    *reinterpret_cast<uint32_t *>(sm + S::UST + vr * 128 + (((tk >> 3) ^ (vr & 7)) << 4) + (tk & 7) * 2) =
                        pack_f16(u[nt][2 * hr], u[nt][2 * hr + 1]);
                }
        }
    }
    // -W and U^T leave through two bulk copies (their smem images match the item layout)
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
        bulk_store(out + ITEM_WN, sb + S::WST, 16384);
        bulk_store(out + ITEM_U, sb + S::UST, 16384);
        bulk_commit();
        bulk_wait_read();  // the shared-memory images must outlive the reads, not the global writes
    }
}

}  // namespace kda
