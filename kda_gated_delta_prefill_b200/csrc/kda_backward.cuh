// kda_backward.cuh -- backward of the KDA chunk prefill.
//
// "KDA Chunk Prefill on Ascend A3" leaves the backward optional (section
// "Timing and required submission") and fixes its loss, sum(o * do) +
// sum(final_state * dht), and its outputs, the gradients of q, k, v, g, beta
// and the initial state.  The chunk form of the forward (section
// "Mathematical definition") is differentiated one chunk at a time.  For a
// chunk with start state S, inclusive cumulative gate G (last row G_L),
// E = diag(exp G_L), normalised rows qn/kn and s = K^-0.5:
//   P_ij  = sum_d kn_id kn_jd exp(G_id - G_jd) (j < i),  L = diag(beta) P
//   Aqk   = s sum_d qn_id kn_jd exp(G_id - G_jd) (j <= i)
//   T     = (I + L)^-1,  A = T diag(beta),  Kb = kn exp(G),  Kg = kn exp(G_L - G)
//   D     = v - Kb S,  Vnew = A D,  O = s qn exp(G) S + Aqk Vnew,  S' = E S + Kg^T Vnew
// Given dO and dS' (the gradient at the chunk's end state):
//   dVnew = Kg dS' + Aqk^T dO                dS    = E dS' + Qg^T dO - W^T dVnew  (W = A Kb)
//   dv    = A^T dVnew                        dA    = dVnew D^T
//   dQg   = dO S^T,  dKb = -dv S^T,  dKg = Vnew dS'^T,  dAqk = dO Vnew^T (j <= i)
//   dbeta_j += sum_i dA_ij T_ij,  dL = -T^T (dA diag beta) T^T (j < i),  dbeta_i += sum_j dL_ij P_ij
// and, with M = diag(beta) dL and N = dAqk, the pairwise terms
//   dkn_i += sum_j M_ij kn_j f_ij + sum_k M_ki kn_k f_ki + s sum_k N_ki qn_k f_ki,
//   dqn_i += s sum_j N_ij kn_j f_ij   (f_ij = exp(G_i - G_j) per channel),
// plus the elementwise terms through Qg, Kb and Kg, and dG, whose reverse
// cumulative sum is dg.  Three kernels:
//   kda_bwd_carry_kernel  dS' of every chunk, walking each sequence backwards
//                         (reads the forward's per-chunk blocks),
//   kda_bwd_chunk_kernel  every chunk's gradients at once (fp32 arithmetic,
//                         TF32 tensor-core MMAs for the products),
//   kda_bwd_norm_kernel   sums a Q/K head's group and applies the L2
//                         normalisation's Jacobian.
// Gate factors exp(G_i - G_j) are formed per 16-token block I with the
// reference m_I = G at the block's eighth token:
//   exp(G_i - G_j) = exp(G_i - m_I) * exp(m_I - m_J) * exp(m_J - G_j),
// every factor at most exp(8 |g|max) away from 1 and the middle one <= 1.
#pragma once
#include "kda_common.cuh"
#include "kda_norm.cuh"
#include "ptx.cuh"

namespace kda {

struct BwdParams {
    const __nv_bfloat16 *q, *k, *v, *dout;  // q, k: [rows][H][K]; v, dout: [rows][HV][V]
    const float *g, *beta;                  // [rows][HV][K], [rows][HV]
    const uint8_t *items;                   // the forward's per-(chunk, head) blocks
    const __nv_bfloat16 *states;            // [chunks][HV][K][V] bf16: state at each chunk's start
    __nv_bfloat16 *dstates;                 // [chunks][HV][K][V] bf16: gradient at each chunk's end state
    const float *dht;                       // [N][HV][K][V] or null (zero)
    float *dh0;                             // [N][HV][K][V] or null (not wanted)
    float *dqn, *dkn;                       // [rows][HV][K]: gradient at the normalised rows, per value head
    __nv_bfloat16 *dq, *dk, *dv;            // [rows][H][K], [rows][H][K], [rows][HV][V]
    float *dg, *dbeta;                      // [rows][HV][K], [rows][HV]
    const int32_t *cu, *chunk_off;          // packed sequences (cu [N+1], chunk_off [N+1]) or null
    unsigned *err;
    int T, H, HV, N, chunks_per_seq;
    // H == HV: the chunk kernel applies the normalisation's Jacobian itself and writes dq, dk (no dqn, dkn)
    int fuse_norm;
};

// (sequence, first token row, valid rows) of global chunk index `chunk`
__device__ __forceinline__ void bwd_locate(const BwdParams &p, int chunk, int &n, int64_t &row0, int &c_in_seq,
                                           int &nvalid)
{
    int len;
    if (p.cu) {
        int lo = 0, hi = p.N - 1;  // last sequence whose first chunk is <= chunk
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.chunk_off[mid] <= chunk) lo = mid;
            else hi = mid - 1;
        }
        n = lo;
        c_in_seq = chunk - p.chunk_off[n];
        row0 = p.cu[n] + static_cast<int64_t>(c_in_seq) * CH;
        len = p.cu[n + 1] - p.cu[n];
    } else {
        n = chunk / p.chunks_per_seq;
        c_in_seq = chunk - n * p.chunks_per_seq;
        row0 = static_cast<int64_t>(n) * p.T + static_cast<int64_t>(c_in_seq) * CH;
        len = p.T;
    }
    nvalid = min(CH, len - c_in_seq * CH);
}

__device__ __forceinline__ float bwd_exp(float x) { return ex2(x * 1.4426950408889634f); }

// ---------------------------------------------------------------------------------------------------------
// Reverse carry: one CTA (16 warps) per (sequence, value head, half of the value columns), on fp16 tensor-core
// MMAs (mma.sync m16n8k16, fp32 accumulate).  The fp32 gradient dS (128 keys x 64 columns) stays in the warps'
// accumulator registers; an fp16 copy in shared memory feeds the next chunk's Kg dS.  Chunk c's block (the -W,
// Qg, Kg, Aqk tiles in their SW128 layout, and exp(G_L)) arrives by bulk copy one chunk ahead.  Before chunk c
// is folded in, dS is the gradient at chunk c's end state and is stored for the chunk kernel.
constexpr int kBcThreads = 512, kBcCols = 64, kBcPad = 72;  // fp16 row stride (halves) of dS, dO, dVnew copies
struct BcSmem {
    static constexpr int PART = ITEM_U;                   // bytes [0, ITEM_U) of a block: -W, Qg, Kg, Aqk
    static constexpr int STAGE = PART + 512;              // + exp(G_L)
    static constexpr int DSH = 2 * STAGE;                 // fp16 [128][72]  dS
    static constexpr int DOH = DSH + DK * kBcPad * 2;     // fp16 [64][72]   dO
    static constexpr int DVH = DOH + CH * kBcPad * 2;     // fp16 [64][72]   dVnew
    static constexpr int DSB = DVH + CH * kBcPad * 2;     // bf16 [128][72]  dS, as stored for the chunk kernel
    static constexpr int BAR = DSB + DK * kBcPad * 2;     // mbarriers [2]
    static constexpr int FLAG = BAR + 16;
    static constexpr int TOTAL = FLAG + 16;
};
static_assert(ITEM_GL == ITEM_U + 16384, "block layout");

// byte offset of the 16-byte group (row r, columns c..c+7) of a [64][128] SW128 tile pair / a [64][64] tile
__device__ __forceinline__ uint32_t sw_off128(int r, int c)
{
    return static_cast<uint32_t>((c >> 6) * 8192 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint32_t sw_off64(int r, int c)
{
    return static_cast<uint32_t>(r * 128 + (((c >> 3) ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(kBcThreads, 1) kda_bwd_carry_kernel(const BwdParams p)
{
    using S = BcSmem;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    const int unit = blockIdx.x >> 1, vc0 = (blockIdx.x & 1) * kBcCols;
    const int n = unit / p.HV, h = unit % p.HV;
    int64_t c_begin, row0;
    int nck, len;
    if (p.cu) {
        c_begin = p.chunk_off[n];
        nck = p.chunk_off[n + 1] - p.chunk_off[n];
        row0 = p.cu[n];
        len = p.cu[n + 1] - p.cu[n];
    } else {
        c_begin = static_cast<int64_t>(n) * p.chunks_per_seq;
        nck = p.chunks_per_seq;
        row0 = static_cast<int64_t>(n) * p.T;
        len = p.T;
    }
    __half *dSh = reinterpret_cast<__half *>(sm + S::DSH);
    __half *dOh = reinterpret_cast<__half *>(sm + S::DOH);
    __half *dVh = reinterpret_cast<__half *>(sm + S::DVH);
    volatile int *flag = reinterpret_cast<volatile int *>(sm + S::FLAG);
    const int64_t unit_off = (static_cast<int64_t>(n) * p.HV + h) * DK * DV;

    // thread 0 bookkeeping: copies issued into / completions waited for, per stage
    int issued[2] = {0, 0}, waited[2] = {0, 0};
    auto request = [&](int c, int st) {  // thread 0: chunk c's block into stage st
        ++issued[st];
        const uint8_t *src = p.items + ((c_begin + c) * p.HV + h) * ITEM_BYTES;
        const uint32_t bar = sb + S::BAR + 8 * st, dst = sb + st * S::STAGE;
        mbar_expect_tx(bar, S::STAGE);
        bulk_load(dst, src, S::PART, bar);
        bulk_load(dst + S::PART, src + ITEM_GL, 512, bar);
    };
    if (tid == 0) {
        mbar_init(sb + S::BAR, 1);
        mbar_init(sb + S::BAR + 8, 1);
        fence_mbar_init();
        if (nck > 0) request(nck - 1, 0);
    }
    // the warp's dS tile: keys 16 ms .. +15, value columns 32 nh .. +31 of this CTA's 64 (four n8 tiles)
    const int ms = warp & 7, nh = warp >> 3;
    float acc[4][4];
    auto key_of = [&](int half) { return 16 * ms + g + 8 * half; };
    auto col_of = [&](int j, int e) { return 32 * nh + 8 * j + 2 * t4 + e; };
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            acc[j][q] = p.dht ? p.dht[unit_off + key_of(q >> 1) * DV + vc0 + col_of(j, q & 1)] : 0.f;
    // dS into shared memory: fp16 for the next chunk's MMAs, bf16 for the dstates row copy
    __nv_bfloat16 *dSb = reinterpret_cast<__nv_bfloat16 *>(sm + S::DSB);
    auto store_dsh = [&]() {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                *reinterpret_cast<__half2 *>(dSh + key_of(hf) * kBcPad + col_of(j, 0)) =
                    __floats2half2_rn(acc[j][2 * hf], acc[j][2 * hf + 1]);
                *reinterpret_cast<__nv_bfloat162 *>(dSb + key_of(hf) * kBcPad + col_of(j, 0)) =
                    __floats2bfloat162_rn(acc[j][2 * hf], acc[j][2 * hf + 1]);
            }
    };
    store_dsh();
    __syncthreads();

    // this thread's share of a chunk's dO rows (row tid / 8, eight columns), loaded one chunk ahead
    auto load_dout = [&](int c) {
        const int i = tid >> 3, cc = 8 * (tid & 7);
        uint4 raw = make_uint4(0u, 0u, 0u, 0u);
        if (c >= 0 && i < min(CH, len - c * CH))
            raw = *reinterpret_cast<const uint4 *>(p.dout + ((row0 + static_cast<int64_t>(c) * CH + i) * p.HV + h) * DV +
                                                   vc0 + cc);
        return raw;
    };
    auto put_dout = [&](uint4 raw) {  // as fp16 (zero past the sequence's end)
        const int i = tid >> 3, cc = 8 * (tid & 7);
        const uint4 w = make_uint4(pack_f16(bf16lo(raw.x), bf16hi(raw.x)), pack_f16(bf16lo(raw.y), bf16hi(raw.y)),
                                   pack_f16(bf16lo(raw.z), bf16hi(raw.z)), pack_f16(bf16lo(raw.w), bf16hi(raw.w)));
        *reinterpret_cast<uint4 *>(dOh + i * kBcPad + cc) = w;
    };
    if (nck > 0) put_dout(load_dout(nck - 1));  // visible after the first barrier below

    bool ok = true;
    for (int it = 0; it < nck; ++it) {
        const int c = nck - 1 - it, st = it & 1;
        const uint32_t blk = sb + st * S::STAGE;
        if (tid == 0 && c > 0) request(c - 1, st ^ 1);  // that stage was released by the previous iteration
        const uint4 next_dout = load_dout(c - 1);       // lands while this chunk computes
        if (tid == 0) {
            const bool landed = mbar_wait(sb + S::BAR + 8 * st, waited[st] & 1);
            if (landed) ++waited[st];
            flag[0] = landed;
        }
        __syncthreads();
        if (!flag[0]) {
            ok = false;
            break;
        }
        {
            // dS is the gradient at chunk c's end state: store its bf16 copy (written to shared memory before the
            // barrier above) as whole 128-byte rows, 16 bytes per thread
            __nv_bfloat16 *dst = p.dstates + ((c_begin + c) * p.HV + h) * DK * DV + vc0;
#pragma unroll
            for (int i = 0; i < DK * kBcCols / 8 / kBcThreads; ++i) {
                const int r = (tid >> 3) + i * (kBcThreads / 8), q = tid & 7;
                *reinterpret_cast<uint4 *>(dst + r * DV + 8 * q) =
                    *reinterpret_cast<const uint4 *>(dSb + r * kBcPad + 8 * q);
            }
        }
        const uint32_t dsh = smem_u32(dSh), doh = smem_u32(dOh), dvh = smem_u32(dVh);
        {
            // dVnew = Kg dS + Aqk^T dO; warp: tokens 16 mt .., columns 16 nq .. +15 (two n8 tiles)
            const int mt = warp & 3, nq = warp >> 2;
            float v[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t a[4], b[4];
                ldsm_x4(blk + ITEM_KG + sw_off128(16 * mt + (lane & 15), 16 * ks + (lane >> 4) * 8), a[0], a[1], a[2],
                        a[3]);
                ldsm_x4_t(dsh + 2 * ((16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8) * kBcPad + 16 * nq + (lane >> 4) * 8),
                          b[0], b[1], b[2], b[3]);
                mma_f16(v[0], a, b[0], b[1]);
                mma_f16(v[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4];
                ldsm_x4_t(blk + ITEM_AQK + sw_off64(16 * ks + (lane & 7) + ((lane >> 4) & 1) * 8,
                                                   16 * mt + ((lane >> 3) & 1) * 8),
                          a[0], a[1], a[2], a[3]);
                ldsm_x4_t(doh + 2 * ((16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8) * kBcPad + 16 * nq + (lane >> 4) * 8),
                          b[0], b[1], b[2], b[3]);
                mma_f16(v[0], a, b[0], b[1]);
                mma_f16(v[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                    *reinterpret_cast<__half2 *>(dVh + (16 * mt + g + 8 * hf) * kBcPad + 16 * nq + 8 * j + 2 * t4) =
                        __floats2half2_rn(v[j][2 * hf], v[j][2 * hf + 1]);
        }
        __syncthreads();
        {
            // dS <- exp(G_L) dS + Qg^T dO + (-W)^T dVnew
            const float *egl = reinterpret_cast<const float *>(sm + st * S::STAGE + S::PART);
            const float e0 = egl[key_of(0)], e1 = egl[key_of(1)];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[j][0] *= e0;
                acc[j][1] *= e0;
                acc[j][2] *= e1;
                acc[j][3] *= e1;
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int tr = 16 * ks + (lane & 7) + ((lane >> 4) & 1) * 8, kc = 16 * ms + ((lane >> 3) & 1) * 8;
                const int br = 16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8;
                uint32_t a[4], b[4], c2[4];
                ldsm_x4_t(blk + ITEM_QG + sw_off128(tr, kc), a[0], a[1], a[2], a[3]);
                ldsm_x4_t(doh + 2 * (br * kBcPad + 32 * nh + (lane >> 4) * 8), b[0], b[1], b[2], b[3]);
                ldsm_x4_t(doh + 2 * (br * kBcPad + 32 * nh + 16 + (lane >> 4) * 8), c2[0], c2[1], c2[2], c2[3]);
                mma_f16(acc[0], a, b[0], b[1]);
                mma_f16(acc[1], a, b[2], b[3]);
                mma_f16(acc[2], a, c2[0], c2[1]);
                mma_f16(acc[3], a, c2[2], c2[3]);
                ldsm_x4_t(blk + ITEM_WN + sw_off128(tr, kc), a[0], a[1], a[2], a[3]);
                ldsm_x4_t(dvh + 2 * (br * kBcPad + 32 * nh + (lane >> 4) * 8), b[0], b[1], b[2], b[3]);
                ldsm_x4_t(dvh + 2 * (br * kBcPad + 32 * nh + 16 + (lane >> 4) * 8), c2[0], c2[1], c2[2], c2[3]);
                mma_f16(acc[0], a, b[0], b[1]);
                mma_f16(acc[1], a, b[2], b[3]);
                mma_f16(acc[2], a, c2[0], c2[1]);
                mma_f16(acc[3], a, c2[2], c2[3]);
            }
        }
        __syncthreads();  // every read of dS's fp16 copy, dO, dVnew and the stage is done
        store_dsh();
        put_dout(next_dout);
        // (the next iteration's barrier orders these writes before their reads)
    }
    if (!ok) {
        if (tid == 0) {
            atomicOr(p.err, ERR_TMA_WAIT);
            // copies may still be in flight: wait for them (bounded) before leaving
            for (int st = 0; st < 2; ++st)
                for (int w = waited[st]; w < issued[st]; ++w)
                    if (!mbar_wait(sb + S::BAR + 8 * st, w & 1)) break;
        }
        __syncthreads();
        return;
    }
    if (p.dh0) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
                *reinterpret_cast<float2 *>(p.dh0 + unit_off + key_of(hf) * DV + vc0 + col_of(j, 0)) =
                    make_float2(acc[j][2 * hf], acc[j][2 * hf + 1]);
    }
}

// ---------------------------------------------------------------------------------------------------------
// Chunk gradients: one CTA of 512 threads (16 warps) per (chunk, value head); fp32 values, TF32 MMAs (fp32
// accumulate).  The MMA phases (the value-column passes and the pairwise terms) give each warp a row block and a
// quarter of the columns; the phases written for 8 warps (gates, P/Aqk, the solve, dL) run on threads 0-255 while
// the rest wait at the next barrier.  One CTA per SM: 16 warps hide more of the MMA chains' latency than 8.
constexpr int kBwThreads = 512, kBwCols = 16;  // value columns per pass over the state
constexpr int kRow = 132;                      // padded row stride (floats) of the [64][128] operand tiles
constexpr int kRowC = 68;                      // padded row stride of the [64][64] tiles
// element (r, c) of a [64][16] fp32 value-column tile: rows of 16 floats, the two 8-column halves swapped in
// rows with bit 1 set.  Scalar reads of 4 rows x 8 columns and 8-byte accesses of 4 rows x 4 column pairs
// (a half warp) then fall into 32 distinct banks.
__device__ __forceinline__ int vsw(int r, int c) { return r * kBwCols + (c ^ (((r >> 1) & 1) << 3)); }
// column of element (r, c) in a [rows][16] bf16 pass buffer (S, dS', dO): the two 16-byte halves of a row swapped
// in rows with bit 2 set, so that 4-byte reads of one column pair from 8 consecutive rows hit 8 distinct bank quads
__device__ __forceinline__ int bsw(int r, int c) { return c ^ (((r >> 2) & 1) << 3); }
struct BwSmem {
    static constexpr int KA = 0;                          // kn_id exp(G_id - m_Id)
    static constexpr int QA = KA + CH * kRow * 4;         // qn_id exp(G_id - m_Id)
    static constexpr int KB = QA + CH * kRow * 4;         // kn_id exp(m_Id - G_id)
    static constexpr int GG = KB + CH * kRow * 4;         // G [64][128]
    static constexpr int PP = GG + CH * DK * 4;           // P, later M = diag(beta) dL
    static constexpr int AQ = PP + CH * kRowC * 4;        // Aqk, later N = dAqk
    static constexpr int TT = AQ + CH * kRowC * 4;        // T
    static constexpr int BETA = TT + CH * kRowC * 4;      // [64]
    static constexpr int DENQ = BETA + 256, DENK = DENQ + 256;  // [64] norms of the q, k rows
    static constexpr int EM = DENK + 256;                 // [4][128] exp(m_I)
    static constexpr int EGLM = EM + 2048;                // [4][128] exp(G_L - m_I)
    static constexpr int CF = EGLM + 2048;                // [6][128] exp(m_I - m_J), J < I
    static constexpr int EGL = CF + 3072;                 // [128] exp(G_L)
    static constexpr int DGL = EGL + 512;                 // [128] gradient at G_L
    static constexpr int DBETA = DGL + 512;               // [64]
    static constexpr int WK = DBETA + 256;                // work region
    // V pass buffers (inside WK); S, dS' and dO columns are double-buffered (cp.async, one pass ahead)
    static constexpr int SV = WK;                         // bf16 [2][128][16]  S[:, cols]
    static constexpr int DSV = SV + 2 * DK * kBwCols * 2; // bf16 [2][128][16]  dS'[:, cols]
    static constexpr int DOB = DSV + 2 * DK * kBwCols * 2;  // bf16 [2][64][16] dO
    static constexpr int DD = DOB + 2 * CH * kBwCols * 2; // [64][16] (vsw) D = v - Kb S
    static constexpr int VN = DD + CH * kBwCols * 4;      // [64][16] Vnew
    static constexpr int DVN = VN + CH * kBwCols * 4;     // [64][16] dVnew
    static constexpr int DV = DVN + CH * kBwCols * 4;     // [64][16] dv
    static constexpr int WK_END = DV + CH * kBwCols * 4;
    // phase-3 use of WK: the solve's products, 3 x [16][16] then [32][33]
    // phase-6 use of WK: dA, then Y = T^T dA diag(beta)
    static constexpr int DA = WK;                         // [64][kRowC]
    static constexpr int TOTAL = (WK_END > DA + CH * kRowC * 4 ? WK_END : DA + CH * kRowC * 4);
};
static_assert(BwSmem::TOTAL <= 232448, "shared memory");

__device__ __forceinline__ int cf_index(int I, int J) { return I * (I - 1) / 2 + J; }

__global__ void __launch_bounds__(kBwThreads, 1) kda_bwd_chunk_kernel(const BwdParams p)
{
    using S = BwSmem;
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = blockIdx.x / p.HV, h = blockIdx.x % p.HV, hq = h / (p.HV / p.H);
    if (p.cu && chunk >= p.chunk_off[p.N]) return;  // the grid covers the bound on packed chunks
    int n, c_in_seq, nvalid;
    int64_t row0;
    bwd_locate(p, chunk, n, row0, c_in_seq, nvalid);
    (void)n;
    (void)c_in_seq;
    const float s = 0.08838834764831845f;  // K^-0.5

    float(*KA)[kRow] = reinterpret_cast<float(*)[kRow]>(sm + S::KA);
    float(*QA)[kRow] = reinterpret_cast<float(*)[kRow]>(sm + S::QA);
    float(*KB)[kRow] = reinterpret_cast<float(*)[kRow]>(sm + S::KB);
    float(*G)[DK] = reinterpret_cast<float(*)[DK]>(sm + S::GG);
    float(*PP)[kRowC] = reinterpret_cast<float(*)[kRowC]>(sm + S::PP);
    float(*AQ)[kRowC] = reinterpret_cast<float(*)[kRowC]>(sm + S::AQ);
    float(*TT)[kRowC] = reinterpret_cast<float(*)[kRowC]>(sm + S::TT);
    float *beta = reinterpret_cast<float *>(sm + S::BETA);
    float *denq = reinterpret_cast<float *>(sm + S::DENQ), *denk = reinterpret_cast<float *>(sm + S::DENK);
    float(*EM)[DK] = reinterpret_cast<float(*)[DK]>(sm + S::EM);
    float(*EGLM)[DK] = reinterpret_cast<float(*)[DK]>(sm + S::EGLM);
    float(*CF)[DK] = reinterpret_cast<float(*)[DK]>(sm + S::CF);
    float *egl = reinterpret_cast<float *>(sm + S::EGL), *dgl = reinterpret_cast<float *>(sm + S::DGL);
    float *dbeta = reinterpret_cast<float *>(sm + S::DBETA);
    const int64_t item = static_cast<int64_t>(chunk) * p.HV + h;

    // ---- 1. gates: G = cumulative g, block references, beta ----
    // this warp's eight q and k rows, requested first so that their latency overlaps the gate work
    uint2 rqv[CH / 16], rkv[CH / 16];
#pragma unroll
    for (int m = 0; m < CH / 16; ++m) {
        const int r = warp + 16 * m;
        rqv[m] = rkv[m] = make_uint2(0u, 0u);
        if (r < nvalid) {
            rqv[m] = *reinterpret_cast<const uint2 *>(p.q + ((row0 + r) * p.H + hq) * DK + 4 * lane);
            rkv[m] = *reinterpret_cast<const uint2 *>(p.k + ((row0 + r) * p.H + hq) * DK + 4 * lane);
        }
    }
    {
        const int i = tid >> 3, c0 = 16 * (tid & 7);
        const float *gr = p.g + ((row0 + i) * p.HV + h) * DK + c0;
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < nvalid) x = *reinterpret_cast<const float4 *>(gr + e);
            *reinterpret_cast<float4 *>(&G[i][c0 + e]) = x;
        }
        if (tid < CH) beta[tid] = tid < nvalid ? p.beta[(row0 + tid) * p.HV + h] : 0.f;
        if (tid < DK) dgl[tid] = 0.f;
        if (tid < CH) dbeta[tid] = 0.f;
    }
    __syncthreads();
    if (tid < DK) {
        float acc = 0.f;
        for (int i = 0; i < CH; ++i) {
            acc = __fadd_rn(acc, G[i][tid]);
            G[i][tid] = acc;
        }
        const float gl = acc;
        egl[tid] = bwd_exp(gl);
#pragma unroll
        for (int I = 0; I < 4; ++I) {
            const float m = G[16 * I + 7][tid];
            EM[I][tid] = bwd_exp(m);
            EGLM[I][tid] = bwd_exp(__fsub_rn(gl, m));
        }
#pragma unroll
        for (int I = 1; I < 4; ++I)
#pragma unroll
            for (int J = 0; J < I; ++J)
                CF[cf_index(I, J)][tid] = bwd_exp(__fsub_rn(G[16 * I + 7][tid], G[16 * J + 7][tid]));
    }
    __syncthreads();
    // ---- normalised q/k rows and the gate-scaled operands ----
#pragma unroll
    for (int m = 0; m < CH / 16; ++m) {
        const int r = warp + 16 * m;
        const uint2 rq = rqv[m], rk = rkv[m];
        // the forward's row denominators, kept to rebuild qn/kn bit for bit at the end
        const float dq = l2norm_den128_warp(rq), dk = l2norm_den128_warp(rk);
        const uint2 nq = l2norm_apply128(rq, dq), nk = l2norm_apply128(rk, dk);
        if (lane == 0) {
            denq[r] = dq;
            denk[r] = dk;
        }
        const float qv[4] = {bf16lo(nq.x), bf16hi(nq.x), bf16lo(nq.y), bf16hi(nq.y)};
        const float kv[4] = {bf16lo(nk.x), bf16hi(nk.x), bf16lo(nk.y), bf16hi(nk.y)};
        const int I = r >> 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d = 4 * lane + e;
            const float x = __fsub_rn(G[r][d], G[16 * I + 7][d]);
            const float a = bwd_exp(x), b = bwd_exp(-x);
            KA[r][d] = __fmul_rn(kv[e], a);
            QA[r][d] = __fmul_rn(qv[e], a);
            KB[r][d] = __fmul_rn(kv[e], b);
        }
    }
    __syncthreads();

    // ---- 2. P (j < i) and Aqk (j <= i); thread: rows 4rg..4rg+3 (block I), columns cg + 16 jb (threads 0-255:
    //         with more threads each would reread the same q/k rows for fewer column blocks, and the phase is
    //         bound by those shared-memory reads) ----
    if (tid < 256) {
        const int rg = tid >> 4, cg = tid & 15, I = rg >> 2;
        float pa[4][4] = {}, aa[4][4] = {};
        for (int d = 0; d < DK; d += 4) {
            float4 ka[4], qa[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                ka[ii] = *reinterpret_cast<const float4 *>(&KA[4 * rg + ii][d]);
                qa[ii] = *reinterpret_cast<const float4 *>(&QA[4 * rg + ii][d]);
            }
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {
                if (jb > I) break;
                float4 kb = *reinterpret_cast<const float4 *>(&KB[cg + 16 * jb][d]);
                if (jb < I) {
                    const float4 cf = *reinterpret_cast<const float4 *>(&CF[cf_index(I, jb)][d]);
                    kb = make_float4(__fmul_rn(kb.x, cf.x), __fmul_rn(kb.y, cf.y), __fmul_rn(kb.z, cf.z),
                                     __fmul_rn(kb.w, cf.w));
                }
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    float x = pa[ii][jb], y = aa[ii][jb];
                    x = __fmaf_rn(ka[ii].x, kb.x, x);
                    x = __fmaf_rn(ka[ii].y, kb.y, x);
                    x = __fmaf_rn(ka[ii].z, kb.z, x);
                    x = __fmaf_rn(ka[ii].w, kb.w, x);
                    y = __fmaf_rn(qa[ii].x, kb.x, y);
                    y = __fmaf_rn(qa[ii].y, kb.y, y);
                    y = __fmaf_rn(qa[ii].z, kb.z, y);
                    y = __fmaf_rn(qa[ii].w, kb.w, y);
                    pa[ii][jb] = x;
                    aa[ii][jb] = y;
                }
            }
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {
                const int i = 4 * rg + ii, j = cg + 16 * jb;
                PP[i][j] = j < i ? pa[ii][jb] : 0.f;
                AQ[i][j] = j <= i ? __fmul_rn(s, aa[ii][jb]) : 0.f;
                TT[i][j] = i == j ? 1.f : 0.f;
            }
    }
    __syncthreads();

    // ---- 3. T = (I + L)^-1, L = diag(beta) P, in three steps:
    //         the four 16 x 16 diagonal blocks by right-looking substitution in registers (thread = block I,
    //         column c, rows r4 + 4q; row m reaches the column's lanes by shuffle), then the blocks next to the
    //         diagonal T_{I,I-1} = -T_II L_{I,I-1} T_{I-1,I-1}, then the lower-left 32 x 32 block as
    //         -T_B (L_C T_A) with T_A, T_B the two 32 x 32 diagonal blocks ----
    if (tid < 256) {
        const int I = tid >> 6, c = (tid >> 2) & 15, r4 = tid & 3;
        float x[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) x[q] = (4 * q + r4 == c) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < 15; ++m) {
            const float xm = __shfl_sync(0xffffffffu, x[m >> 2], (lane & ~3) | (m & 3));
#pragma unroll
            for (int q = m >> 2; q < 4; ++q) {
                const int j = 4 * q + r4;
                if (j > m) x[q] = __fmaf_rn(-__fmul_rn(beta[16 * I + j], PP[16 * I + j][16 * I + m]), xm, x[q]);
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) TT[16 * I + 4 * q + r4][16 * I + c] = x[q];
    }
    __syncthreads();
    {
        // (the blocks above the diagonal of T are zero, so every sum below runs over a fixed range)
        float(*X)[16][16] = reinterpret_cast<float(*)[16][16]>(sm + S::WK);  // L_{I,I-1} T_{I-1,I-1}, I = 1..3
        if (tid < 256) {
            const int i = (tid >> 4) & 15, j = tid & 15;  // this thread: element (i, j) of each of the three blocks
            float acc[3] = {};
#pragma unroll
            for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int b = 0; b < 3; ++b)
                    acc[b] = __fmaf_rn(PP[16 * (b + 1) + i][16 * b + k], TT[16 * b + k][16 * b + j], acc[b]);
#pragma unroll
            for (int b = 0; b < 3; ++b) X[b][i][j] = __fmul_rn(beta[16 * (b + 1) + i], acc[b]);
        }
        __syncthreads();
        if (tid < 256) {
            const int i = (tid >> 4) & 15, j = tid & 15;
            float acc[3] = {};
#pragma unroll
            for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int b = 0; b < 3; ++b) acc[b] = __fmaf_rn(TT[16 * (b + 1) + i][16 * (b + 1) + k], X[b][k][j], acc[b]);
#pragma unroll
            for (int b = 0; b < 3; ++b) TT[16 * (b + 1) + i][16 * b + j] = -acc[b];
        }
        __syncthreads();
        float(*Y)[33] = reinterpret_cast<float(*)[33]>(sm + S::WK + 3 * 256 * 4);  // L_C T_A, [32][33]
        {
            const int j = tid & 31, i0 = tid >> 5;  // this thread: rows i0 + 16 it, column j
            float acc[2] = {};
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float tk = TT[k][j];
#pragma unroll
                for (int it = 0; it < 2; ++it) acc[it] = __fmaf_rn(PP[32 + i0 + 16 * it][k], tk, acc[it]);
            }
#pragma unroll
            for (int it = 0; it < 2; ++it) Y[i0 + 16 * it][j] = __fmul_rn(beta[32 + i0 + 16 * it], acc[it]);
        }
        __syncthreads();
        {
            const int j = tid & 31, i0 = tid >> 5;
            float acc[2] = {};
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float yk = Y[k][j];
#pragma unroll
                for (int it = 0; it < 2; ++it) acc[it] = __fmaf_rn(TT[32 + i0 + 16 * it][32 + k], yk, acc[it]);
            }
#pragma unroll
            for (int it = 0; it < 2; ++it) TT[32 + i0 + 16 * it][j] = -acc[it];
        }
        __syncthreads();
    }

    // ---- 4-5. passes over 16 value columns at a time, on TF32 tensor-core MMAs (m16n8k8, fp32 accumulate) ----
    // S, dS' (bf16 [128][16]) and dO (bf16 [64][16]) of the current pass, the next pass's in the other buffer
    auto SVb = [&](int b) { return reinterpret_cast<__nv_bfloat16(*)[kBwCols]>(sm + S::SV + b * DK * kBwCols * 2); };
    auto DSVb = [&](int b) { return reinterpret_cast<__nv_bfloat16(*)[kBwCols]>(sm + S::DSV + b * DK * kBwCols * 2); };
    auto DOBb = [&](int b) { return reinterpret_cast<__nv_bfloat16(*)[kBwCols]>(sm + S::DOB + b * CH * kBwCols * 2); };
    float *DDv = reinterpret_cast<float *>(sm + S::DD);
    float *VN = reinterpret_cast<float *>(sm + S::VN);
    float *DVN = reinterpret_cast<float *>(sm + S::DVN);
    float *DVv = reinterpret_cast<float *>(sm + S::DV);
    const __nv_bfloat16 *Sg = p.states + item * DK * DV;
    const __nv_bfloat16 *dSg = p.dstates + item * DK * DV;
    const int cg = tid & 15;  // column of the 64 x 64 steps of phase 6 (with the row group and half below)
    // MMA fragment ownership (g = lane / 4, t4 = lane % 4): warp (mt, nh), nh = 0..3, holds rows 16 mt + g and + 8,
    // and key columns 32 nh + 8 j + 2 t4 (+1), j = 0..3 (dQg, dKb, dKg), or token columns 16 nh + 8 j + 2 t4 (+1),
    // j = 0..1 (dAqk, dA).  In steps (a)-(d) of a pass, warp (mt, role, ntw) = (warp % 4, warp / 4 % 2, warp / 8)
    // computes rows 16 mt of the ntw-th 8-column tile of D and Vnew (role 0) or dVnew and dv (role 1).
    const int g = lane >> 2, t4 = lane & 3, mt = warp & 3, nh = warp >> 2;
    const int role = (warp >> 2) & 1, ntw = warp >> 3;
    const int r0 = 16 * mt + g, r1 = r0 + 8;
    // bf16 values are exact in TF32 (8 of its 10 mantissa bits): the widened bits are the operand as they are
    auto bf = [](__nv_bfloat16 x) { return static_cast<uint32_t>(__bfloat16_as_ushort(x)) << 16; };
    float aQ[4][4] = {}, aB[4][4] = {}, aG[4][4] = {}, aAq[2][4] = {}, aA[2][4] = {};
    // pass vb's columns into buffer b: S, dS' and dO rows are 32 bytes (two 16-byte copies each)
    auto fetch = [&](int vb, int b) {
        const int row = tid >> 1, half = 8 * (tid & 1);
        if (tid < 256) {
            cp_async16(smem_u32(&SVb(b)[row][bsw(row, half)]), Sg + row * DV + vb + half);
            cp_async16(smem_u32(&DSVb(b)[row][bsw(row, half)]), dSg + row * DV + vb + half);
        }
        if (row < nvalid && tid < 2 * CH)
            cp_async16(smem_u32(&DOBb(b)[row][bsw(row, half)]), p.dout + ((row0 + row) * p.HV + h) * DV + vb + half);
        cp_async_commit();
    };
    if (tid < CH && tid >= nvalid) {  // rows past the end stay zero in both buffers
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            *reinterpret_cast<uint4 *>(&DOBb(b)[tid][0]) = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(&DOBb(b)[tid][8]) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    fetch(0, 0);
    float gl_acc = 0.f;  // thread d < 128: sum over all columns of S[d][.] dS'[d][.]
    for (int vb = 0; vb < DV; vb += kBwCols) {
        const int buf = (vb / kBwCols) & 1;
        if (vb + kBwCols < DV) {
            fetch(vb + kBwCols, buf ^ 1);  // that buffer was released by the previous pass's last barrier
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const __nv_bfloat16(*SVT)[kBwCols] = SVb(buf);
        const __nv_bfloat16(*DST)[kBwCols] = DSVb(buf);
        const __nv_bfloat16(*DOV)[kBwCols] = DOBb(buf);
        if (tid < DK) {  // S and dS' rows share one column order, so physical positions pair up
#pragma unroll
            for (int c = 0; c < kBwCols; c += 2) {
                const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&SVT[tid][c]));
                const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&DST[tid][c]));
                gl_acc = __fmaf_rn(x.y, y.y, __fmaf_rn(x.x, y.x, gl_acc));
            }
        }
        const int cn = 8 * ntw + g;  // this warp's tile: B-fragment column of steps (a)-(d)
        if (role == 0) {
            // (a) D = v - Kb S for rows 16 mt .. (Kb = KA exp(m_I), block I = mt), columns 8 ntw ..
            float c[4] = {};
            for (int ks = 0; ks < DK; ks += 8) {
                const float e0 = EM[mt][ks + t4], e1 = EM[mt][ks + t4 + 4];
                const uint32_t a[4] = {to_tf32(__fmul_rn(KA[r0][ks + t4], e0)), to_tf32(__fmul_rn(KA[r1][ks + t4], e0)),
                                       to_tf32(__fmul_rn(KA[r0][ks + t4 + 4], e1)),
                                       to_tf32(__fmul_rn(KA[r1][ks + t4 + 4], e1))};
                const int k0 = ks + t4, k1 = ks + t4 + 4;
                mma_tf32(c, a, bf(SVT[k0][bsw(k0, cn)]), bf(SVT[k1][bsw(k1, cn)]));
            }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int i = hf ? r1 : r0, cc = 8 * ntw + 2 * t4;
                float2 vv = make_float2(0.f, 0.f);
                if (i < nvalid)
                    vv = __bfloat1622float2(
                        *reinterpret_cast<const __nv_bfloat162 *>(p.v + ((row0 + i) * p.HV + h) * DV + vb + cc));
                *reinterpret_cast<float2 *>(&DDv[vsw(i, cc)]) =
                    make_float2(__fsub_rn(vv.x, c[2 * hf]), __fsub_rn(vv.y, c[2 * hf + 1]));
            }
        } else {
            // (c) dVnew = Kg dS' + Aqk^T dO for rows 16 mt .. (Kg = KB exp(G_L - m_I)), columns 8 ntw ..
            float c[4] = {};
            for (int ks = 0; ks < DK; ks += 8) {
                const float e0 = EGLM[mt][ks + t4], e1 = EGLM[mt][ks + t4 + 4];
                const uint32_t a[4] = {to_tf32(__fmul_rn(KB[r0][ks + t4], e0)), to_tf32(__fmul_rn(KB[r1][ks + t4], e0)),
                                       to_tf32(__fmul_rn(KB[r0][ks + t4 + 4], e1)),
                                       to_tf32(__fmul_rn(KB[r1][ks + t4 + 4], e1))};
                const int k0 = ks + t4, k1 = ks + t4 + 4;
                mma_tf32(c, a, bf(DST[k0][bsw(k0, cn)]), bf(DST[k1][bsw(k1, cn)]));
            }
            for (int js = 16 * mt; js < CH; js += 8) {  // Aqk^T[i][j] = Aqk[j][i], nonzero for j >= i
                const uint32_t a[4] = {to_tf32(AQ[js + t4][r0]), to_tf32(AQ[js + t4][r1]), to_tf32(AQ[js + t4 + 4][r0]),
                                       to_tf32(AQ[js + t4 + 4][r1])};
                const int k0 = js + t4, k1 = js + t4 + 4;
                mma_tf32(c, a, bf(DOV[k0][bsw(k0, cn)]), bf(DOV[k1][bsw(k1, cn)]));
            }
            *reinterpret_cast<float2 *>(&DVN[vsw(r0, 8 * ntw + 2 * t4)]) = make_float2(c[0], c[1]);
            *reinterpret_cast<float2 *>(&DVN[vsw(r1, 8 * ntw + 2 * t4)]) = make_float2(c[2], c[3]);
        }
        __syncthreads();
        if (role == 0) {
            // (b) Vnew = T diag(beta) D (T lower triangular: j < 16 (mt + 1))
            float c[4] = {};
            for (int js = 0; js < 16 * (mt + 1); js += 8) {
                const float b0 = beta[js + t4], b1 = beta[js + t4 + 4];
                const uint32_t a[4] = {to_tf32(__fmul_rn(TT[r0][js + t4], b0)), to_tf32(__fmul_rn(TT[r1][js + t4], b0)),
                                       to_tf32(__fmul_rn(TT[r0][js + t4 + 4], b1)),
                                       to_tf32(__fmul_rn(TT[r1][js + t4 + 4], b1))};
                mma_tf32(c, a, to_tf32(DDv[vsw(js + t4, cn)]), to_tf32(DDv[vsw(js + t4 + 4, cn)]));
            }
            *reinterpret_cast<float2 *>(&VN[vsw(r0, 8 * ntw + 2 * t4)]) = make_float2(c[0], c[1]);
            *reinterpret_cast<float2 *>(&VN[vsw(r1, 8 * ntw + 2 * t4)]) = make_float2(c[2], c[3]);
        } else {
            // (d) dv = diag(beta) T^T dVnew (j >= i)
            float c[4] = {};
            for (int js = 16 * mt; js < CH; js += 8) {
                const uint32_t a[4] = {to_tf32(TT[js + t4][r0]), to_tf32(TT[js + t4][r1]), to_tf32(TT[js + t4 + 4][r0]),
                                       to_tf32(TT[js + t4 + 4][r1])};
                mma_tf32(c, a, to_tf32(DVN[vsw(js + t4, cn)]), to_tf32(DVN[vsw(js + t4 + 4, cn)]));
            }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int i = hf ? r1 : r0, cc = 8 * ntw + 2 * t4;
                const float x0 = __fmul_rn(beta[i], c[2 * hf]), x1 = __fmul_rn(beta[i], c[2 * hf + 1]);
                *reinterpret_cast<float2 *>(&DVv[vsw(i, cc)]) = make_float2(x0, x1);
                if (i < nvalid)
                    *reinterpret_cast<__nv_bfloat162 *>(p.dv + ((row0 + i) * p.HV + h) * DV + vb + cc) =
                        __floats2bfloat162_rn(x0, x1);
            }
        }
        __syncthreads();
        // (e) dQg += dO S^T, dKb -= dv S^T, dKg += Vnew dS'^T (K = these 16 columns, two k8 steps);
        //     dAqk += dO Vnew^T, dA += dVnew D^T.  A k8 step's slots t4 and t4 + 4 carry this thread's column pair
        //     cp, cp + 1 (any order of K is a valid order as long as A and B share it), so every operand pair
        //     comes from one 4- or 8-byte shared-memory read.
        auto pair = [](const __nv_bfloat16(*B)[kBwCols], int r, int c) {
            return *reinterpret_cast<const uint32_t *>(&B[r][bsw(r, c)]);
        };
        constexpr uint32_t kHi = 0xffff0000u;
#pragma unroll
        for (int kc = 0; kc < kBwCols; kc += 8) {
            const int cp = kc + 2 * t4;
            const uint32_t o0 = pair(DOV, r0, cp), o1 = pair(DOV, r1, cp);
            const uint32_t aO[4] = {o0 << 16, o1 << 16, o0 & kHi, o1 & kHi};
            const float2 v0 = *reinterpret_cast<const float2 *>(&DVv[vsw(r0, cp)]);
            const float2 v1 = *reinterpret_cast<const float2 *>(&DVv[vsw(r1, cp)]);
            const float2 n0 = *reinterpret_cast<const float2 *>(&VN[vsw(r0, cp)]);
            const float2 n1 = *reinterpret_cast<const float2 *>(&VN[vsw(r1, cp)]);
            const float2 e0 = *reinterpret_cast<const float2 *>(&DVN[vsw(r0, cp)]);
            const float2 e1 = *reinterpret_cast<const float2 *>(&DVN[vsw(r1, cp)]);
            const uint32_t aV[4] = {to_tf32(-v0.x), to_tf32(-v1.x), to_tf32(-v0.y), to_tf32(-v1.y)};
            const uint32_t aN[4] = {to_tf32(n0.x), to_tf32(n1.x), to_tf32(n0.y), to_tf32(n1.y)};
            const uint32_t aD[4] = {to_tf32(e0.x), to_tf32(e1.x), to_tf32(e0.y), to_tf32(e1.y)};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int d = 32 * nh + 8 * j + g;
                const uint32_t sp = pair(SVT, d, cp), qp = pair(DST, d, cp);
                mma_tf32(aQ[j], aO, sp << 16, sp & kHi);
                mma_tf32(aB[j], aV, sp << 16, sp & kHi);
                mma_tf32(aG[j], aN, qp << 16, qp & kHi);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int tk = 16 * nh + 8 * j + g;
                const float2 vn = *reinterpret_cast<const float2 *>(&VN[vsw(tk, cp)]);
                const float2 dd = *reinterpret_cast<const float2 *>(&DDv[vsw(tk, cp)]);
                mma_tf32(aAq[j], aO, to_tf32(vn.x), to_tf32(vn.y));
                mma_tf32(aA[j], aD, to_tf32(dd.x), to_tf32(dd.y));
            }
        }
        __syncthreads();
    }

    if (tid < DK) dgl[tid] = __fmaf_rn(egl[tid], gl_acc, dgl[tid]);  // the exp(G_L) S dS' term of dG_L

    // ---- 6. dbeta, dL, M = diag(beta) dL, N = dAqk ----
    float(*DA)[kRowC] = reinterpret_cast<float(*)[kRowC]>(sm + S::DA);
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = (q >> 1) ? r1 : r0, tk = 16 * nh + 8 * j + 2 * t4 + (q & 1);
            DA[i][tk] = aA[j][q];
            AQ[i][tk] = tk <= i ? aAq[j][q] : 0.f;  // Aqk is no longer needed: N takes its place
        }
    __syncthreads();
    if (tid < CH) {  // dbeta_j += sum_{i >= j} dA_ij T_ij
        float acc = 0.f;
        for (int i = tid; i < CH; ++i) acc = __fmaf_rn(DA[i][tid], TT[i][tid], acc);
        dbeta[tid] = acc;
    }
    // Y = T^T (dA diag(beta)): Y[a][e] = beta_e sum_{c >= a} T[c][a] dA[c][e].  Thread: rows 4 rg6 .. 4 rg6 + 3
    // and columns cg + 16 jb for the two column blocks jb = 2 jh, 2 jh + 1 of its half of the CTA.
    const int rg6 = (tid >> 4) & 15, jh = tid >> 8;
    float y[4][2] = {};
    for (int c = 4 * rg6; c < CH; ++c) {
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const float t = TT[c][4 * rg6 + ii];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) y[ii][jj] = __fmaf_rn(t, DA[c][cg + 16 * (2 * jh + jj)], y[ii][jj]);
        }
    }
    __syncthreads();  // every read of dA is done
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int col = cg + 16 * (2 * jh + jj);
            DA[4 * rg6 + ii][col] = __fmul_rn(beta[col], y[ii][jj]);
        }
    __syncthreads();
    // dL[a][b] = -sum_{e <= b} Y[a][e] T[b][e] (a > b); dbeta_a += sum_b dL_ab P_ab; M = diag(beta) dL
    {
        float *rowp2 = reinterpret_cast<float *>(sm + S::DA + CH * kRowC * 4);  // [2 halves][64 rows]
        float dl[4][2] = {}, rowp[4] = {};
        for (int e = 0; e < CH; ++e) {
            float ye[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) ye[ii] = DA[4 * rg6 + ii][e];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const float t = TT[cg + 16 * (2 * jh + jj)][e];  // zero for e > b
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) dl[ii][jj] = __fmaf_rn(-ye[ii], t, dl[ii][jj]);
            }
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int a = 4 * rg6 + ii, b = cg + 16 * (2 * jh + jj);
                if (b < a) rowp[ii] = __fmaf_rn(dl[ii][jj], PP[a][b], rowp[ii]);
                else dl[ii][jj] = 0.f;
            }
        // the 16 threads of a row group are 16 consecutive lanes
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
#pragma unroll
            for (int off = 8; off > 0; off >>= 1)
                rowp[ii] = __fadd_rn(rowp[ii], __shfl_xor_sync(0xffffffffu, rowp[ii], off));
        }
        if (cg == 0) {
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) rowp2[jh * CH + 4 * rg6 + ii] = rowp[ii];
        }
        __syncthreads();  // every read of P and T is done (dbeta's column sums above included); halves stored
        if (tid < CH) dbeta[tid] = __fadd_rn(dbeta[tid], __fadd_rn(rowp2[tid], rowp2[CH + tid]));
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int jj = 0; jj < 2; ++jj)
                PP[4 * rg6 + ii][cg + 16 * (2 * jh + jj)] = __fmul_rn(beta[4 * rg6 + ii], dl[ii][jj]);
    }
    __syncthreads();
    float(*MM)[kRowC] = PP;
    float(*NN)[kRowC] = AQ;

    // ---- 7. element terms and pairwise terms, in the fragment ownership of phase 5 ----
    float rq[4][4], rk[4][4], rG[4][4];
    {
        // qn/kn of the owned elements, rebuilt from the raw rows (the same normalisation, bit for bit)
        float glp[4][2] = {};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int i = hf ? r1 : r0;
            const float dq = denq[i], dk = denk[i], rqi = __frcp_rn(dq), rki = __frcp_rn(dk);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int d = 32 * nh + 8 * j + 2 * t4;
                uint32_t wq = 0u, wk = 0u;
                if (i < nvalid) {
                    wq = *reinterpret_cast<const uint32_t *>(p.q + ((row0 + i) * p.H + hq) * DK + d);
                    wk = *reinterpret_cast<const uint32_t *>(p.k + ((row0 + i) * p.H + hq) * DK + d);
                }
                const uint32_t pq = pack_bf16(div_rn_with_rcp(bf16lo(wq), dq, rqi), div_rn_with_rcp(bf16hi(wq), dq, rqi));
                const uint32_t pk = pack_bf16(div_rn_with_rcp(bf16lo(wk), dk, rki), div_rn_with_rcp(bf16hi(wk), dk, rki));
                const float qn[2] = {bf16lo(pq), bf16hi(pq)}, kn[2] = {bf16lo(pk), bf16hi(pk)};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int q = 2 * hf + e, dd = d + e;
                    // X3 = s exp(G) dQg, X1 = exp(G) dKb, X2 = exp(G_L - G) dKg
                    const float x = __fsub_rn(G[i][dd], G[16 * mt + 7][dd]);
                    const float eg = __fmul_rn(bwd_exp(x), EM[mt][dd]), eglg = __fmul_rn(bwd_exp(-x), EGLM[mt][dd]);
                    const float x3 = __fmul_rn(__fmul_rn(s, eg), aQ[j][q]);
                    const float x1 = __fmul_rn(eg, aB[j][q]);
                    const float x2 = __fmul_rn(eglg, aG[j][q]);
                    rq[j][q] = x3;
                    rk[j][q] = __fadd_rn(x1, x2);
                    rG[j][q] = __fmaf_rn(qn[e], x3, __fmul_rn(kn[e], __fsub_rn(x1, x2)));
                    glp[j][e] = __fmaf_rn(kn[e], x2, glp[j][e]);
                }
            }
        }
        // dG_L += sum over rows of kn X2: the eight lanes g of a column, then (in a fixed order, after the next
        // barrier) the four row blocks' partial sums, kept in the work region (free since phase 6)
        float(*glpart)[DK] = reinterpret_cast<float(*)[DK]>(sm + S::WK);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float x = glp[j][e];
                x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, 4));
                x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, 8));
                x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, 16));
                if (g == 0) glpart[mt][32 * nh + 8 * j + 2 * t4 + e] = x;
            }
    }
    {
        // R1'_id = sum_{J <= I} sum_{j in J} M_ij KB_jd c_IJd and R3' the same with N (I = mt)
        float ra[4][4] = {}, rb[4][4] = {};
        for (int J = 0; J <= mt; ++J) {
            const float *cf = J < mt ? CF[cf_index(mt, J)] : nullptr;
            for (int ks = 16 * J; ks < 16 * J + 16; ks += 8) {
                const uint32_t am[4] = {to_tf32(MM[r0][ks + t4]), to_tf32(MM[r1][ks + t4]), to_tf32(MM[r0][ks + t4 + 4]),
                                        to_tf32(MM[r1][ks + t4 + 4])};
                const uint32_t an[4] = {to_tf32(NN[r0][ks + t4]), to_tf32(NN[r1][ks + t4]), to_tf32(NN[r0][ks + t4 + 4]),
                                        to_tf32(NN[r1][ks + t4 + 4])};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int d = 32 * nh + 8 * j + g;
                    float b0 = KB[ks + t4][d], b1 = KB[ks + t4 + 4][d];
                    if (cf) {
                        b0 = __fmul_rn(b0, cf[d]);
                        b1 = __fmul_rn(b1, cf[d]);
                    }
                    const uint32_t u0 = to_tf32(b0), u1 = to_tf32(b1);
                    mma_tf32(ra[j], am, u0, u1);
                    mma_tf32(rb[j], an, u0, u1);
                }
            }
        }
        // R1 = a R1', R3 = s a R3' (a = exp(G - m_I)): dkn += R1, dqn += R3, dG += kn R1 + qn R3
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = (q >> 1) ? r1 : r0, d = 32 * nh + 8 * j + 2 * t4 + (q & 1);
                const float a = bwd_exp(__fsub_rn(G[i][d], G[16 * mt + 7][d]));
                rk[j][q] = __fmaf_rn(a, ra[j][q], rk[j][q]);
                rq[j][q] = __fmaf_rn(__fmul_rn(s, a), rb[j][q], rq[j][q]);
                rG[j][q] = __fmaf_rn(KA[i][d], ra[j][q], rG[j][q]);
                rG[j][q] = __fmaf_rn(__fmul_rn(s, QA[i][d]), rb[j][q], rG[j][q]);
            }
    }
    // the raw q/k pairs of the owned elements, for the normalisation's Jacobian at the end (requested here, so
    // that their latency hides behind the MMAs below)
    uint32_t xq[2][4] = {}, xk[2][4] = {};
    if (p.fuse_norm) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int i = hf ? r1 : r0;
            if (i < nvalid) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int64_t off = ((row0 + i) * p.H + hq) * DK + 32 * nh + 8 * j + 2 * t4;
                    xq[hf][j] = *reinterpret_cast<const uint32_t *>(p.q + off);
                    xk[hf][j] = *reinterpret_cast<const uint32_t *>(p.k + off);
                }
            }
        }
    }
    {
        // R24'_jd = sum_{I' >= J} sum_{i in I'} (M_ij KA_id + s N_ij QA_id) c_I'Jd for rows j of block J = mt
        float ra[4][4] = {};
        for (int I2 = mt; I2 < 4; ++I2) {
            const float *cf = I2 > mt ? CF[cf_index(I2, mt)] : nullptr;
            for (int ks = 16 * I2; ks < 16 * I2 + 16; ks += 8) {
                const uint32_t am[4] = {to_tf32(MM[ks + t4][r0]), to_tf32(MM[ks + t4][r1]), to_tf32(MM[ks + t4 + 4][r0]),
                                        to_tf32(MM[ks + t4 + 4][r1])};
                const uint32_t an[4] = {to_tf32(NN[ks + t4][r0]), to_tf32(NN[ks + t4][r1]), to_tf32(NN[ks + t4 + 4][r0]),
                                        to_tf32(NN[ks + t4 + 4][r1])};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int d = 32 * nh + 8 * j + g;
                    float k0 = KA[ks + t4][d], k1 = KA[ks + t4 + 4][d];
                    float q0 = __fmul_rn(s, QA[ks + t4][d]), q1 = __fmul_rn(s, QA[ks + t4 + 4][d]);
                    if (cf) {
                        const float c = cf[d];
                        k0 = __fmul_rn(k0, c);
                        k1 = __fmul_rn(k1, c);
                        q0 = __fmul_rn(q0, c);
                        q1 = __fmul_rn(q1, c);
                    }
                    mma_tf32(ra[j], am, to_tf32(k0), to_tf32(k1));
                    mma_tf32(ra[j], an, to_tf32(q0), to_tf32(q1));
                }
            }
        }
        // R24 = b R24' (b = exp(m_J - G)): dkn += R24, dG -= kn R24 = KB R24'
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = (q >> 1) ? r1 : r0, d = 32 * nh + 8 * j + 2 * t4 + (q & 1);
                const float b = bwd_exp(__fsub_rn(G[16 * mt + 7][d], G[i][d]));
                rk[j][q] = __fmaf_rn(b, ra[j][q], rk[j][q]);
                rG[j][q] = __fmaf_rn(-KB[i][d], ra[j][q], rG[j][q]);
            }
    }
    // dqn, dkn out (valid rows), for kda_bwd_norm_kernel; or, with one value head per Q/K head, dq and dk here:
    // dx = dy / n - x (x . dy) / n^3 (n: the row's denominator of the forward's normalisation), with x . dy
    // summed by the four lanes that share a row in this warp and then across the four warps that hold its quarters.
    float xdy[2][2] = {};  // [row r0 / r1][q / k] partial x . dy of this thread's 16 columns
    if (!p.fuse_norm) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int i = hf ? r1 : r0;
            if (i < nvalid) {
                float *dq = p.dqn + ((row0 + i) * p.HV + h) * DK + 32 * nh + 2 * t4;
                float *dk = p.dkn + ((row0 + i) * p.HV + h) * DK + 32 * nh + 2 * t4;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    *reinterpret_cast<float2 *>(dq + 8 * j) = make_float2(rq[j][2 * hf], rq[j][2 * hf + 1]);
                    *reinterpret_cast<float2 *>(dk + 8 * j) = make_float2(rk[j][2 * hf], rk[j][2 * hf + 1]);
                }
            }
        }
    } else {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int i = hf ? r1 : r0;
            if (i < nvalid) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t wq = xq[hf][j], wk = xk[hf][j];
                    xdy[hf][0] = __fmaf_rn(bf16lo(wq), rq[j][2 * hf], xdy[hf][0]);
                    xdy[hf][0] = __fmaf_rn(bf16hi(wq), rq[j][2 * hf + 1], xdy[hf][0]);
                    xdy[hf][1] = __fmaf_rn(bf16lo(wk), rk[j][2 * hf], xdy[hf][1]);
                    xdy[hf][1] = __fmaf_rn(bf16hi(wk), rk[j][2 * hf + 1], xdy[hf][1]);
                }
            }
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                xdy[hf][w] = __fadd_rn(xdy[hf][w], __shfl_xor_sync(0xffffffffu, xdy[hf][w], 1));
                xdy[hf][w] = __fadd_rn(xdy[hf][w], __shfl_xor_sync(0xffffffffu, xdy[hf][w], 2));
            }
        }
    }
    __syncthreads();  // KA/QA/KB/G reads done; dgl complete
    if (p.fuse_norm) {
        float *red = reinterpret_cast<float *>(sm + S::EM);  // [q|k][row][quarter]; exp(m_I) is no longer read
        if (t4 == 0) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                for (int w = 0; w < 2; ++w) red[(w * CH + (hf ? r1 : r0)) * 4 + nh] = xdy[hf][w];
        }
        __syncthreads();
        // row i's half of dx from dy = this thread's columns of dqn (or dkn), w = 0 (q) or 1 (k)
        auto emit = [&](const float (&dy)[4][4], int hf, int w, const uint32_t (&xw)[2][4], __nv_bfloat16 *dx,
                        float den) {
            const int i = hf ? r1 : r0;
            const float *rr = red + (w * CH + i) * 4;
            const float tot = __fadd_rn(__fadd_rn(rr[0], rr[1]), __fadd_rn(rr[2], rr[3]));
            const float inv = __frcp_rn(den);
            const float c3 = __fmul_rn(tot, __fmul_rn(inv, __fmul_rn(inv, inv)));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t off = ((row0 + i) * p.H + hq) * DK + 32 * nh + 8 * j + 2 * t4;
                const uint32_t wx = xw[hf][j];
                const float o0 = __fmaf_rn(-bf16lo(wx), c3, __fmul_rn(dy[j][2 * hf], inv));
                const float o1 = __fmaf_rn(-bf16hi(wx), c3, __fmul_rn(dy[j][2 * hf + 1], inv));
                *reinterpret_cast<uint32_t *>(dx + off) = pack_bf16(o0, o1);
            }
        };
        if (r0 < nvalid) {
            emit(rq, 0, 0, xq, p.dq, denq[r0]);
            emit(rk, 0, 1, xk, p.dk, denk[r0]);
        }
        if (r1 < nvalid) {
            emit(rq, 1, 0, xq, p.dq, denq[r1]);
            emit(rk, 1, 1, xk, p.dk, denk[r1]);
        }
    }
    // dG rows into the KA region (unpadded [64][128]), then the reverse cumulative sum per key column
    float(*dG)[DK] = reinterpret_cast<float(*)[DK]>(sm + S::KA);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        *reinterpret_cast<float2 *>(&dG[r0][32 * nh + 8 * j + 2 * t4]) = make_float2(rG[j][0], rG[j][1]);
        *reinterpret_cast<float2 *>(&dG[r1][32 * nh + 8 * j + 2 * t4]) = make_float2(rG[j][2], rG[j][3]);
    }
    __syncthreads();
    if (tid < DK) {
        const float(*glpart)[DK] = reinterpret_cast<const float(*)[DK]>(sm + S::WK);
        float acc = dgl[tid];  // G_L = G of the last row
#pragma unroll
        for (int m = 0; m < 4; ++m) acc = __fadd_rn(acc, glpart[m][tid]);
        for (int i = CH - 1; i >= 0; --i) {
            acc = __fadd_rn(acc, dG[i][tid]);
            if (i < nvalid) p.dg[((row0 + i) * p.HV + h) * DK + tid] = acc;
        }
    }
    if (tid < nvalid) p.dbeta[(row0 + tid) * p.HV + h] = dbeta[tid];
}

// ---------------------------------------------------------------------------------------------------------
// dq (dk) row of Q/K head hq = J(x)^T sum over the value heads of its group of dqn (dkn), with
// J(x) the Jacobian of x / sqrt(sum x^2 + 1e-6): dx = dy / n - x (x . dy) / n^3.  A unit is one (row, head, q|k);
// a warp takes kNormUnits consecutive units and issues all their loads before any arithmetic, so that several
// rows' loads are in flight per warp (each unit alone is too little work to hide a DRAM round trip).
constexpr int kNormUnits = 4;
__global__ void __launch_bounds__(256) kda_bwd_norm_kernel(const BwdParams p, int64_t rows)
{
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kNormUnits;
    const int64_t units = rows * p.H * 2;
    if (w0 >= units) return;
    const int grp = p.HV / p.H;
    const int64_t end = p.cu ? p.cu[p.N] : rows;  // rows past it belong to no sequence
    bool live[kNormUnits];
    int64_t xoff[kNormUnits], yoff[kNormUnits];
    uint2 raw[kNormUnits];
#pragma unroll
    for (int u = 0; u < kNormUnits; ++u) {
        const int64_t w = w0 + u;
        const int which = static_cast<int>(w & 1);
        const int64_t rh = w >> 1, row = rh / p.H;
        const int hq = static_cast<int>(rh % p.H);
        live[u] = w < units && row < end;
        xoff[u] = (row * p.H + hq) * DK + 4 * lane;  // into q or k, and into dq or dk
        yoff[u] = (row * p.HV + hq * grp) * DK + 4 * lane;
        raw[u] = make_uint2(0u, 0u);
        if (live[u]) raw[u] = *reinterpret_cast<const uint2 *>((which ? p.k : p.q) + xoff[u]);
    }
    float g[kNormUnits][4] = {};
    for (int j = 0; j < grp; ++j) {
        float4 t[kNormUnits];
#pragma unroll
        for (int u = 0; u < kNormUnits; ++u) {
            t[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (live[u]) t[u] = *reinterpret_cast<const float4 *>((((w0 + u) & 1) ? p.dkn : p.dqn) + yoff[u] + j * DK);
        }
#pragma unroll
        for (int u = 0; u < kNormUnits; ++u) {
            g[u][0] = __fadd_rn(g[u][0], t[u].x);
            g[u][1] = __fadd_rn(g[u][1], t[u].y);
            g[u][2] = __fadd_rn(g[u][2], t[u].z);
            g[u][3] = __fadd_rn(g[u][3], t[u].w);
        }
    }
#pragma unroll
    for (int u = 0; u < kNormUnits; ++u) {
        const float xv[4] = {bf16lo(raw[u].x), bf16hi(raw[u].x), bf16lo(raw[u].y), bf16hi(raw[u].y)};
        float ss = 0.f, xd = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            ss = __fmaf_rn(xv[e], xv[e], ss);
            xd = __fmaf_rn(xv[e], g[u][e], xd);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
            xd = __fadd_rn(xd, __shfl_xor_sync(0xffffffffu, xd, off));
        }
        const float nrm = __fsqrt_rn(__fadd_rn(ss, 1e-6f));
        const float inv = __frcp_rn(nrm), c3 = __fmul_rn(xd, __fmul_rn(inv, __fmul_rn(inv, inv)));
        float out[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) out[e] = __fmaf_rn(-xv[e], c3, __fmul_rn(g[u][e], inv));
        if (live[u])
            *reinterpret_cast<uint2 *>((((w0 + u) & 1) ? p.dk : p.dq) + xoff[u]) =
                make_uint2(pack_bf16(out[0], out[1]), pack_bf16(out[2], out[3]));
    }
}

}  // namespace kda
