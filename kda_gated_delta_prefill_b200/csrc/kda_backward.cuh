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
//   kda_bwd_chunk_kernel  every chunk's gradients at once (fp32 CUDA cores),
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
    const float *states;                    // [chunks][HV][K][V]: state at each chunk's start
    float *dstates;                         // [chunks][HV][K][V]: gradient at each chunk's end state
    const float *dht;                       // [N][HV][K][V] or null (zero)
    float *dh0;                             // [N][HV][K][V] or null (not wanted)
    float *dqn, *dkn;                       // [rows][HV][K]: gradient at the normalised rows, per value head
    __nv_bfloat16 *dq, *dk, *dv;            // [rows][H][K], [rows][H][K], [rows][HV][V]
    float *dg, *dbeta;                      // [rows][HV][K], [rows][HV]
    const int32_t *cu, *chunk_off;          // packed sequences (cu [N+1], chunk_off [N+1]) or null
    unsigned *err;
    int T, H, HV, N, chunks_per_seq, total_chunks;
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
// Reverse carry: one CTA per (sequence, value head, half of the value columns).  dS (128 x 64 fp32) lives in
// shared memory; chunk c's block (the -W, Qg, Kg, Aqk tiles and exp(G_L)) arrives by bulk copy one chunk ahead.
// Before chunk c is folded in, dS is the gradient at chunk c's end state and is stored for the chunk kernel.
constexpr int kBcThreads = 512, kBcCols = 64;
struct BcSmem {
    static constexpr int PART = ITEM_U;                 // bytes [0, ITEM_U) of a block: -W, Qg, Kg, Aqk
    static constexpr int STAGE = PART + 512;            // + exp(G_L)
    static constexpr int DS = 2 * STAGE;                // float [128][64]
    static constexpr int DO = DS + DK * kBcCols * 4;    // float [64][64]
    static constexpr int DVN = DO + CH * kBcCols * 4;   // float [64][64]
    static constexpr int BAR = DVN + CH * kBcCols * 4;  // mbarriers [2]
    static constexpr int FLAG = BAR + 16;
    static constexpr int TOTAL = FLAG + 16;
};
static_assert(ITEM_GL == ITEM_U + 16384, "block layout");

// fp16 element (r, col) of a [64][128] SW128 tile pair, and of a [64][64] SW128 tile
__device__ __forceinline__ float tile128_at(const uint8_t *t, int r, int col)
{
    const int cb = (col & 63) * 2;
    const __half hv =
        *reinterpret_cast<const __half *>(t + (col >> 6) * 8192 + r * 128 + ((((cb >> 4) ^ (r & 7))) << 4) + (cb & 15));
    return __half2float(hv);
}
__device__ __forceinline__ float tile64_at(const uint8_t *t, int r, int col)
{
    const int cb = col * 2;
    const __half hv = *reinterpret_cast<const __half *>(t + r * 128 + ((((cb >> 4) ^ (r & 7))) << 4) + (cb & 15));
    return __half2float(hv);
}

__global__ void __launch_bounds__(kBcThreads, 1) kda_bwd_carry_kernel(const BwdParams p)
{
    using S = BcSmem;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x;
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
    float(*dS)[kBcCols] = reinterpret_cast<float(*)[kBcCols]>(sm + S::DS);
    float(*dO)[kBcCols] = reinterpret_cast<float(*)[kBcCols]>(sm + S::DO);
    float(*dVn)[kBcCols] = reinterpret_cast<float(*)[kBcCols]>(sm + S::DVN);
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
    // dS <- dht (or zero)
    {
        const int d = tid >> 2, c0 = 16 * (tid & 3);
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p.dht) x = *reinterpret_cast<const float4 *>(p.dht + unit_off + d * DV + vc0 + c0 + e);
            *reinterpret_cast<float4 *>(&dS[d][c0 + e]) = x;
        }
    }
    __syncthreads();

    bool ok = true;
    for (int it = 0; it < nck; ++it) {
        const int c = nck - 1 - it, st = it & 1;
        const uint8_t *blk = sm + st * S::STAGE;
        if (tid == 0 && c > 0) request(c - 1, st ^ 1);  // that stage was released by the previous iteration
        const int nrows = min(CH, len - c * CH);
        {
            // dS is the gradient at chunk c's end state: store it
            const int d = tid >> 2, c0 = 16 * (tid & 3);
            float *dst = p.dstates + ((c_begin + c) * p.HV + h) * DK * DV + d * DV + vc0 + c0;
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4 *>(dst + e) = *reinterpret_cast<const float4 *>(&dS[d][c0 + e]);
            // dO rows of the chunk (zero past the sequence's end)
            const int i = tid >> 3, cc = 8 * (tid & 7);
            float x[8] = {};
            if (i < nrows) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(
                    p.dout + ((row0 + static_cast<int64_t>(c) * CH + i) * p.HV + h) * DV + vc0 + cc);
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[2 * e] = bf16lo(w[e]);
                    x[2 * e + 1] = bf16hi(w[e]);
                }
            }
            *reinterpret_cast<float4 *>(&dO[i][cc]) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4 *>(&dO[i][cc + 4]) = make_float4(x[4], x[5], x[6], x[7]);
        }
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
            // dVnew[i][cc..cc+7] = sum_d Kg[i][d] dS[d][.] + sum_{j >= i} Aqk[j][i] dO[j][.]
            const int i = tid >> 3, cc = 8 * (tid & 7);
            float acc[8] = {};
            for (int d = 0; d < DK; ++d) {
                const float kg = tile128_at(blk + ITEM_KG, i, d);
                const float4 a = *reinterpret_cast<const float4 *>(&dS[d][cc]);
                const float4 b = *reinterpret_cast<const float4 *>(&dS[d][cc + 4]);
                acc[0] = __fmaf_rn(kg, a.x, acc[0]);
                acc[1] = __fmaf_rn(kg, a.y, acc[1]);
                acc[2] = __fmaf_rn(kg, a.z, acc[2]);
                acc[3] = __fmaf_rn(kg, a.w, acc[3]);
                acc[4] = __fmaf_rn(kg, b.x, acc[4]);
                acc[5] = __fmaf_rn(kg, b.y, acc[5]);
                acc[6] = __fmaf_rn(kg, b.z, acc[6]);
                acc[7] = __fmaf_rn(kg, b.w, acc[7]);
            }
            for (int j = i; j < CH; ++j) {
                const float aq = tile64_at(blk + ITEM_AQK, j, i);
                const float4 a = *reinterpret_cast<const float4 *>(&dO[j][cc]);
                const float4 b = *reinterpret_cast<const float4 *>(&dO[j][cc + 4]);
                acc[0] = __fmaf_rn(aq, a.x, acc[0]);
                acc[1] = __fmaf_rn(aq, a.y, acc[1]);
                acc[2] = __fmaf_rn(aq, a.z, acc[2]);
                acc[3] = __fmaf_rn(aq, a.w, acc[3]);
                acc[4] = __fmaf_rn(aq, b.x, acc[4]);
                acc[5] = __fmaf_rn(aq, b.y, acc[5]);
                acc[6] = __fmaf_rn(aq, b.z, acc[6]);
                acc[7] = __fmaf_rn(aq, b.w, acc[7]);
            }
            *reinterpret_cast<float4 *>(&dVn[i][cc]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            *reinterpret_cast<float4 *>(&dVn[i][cc + 4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        __syncthreads();
        {
            // dS[d][.] <- exp(G_L)_d dS[d][.] + sum_i Qg[i][d] dO[i][.] + sum_i (-W)[i][d] dVnew[i][.]
            const int d = tid >> 2, c0 = 16 * (tid & 3);
            const float e = reinterpret_cast<const float *>(blk + S::PART)[d];
            float acc[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) acc[x] = __fmul_rn(e, dS[d][c0 + x]);
            for (int i = 0; i < CH; ++i) {
                const float qg = tile128_at(blk + ITEM_QG, i, d), wn = tile128_at(blk + ITEM_WN, i, d);
#pragma unroll
                for (int x = 0; x < 16; x += 4) {
                    const float4 a = *reinterpret_cast<const float4 *>(&dO[i][c0 + x]);
                    const float4 b = *reinterpret_cast<const float4 *>(&dVn[i][c0 + x]);
                    acc[x] = __fmaf_rn(wn, b.x, __fmaf_rn(qg, a.x, acc[x]));
                    acc[x + 1] = __fmaf_rn(wn, b.y, __fmaf_rn(qg, a.y, acc[x + 1]));
                    acc[x + 2] = __fmaf_rn(wn, b.z, __fmaf_rn(qg, a.z, acc[x + 2]));
                    acc[x + 3] = __fmaf_rn(wn, b.w, __fmaf_rn(qg, a.w, acc[x + 3]));
                }
            }
#pragma unroll
            for (int x = 0; x < 16; ++x) dS[d][c0 + x] = acc[x];
        }
        __syncthreads();  // dS complete; this stage, dO and dVnew are free
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
        const int d = tid >> 2, c0 = 16 * (tid & 3);
#pragma unroll
        for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4 *>(p.dh0 + unit_off + d * DV + vc0 + c0 + e) =
                *reinterpret_cast<const float4 *>(&dS[d][c0 + e]);
    }
}

// ---------------------------------------------------------------------------------------------------------
// Chunk gradients: one CTA of 256 threads per (chunk, value head), fp32 throughout.
constexpr int kBwThreads = 256, kBwCols = 8;  // value columns per pass over the state
constexpr int kRow = 132;                     // padded row stride (floats) of the [64][128] operand tiles
constexpr int kRowC = 68;                     // padded row stride of the [64][64] tiles
constexpr int kVl = 12;                       // padded row stride of the [64][8] value-column tiles
constexpr int kSt = 132;                      // padded row stride of the transposed [8][128] state tiles
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
    // V pass buffers (inside WK)
    static constexpr int SVT = WK;                        // [8][kSt]  S[:, cols]^T
    static constexpr int DST = SVT + kBwCols * kSt * 4;   // [8][kSt]  dS'[:, cols]^T
    static constexpr int DOV = DST + kBwCols * kSt * 4;   // [64][kVl] dO
    static constexpr int DD = DOV + CH * kVl * 4;         // [64][kVl] D = v - Kb S
    static constexpr int VN = DD + CH * kVl * 4;          // [64][kVl] Vnew
    static constexpr int DVN = VN + CH * kVl * 4;         // [64][kVl] dVnew
    static constexpr int DV = DVN + CH * kVl * 4;         // [64][kVl] dv
    static constexpr int WK_END = DV + CH * kVl * 4;
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
    {
        const int i = tid >> 2, c0 = 32 * (tid & 3);
        const float *gr = p.g + ((row0 + i) * p.HV + h) * DK + c0;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
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
    for (int r = warp; r < CH; r += kBwThreads / 32) {
        uint2 rq = make_uint2(0u, 0u), rk = make_uint2(0u, 0u);
        if (r < nvalid) {
            rq = *reinterpret_cast<const uint2 *>(p.q + ((row0 + r) * p.H + hq) * DK + 4 * lane);
            rk = *reinterpret_cast<const uint2 *>(p.k + ((row0 + r) * p.H + hq) * DK + 4 * lane);
        }
        const uint2 nq = l2norm_row128_warp(rq), nk = l2norm_row128_warp(rk);
        // the forward's row denominators, kept to rebuild qn/kn bit for bit at the end
        const float dq = l2norm_den128_warp(rq), dk = l2norm_den128_warp(rk);
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

    // ---- 2. P (j < i) and Aqk (j <= i); thread: rows 4rg..4rg+3 (block I), columns cg + 16 jb ----
    {
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

    // ---- 3. T = (I + diag(beta) P)^-1, right-looking: row k is final before step k ----
    for (int k = 0; k < CH - 1; ++k) {
        const int rows = CH - 1 - k, cols = k + 1;
        for (int x = tid; x < rows * cols; x += kBwThreads) {
            const int i = k + 1 + x / cols, j = x % cols;
            TT[i][j] = __fmaf_rn(-__fmul_rn(beta[i], PP[i][k]), TT[k][j], TT[i][j]);
        }
        __syncthreads();
    }

    // ---- 4-5. passes over 8 value columns at a time ----
    float(*SVT)[kSt] = reinterpret_cast<float(*)[kSt]>(sm + S::SVT);
    float(*DST)[kSt] = reinterpret_cast<float(*)[kSt]>(sm + S::DST);
    float(*DOV)[kVl] = reinterpret_cast<float(*)[kVl]>(sm + S::DOV);
    float(*DDv)[kVl] = reinterpret_cast<float(*)[kVl]>(sm + S::DD);
    float(*VN)[kVl] = reinterpret_cast<float(*)[kVl]>(sm + S::VN);
    float(*DVN)[kVl] = reinterpret_cast<float(*)[kVl]>(sm + S::DVN);
    float(*DVv)[kVl] = reinterpret_cast<float(*)[kVl]>(sm + S::DV);
    const float *Sg = p.states + item * DK * DV;
    const float *dSg = p.dstates + item * DK * DV;
    // register accumulators over the value columns: thread rows 4rg..+3, key columns 8cg..+7 (dQg, dKb, dKg)
    // and rows 4rg..+3, token columns cg + 16jb (dAqk, dA)
    const int rg = tid >> 4, cg = tid & 15;
    float aQ[4][8] = {}, aB[4][8] = {}, aG[4][8] = {}, aAq[4][4] = {}, aA[4][4] = {};
    for (int vb = 0; vb < DV; vb += kBwCols) {
        {
            // S and dS' columns vb..vb+7, transposed; thread: key row d = tid >> 1, 4 columns
            const int d = tid >> 1, c4 = 4 * (tid & 1);
            const float4 x = *reinterpret_cast<const float4 *>(Sg + d * DV + vb + c4);
            const float4 y = *reinterpret_cast<const float4 *>(dSg + d * DV + vb + c4);
            SVT[c4][d] = x.x;
            SVT[c4 + 1][d] = x.y;
            SVT[c4 + 2][d] = x.z;
            SVT[c4 + 3][d] = x.w;
            DST[c4][d] = y.x;
            DST[c4 + 1][d] = y.y;
            DST[c4 + 2][d] = y.z;
            DST[c4 + 3][d] = y.w;
            // dE_L term of dG_L: sum over these columns of exp(G_L) S dS'
            const float part = __fmaf_rn(x.w, y.w, __fmaf_rn(x.z, y.z, __fmaf_rn(x.y, y.y, __fmul_rn(x.x, y.x))));
            atomicAdd(&dgl[d], __fmul_rn(egl[d], part));
            // dO rows (zero past the end)
            if (tid < 2 * CH) {
                const int i = tid >> 1, cc = 4 * (tid & 1);
                float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < nvalid) {
                    const uint2 raw = *reinterpret_cast<const uint2 *>(p.dout + ((row0 + i) * p.HV + h) * DV + vb + cc);
                    o = make_float4(bf16lo(raw.x), bf16hi(raw.x), bf16lo(raw.y), bf16hi(raw.y));
                }
                *reinterpret_cast<float4 *>(&DOV[i][cc]) = o;
            }
        }
        __syncthreads();
        {
            // (a) D[i][c] = v[i][c] - sum_d Kb_id S[d][c], Kb = KA exp(m_I); thread: row i = tid >> 2, 2 columns
            const int i = tid >> 2, c2 = 2 * (tid & 3), I = i >> 4;
            float a0 = 0.f, a1 = 0.f;
            for (int d = 0; d < DK; ++d) {
                const float kb = __fmul_rn(KA[i][d], EM[I][d]);
                a0 = __fmaf_rn(kb, SVT[c2][d], a0);
                a1 = __fmaf_rn(kb, SVT[c2 + 1][d], a1);
            }
            float v0 = 0.f, v1 = 0.f;
            if (i < nvalid) {
                const __nv_bfloat162 vv =
                    *reinterpret_cast<const __nv_bfloat162 *>(p.v + ((row0 + i) * p.HV + h) * DV + vb + c2);
                v0 = __low2float(vv);
                v1 = __high2float(vv);
            }
            DDv[i][c2] = __fsub_rn(v0, a0);
            DDv[i][c2 + 1] = __fsub_rn(v1, a1);
        }
        __syncthreads();
        {
            // (b) Vnew = T diag(beta) D;  (c) dVnew = Kg dS' + Aqk^T dO, Kg = KB exp(G_L - m_I)
            const int i = tid >> 2, c2 = 2 * (tid & 3), I = i >> 4;
            float x0 = 0.f, x1 = 0.f;
            for (int j = 0; j <= i; ++j) {
                const float t = __fmul_rn(TT[i][j], beta[j]);
                x0 = __fmaf_rn(t, DDv[j][c2], x0);
                x1 = __fmaf_rn(t, DDv[j][c2 + 1], x1);
            }
            VN[i][c2] = x0;
            VN[i][c2 + 1] = x1;
            float y0 = 0.f, y1 = 0.f;
            for (int d = 0; d < DK; ++d) {
                const float kg = __fmul_rn(KB[i][d], EGLM[I][d]);
                y0 = __fmaf_rn(kg, DST[c2][d], y0);
                y1 = __fmaf_rn(kg, DST[c2 + 1][d], y1);
            }
            for (int j = i; j < CH; ++j) {
                y0 = __fmaf_rn(AQ[j][i], DOV[j][c2], y0);
                y1 = __fmaf_rn(AQ[j][i], DOV[j][c2 + 1], y1);
            }
            DVN[i][c2] = y0;
            DVN[i][c2 + 1] = y1;
        }
        __syncthreads();
        {
            // (d) dv = diag(beta) T^T dVnew
            const int i = tid >> 2, c2 = 2 * (tid & 3);
            float x0 = 0.f, x1 = 0.f;
            for (int j = i; j < CH; ++j) {
                x0 = __fmaf_rn(TT[j][i], DVN[j][c2], x0);
                x1 = __fmaf_rn(TT[j][i], DVN[j][c2 + 1], x1);
            }
            x0 = __fmul_rn(beta[i], x0);
            x1 = __fmul_rn(beta[i], x1);
            DVv[i][c2] = x0;
            DVv[i][c2 + 1] = x1;
            if (i < nvalid)
                *reinterpret_cast<__nv_bfloat162 *>(p.dv + ((row0 + i) * p.HV + h) * DV + vb + c2) =
                    __floats2bfloat162_rn(x0, x1);
        }
        __syncthreads();
        // (e) accumulate dQg += dO S^T, dKb -= dv S^T, dKg += Vnew dS'^T, dAqk += dO Vnew^T, dA += dVnew D^T
#pragma unroll
        for (int c = 0; c < kBwCols; ++c) {
            float sv[8], dsv[8];
            *reinterpret_cast<float4 *>(&sv[0]) = *reinterpret_cast<const float4 *>(&SVT[c][8 * cg]);
            *reinterpret_cast<float4 *>(&sv[4]) = *reinterpret_cast<const float4 *>(&SVT[c][8 * cg + 4]);
            *reinterpret_cast<float4 *>(&dsv[0]) = *reinterpret_cast<const float4 *>(&DST[c][8 * cg]);
            *reinterpret_cast<float4 *>(&dsv[4]) = *reinterpret_cast<const float4 *>(&DST[c][8 * cg + 4]);
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int i = 4 * rg + ii;
                const float o = DOV[i][c], dv_ = DVv[i][c], vn = VN[i][c], dvn = DVN[i][c];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    aQ[ii][e] = __fmaf_rn(o, sv[e], aQ[ii][e]);
                    aB[ii][e] = __fmaf_rn(-dv_, sv[e], aB[ii][e]);
                    aG[ii][e] = __fmaf_rn(vn, dsv[e], aG[ii][e]);
                }
#pragma unroll
                for (int jb = 0; jb < 4; ++jb) {
                    const int j = cg + 16 * jb;
                    aAq[ii][jb] = __fmaf_rn(o, VN[j][c], aAq[ii][jb]);
                    aA[ii][jb] = __fmaf_rn(dvn, DDv[j][c], aA[ii][jb]);
                }
            }
        }
        __syncthreads();
    }

    // ---- 6. dbeta, dL, M = diag(beta) dL, N = dAqk ----
    float(*DA)[kRowC] = reinterpret_cast<float(*)[kRowC]>(sm + S::DA);
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
            const int i = 4 * rg + ii, j = cg + 16 * jb;
            DA[i][j] = aA[ii][jb];
            AQ[i][j] = j <= i ? aAq[ii][jb] : 0.f;  // Aqk is no longer needed: N takes its place
        }
    __syncthreads();
    if (tid < CH) {  // dbeta_j += sum_{i >= j} dA_ij T_ij
        float acc = 0.f;
        for (int i = tid; i < CH; ++i) acc = __fmaf_rn(DA[i][tid], TT[i][tid], acc);
        dbeta[tid] = acc;
    }
    // Y = T^T (dA diag(beta)): Y[a][e] = beta_e sum_{c >= a} T[c][a] dA[c][e]
    float y[4][4] = {};
    for (int c = 4 * rg; c < CH; ++c) {
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const float t = TT[c][4 * rg + ii];
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) y[ii][jb] = __fmaf_rn(t, DA[c][cg + 16 * jb], y[ii][jb]);
        }
    }
    __syncthreads();  // every read of dA is done
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) DA[4 * rg + ii][cg + 16 * jb] = __fmul_rn(beta[cg + 16 * jb], y[ii][jb]);
    __syncthreads();
    // dL[a][b] = -sum_{e <= b} Y[a][e] T[b][e] (a > b); dbeta_a += sum_b dL_ab P_ab; M = diag(beta) dL
    {
        float dl[4][4] = {};
        for (int e = 0; e < CH; ++e) {
            float ye[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) ye[ii] = DA[4 * rg + ii][e];
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {
                const float t = TT[cg + 16 * jb][e];  // zero for e > b
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) dl[ii][jb] = __fmaf_rn(-ye[ii], t, dl[ii][jb]);
            }
        }
        float rowp[4] = {};
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {
                const int a = 4 * rg + ii, b = cg + 16 * jb;
                if (b < a) rowp[ii] = __fmaf_rn(dl[ii][jb], PP[a][b], rowp[ii]);
                else dl[ii][jb] = 0.f;
            }
        // the 16 threads of a row group are 16 consecutive lanes
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) rowp[ii] = __fadd_rn(rowp[ii], __shfl_xor_sync(0xffffffffu, rowp[ii], off));
        }
        __syncthreads();  // every read of P and T is done (dbeta's column sums above included)
        if (cg == 0) {
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) atomicAdd(&dbeta[4 * rg + ii], rowp[ii]);
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) PP[4 * rg + ii][cg + 16 * jb] = __fmul_rn(beta[4 * rg + ii], dl[ii][jb]);
    }
    __syncthreads();
    float(*MM)[kRowC] = PP;
    float(*NN)[kRowC] = AQ;

    // ---- 7. element terms and pairwise terms; thread: rows 4rg..+3 (block I), key columns 8cg..+7 ----
    const int I = rg >> 2;
    float rq[4][8], rk[4][8], rG[4][8];
    {
        // rebuild qn/kn of the owned rows from the raw rows (the same normalisation, bit for bit)
        float qn[4][8], kn[4][8];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = 4 * rg + ii;
            uint4 rqw = make_uint4(0u, 0u, 0u, 0u), rkw = rqw;
            if (i < nvalid) {
                rqw = *reinterpret_cast<const uint4 *>(p.q + ((row0 + i) * p.H + hq) * DK + 8 * cg);
                rkw = *reinterpret_cast<const uint4 *>(p.k + ((row0 + i) * p.H + hq) * DK + 8 * cg);
            }
            const uint32_t wq[4] = {rqw.x, rqw.y, rqw.z, rqw.w}, wk[4] = {rkw.x, rkw.y, rkw.z, rkw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                qn[ii][2 * e] = bf16lo(wq[e]);
                qn[ii][2 * e + 1] = bf16hi(wq[e]);
                kn[ii][2 * e] = bf16lo(wk[e]);
                kn[ii][2 * e + 1] = bf16hi(wk[e]);
            }
        }
        // the quotient and rounding of the normalisation, with the row denominators stored above
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const float dq = denq[4 * rg + ii], dk = denk[4 * rg + ii];
            const float rqi = __frcp_rn(dq), rki = __frcp_rn(dk);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const uint32_t pq = pack_bf16(div_rn_with_rcp(qn[ii][e], dq, rqi), div_rn_with_rcp(qn[ii][e + 1], dq, rqi));
                const uint32_t pk = pack_bf16(div_rn_with_rcp(kn[ii][e], dk, rki), div_rn_with_rcp(kn[ii][e + 1], dk, rki));
                qn[ii][e] = bf16lo(pq);
                qn[ii][e + 1] = bf16hi(pq);
                kn[ii][e] = bf16lo(pk);
                kn[ii][e + 1] = bf16hi(pk);
            }
        }
        // X3 = s exp(G) dQg, X1 = exp(G) dKb, X2 = exp(G_L - G) dKg
        float glp[8] = {};
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = 4 * rg + ii;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int d = 8 * cg + e;
                const float x = __fsub_rn(G[i][d], G[16 * I + 7][d]);
                const float eg = __fmul_rn(bwd_exp(x), EM[I][d]), eglg = __fmul_rn(bwd_exp(-x), EGLM[I][d]);
                const float x3 = __fmul_rn(__fmul_rn(s, eg), aQ[ii][e]);
                const float x1 = __fmul_rn(eg, aB[ii][e]);
                const float x2 = __fmul_rn(eglg, aG[ii][e]);
                rq[ii][e] = x3;
                rk[ii][e] = __fadd_rn(x1, x2);
                rG[ii][e] = __fmaf_rn(qn[ii][e], x3, __fmul_rn(kn[ii][e], __fsub_rn(x1, x2)));
                glp[e] = __fmaf_rn(kn[ii][e], x2, glp[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) atomicAdd(&dgl[8 * cg + e], glp[e]);
    }
    {
        // R1'_id = sum_{J <= I} sum_{j in J} M_ij KB_jd c_IJd,  R3'_id = the same with N
        float r1[4][8] = {}, r3[4][8] = {};
        for (int J = 0; J <= I; ++J) {
            for (int j = 16 * J; j < 16 * J + 16; ++j) {
                float kb[8];
                *reinterpret_cast<float4 *>(&kb[0]) = *reinterpret_cast<const float4 *>(&KB[j][8 * cg]);
                *reinterpret_cast<float4 *>(&kb[4]) = *reinterpret_cast<const float4 *>(&KB[j][8 * cg + 4]);
                if (J < I) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) kb[e] = __fmul_rn(kb[e], CF[cf_index(I, J)][8 * cg + e]);
                }
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    const float m = MM[4 * rg + ii][j], nn = NN[4 * rg + ii][j];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        r1[ii][e] = __fmaf_rn(m, kb[e], r1[ii][e]);
                        r3[ii][e] = __fmaf_rn(nn, kb[e], r3[ii][e]);
                    }
                }
            }
        }
        // R1 = a R1', R3 = s a R3' with a = exp(G - m_I); dkn += R1, dqn += R3, dG += kn R1 + qn R3
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = 4 * rg + ii;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int d = 8 * cg + e;
                const float a = bwd_exp(__fsub_rn(G[i][d], G[16 * I + 7][d]));
                const float R1 = __fmul_rn(a, r1[ii][e]), R3 = __fmul_rn(__fmul_rn(s, a), r3[ii][e]);
                rk[ii][e] = __fadd_rn(rk[ii][e], R1);
                rq[ii][e] = __fadd_rn(rq[ii][e], R3);
                rG[ii][e] = __fmaf_rn(KA[i][d], r1[ii][e], rG[ii][e]);
                rG[ii][e] = __fmaf_rn(__fmul_rn(s, QA[i][d]), r3[ii][e], rG[ii][e]);
            }
        }
    }
    {
        // R24'_jd = sum_{I' >= J} sum_{i in I'} (M_ij KA_id + s N_ij QA_id) c_I'Jd  (rows j = 4rg..+3, J = I)
        float r2[4][8] = {};
        for (int I2 = I; I2 < 4; ++I2) {
            for (int i = 16 * I2; i < 16 * I2 + 16; ++i) {
                float ka[8], qa[8];
                *reinterpret_cast<float4 *>(&ka[0]) = *reinterpret_cast<const float4 *>(&KA[i][8 * cg]);
                *reinterpret_cast<float4 *>(&ka[4]) = *reinterpret_cast<const float4 *>(&KA[i][8 * cg + 4]);
                *reinterpret_cast<float4 *>(&qa[0]) = *reinterpret_cast<const float4 *>(&QA[i][8 * cg]);
                *reinterpret_cast<float4 *>(&qa[4]) = *reinterpret_cast<const float4 *>(&QA[i][8 * cg + 4]);
#pragma unroll
                for (int e = 0; e < 8; ++e) qa[e] = __fmul_rn(s, qa[e]);
                if (I2 > I) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float cf = CF[cf_index(I2, I)][8 * cg + e];
                        ka[e] = __fmul_rn(ka[e], cf);
                        qa[e] = __fmul_rn(qa[e], cf);
                    }
                }
                const float4 m4 = *reinterpret_cast<const float4 *>(&MM[i][4 * rg]);
                const float4 n4 = *reinterpret_cast<const float4 *>(&NN[i][4 * rg]);
                const float m[4] = {m4.x, m4.y, m4.z, m4.w}, nn[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                    for (int e = 0; e < 8; ++e) r2[jj][e] = __fmaf_rn(m[jj], ka[e], __fmaf_rn(nn[jj], qa[e], r2[jj][e]));
            }
        }
        // R24 = b R24' with b = exp(m_I - G); dkn += R24, dG -= kn R24 = KB R24'
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int j = 4 * rg + jj;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int d = 8 * cg + e;
                const float b = bwd_exp(__fsub_rn(G[16 * I + 7][d], G[j][d]));
                rk[jj][e] = __fmaf_rn(b, r2[jj][e], rk[jj][e]);
                rG[jj][e] = __fmaf_rn(-KB[j][d], r2[jj][e], rG[jj][e]);
            }
        }
    }
    // dqn, dkn out (valid rows)
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
        const int i = 4 * rg + ii;
        if (i < nvalid) {
            float *dq = p.dqn + ((row0 + i) * p.HV + h) * DK + 8 * cg;
            float *dk = p.dkn + ((row0 + i) * p.HV + h) * DK + 8 * cg;
            *reinterpret_cast<float4 *>(dq) = make_float4(rq[ii][0], rq[ii][1], rq[ii][2], rq[ii][3]);
            *reinterpret_cast<float4 *>(dq + 4) = make_float4(rq[ii][4], rq[ii][5], rq[ii][6], rq[ii][7]);
            *reinterpret_cast<float4 *>(dk) = make_float4(rk[ii][0], rk[ii][1], rk[ii][2], rk[ii][3]);
            *reinterpret_cast<float4 *>(dk + 4) = make_float4(rk[ii][4], rk[ii][5], rk[ii][6], rk[ii][7]);
        }
    }
    __syncthreads();  // KA/QA/KB/G reads done; dgl complete
    // dG rows into the KA region (unpadded [64][128]), then the reverse cumulative sum per key column
    float(*dG)[DK] = reinterpret_cast<float(*)[DK]>(sm + S::KA);
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int e = 0; e < 8; ++e) dG[4 * rg + ii][8 * cg + e] = rG[ii][e];
    __syncthreads();
    if (tid < DK) {
        float acc = dgl[tid];  // G_L = G of the last row
        for (int i = CH - 1; i >= 0; --i) {
            acc = __fadd_rn(acc, dG[i][tid]);
            if (i < nvalid) p.dg[((row0 + i) * p.HV + h) * DK + tid] = acc;
        }
    }
    if (tid < nvalid) p.dbeta[(row0 + tid) * p.HV + h] = dbeta[tid];
}

// ---------------------------------------------------------------------------------------------------------
// dq (dk) row of Q/K head hq = J(x)^T sum over the value heads of its group of dqn (dkn), with
// J(x) the Jacobian of x / sqrt(sum x^2 + 1e-6): dx = dy / n - x (x . dy) / n^3.  One warp per (row, head, q|k).
__global__ void __launch_bounds__(256) kda_bwd_norm_kernel(const BwdParams p, int64_t rows)
{
    const int lane = threadIdx.x & 31;
    const int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int64_t units = rows * p.H * 2;
    if (w >= units) return;
    const int which = static_cast<int>(w & 1);
    const int64_t rh = w >> 1, row = rh / p.H;
    const int hq = static_cast<int>(rh % p.H);
    if (p.cu && row >= p.cu[p.N]) return;  // outside every sequence
    const __nv_bfloat16 *x = (which ? p.k : p.q) + (row * p.H + hq) * DK + 4 * lane;
    const float *dy = (which ? p.dkn : p.dqn) + (row * p.HV) * DK + 4 * lane;
    const int grp = p.HV / p.H;
    const uint2 raw = *reinterpret_cast<const uint2 *>(x);
    const float xv[4] = {bf16lo(raw.x), bf16hi(raw.x), bf16lo(raw.y), bf16hi(raw.y)};
    float g[4] = {};
    for (int j = 0; j < grp; ++j) {
        const float4 t = *reinterpret_cast<const float4 *>(dy + (hq * grp + j) * DK);
        g[0] = __fadd_rn(g[0], t.x);
        g[1] = __fadd_rn(g[1], t.y);
        g[2] = __fadd_rn(g[2], t.z);
        g[3] = __fadd_rn(g[3], t.w);
    }
    float ss = 0.f, xd = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        ss = __fmaf_rn(xv[e], xv[e], ss);
        xd = __fmaf_rn(xv[e], g[e], xd);
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
    for (int e = 0; e < 4; ++e) out[e] = __fmaf_rn(-xv[e], c3, __fmul_rn(g[e], inv));
    __nv_bfloat16 *dst = (which ? p.dk : p.dq) + (row * p.H + hq) * DK + 4 * lane;
    *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16(out[0], out[1]), pack_bf16(out[2], out[3]));
}

}  // namespace kda
