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
//   kda_bwd_chunk_kernel  every chunk's gradients at once (fp32 arithmetic;
//                         fp16 and TF32 tensor-core MMAs for the products),
//   kda_bwd_norm_kernel   sums a Q/K head's group and applies the L2
//                         normalisation's Jacobian.
// Gate factors exp(G_i - G_j) are formed per 16-token block I with the
// reference m_I = G at the block's eighth token:
//   exp(G_i - G_j) = exp(G_i - m_I) * exp(m_I - m_J) * exp(m_J - G_j),
// every factor at most exp(8 |g|max) away from 1 and the middle one <= 1.
#pragma once
#include <type_traits>

#include "kda_common.cuh"
#include "kda_norm.cuh"
#include "ptx.cuh"
#include "tc.cuh"

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
// Reverse carry on the 5th-generation tensor cores: one CTA per (sequence, value head), walking the chunks
// backwards.  Transposed, with the value dimension as the MMA's M = 128 and dS' the gradient at chunk c's end:
//   dVnew^T = dS'^T Kg^T + dO^T Aqk                 (groups 1 and 2: M = 128 values, N = 64 tokens)
//   dS^T    = dS'^T diag(exp(G_L)) + dO^T Qg + dVnew^T (-W)   (groups 3 and 4: N = 128 keys)
// dS^T (fp32) stays in TMEM.  Its fp16 copy there is the A operand of group 1, and the fp16 dVnew^T of group 4.
// dO^T is an MN-major A operand in shared memory: the epilogue stages each chunk's dO rows there in fp16 (the
// blocks' tiles are fp16).  The blocks' -W, Qg, Kg and Aqk tiles are read in place from a three-stage bulk-copy
// ring: Kg K-major (as Kg^T), Aqk, Qg and -W MN-major.
// Warps 0-15 (epilogue) own TMEM lane v = 32 (warp % 4) + lane and a quarter of the key (and token) columns;
// warp 16 streams the blocks; warp 17 allocates TMEM and issues the MMAs.  Every wait is bounded.
__device__ __forceinline__ void bwd_mma_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// kind::f16 instruction descriptor with either operand MN-major (bit 15: A, bit 16: B); fp16 operands
__host__ __device__ constexpr uint32_t bwd_idesc(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

constexpr int kBcEpiWarps = 16;
constexpr int kBcThreads = (kBcEpiWarps + 2) * 32;
struct BcSmem {
    static constexpr int PART = ITEM_U;                           // bytes [0, ITEM_U) of a block: -W, Qg, Kg, Aqk
    static constexpr int GLO = PART;                              // exp(G_L) after them in the stage
    static constexpr int STAGE = ((PART + 512 + 1023) / 1024) * 1024;
    static constexpr int NST = 3;
    static constexpr int DO = NST * STAGE;                        // fp16 dO [64 tok][128 v] x 2 (SW128, 64-v halves)
    static constexpr int BAR = DO + 2 * CH * DV * 2;
    // mbarriers: full[NST] empty[NST] barV barS sready vready dready oready[2]
    static constexpr int TMEM_SLOT = BAR + (2 * NST + 7) * 8;
    static constexpr int ABORT = TMEM_SLOT + 4;
    static constexpr int TOTAL = ABORT + 4;
};
static_assert(BcSmem::TOTAL <= 232448, "reverse carry shared memory");
static_assert(ITEM_GL == ITEM_U + 16384, "block layout");
// TMEM columns: dS^T fp32 (128) | dVnew^T fp32 (64) | fp16 dS'^T (64) | fp16 dVnew^T (32)
constexpr uint32_t BC_DS = 0, BC_DV = 128, BC_AS = 192, BC_AV = 256, BC_COLS = 512;

__global__ void __launch_bounds__(kBcThreads, 1) kda_bwd_carry_kernel(const BwdParams p)
{
    using S = BcSmem;
    constexpr int NST = S::NST;
    static_assert(NST == 3, "the issuer body is instantiated for three stages");
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x / p.HV, h = blockIdx.x % p.HV;
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
    const int64_t unit_off = (static_cast<int64_t>(n) * p.HV + h) * DK * DV;

    const uint32_t full0 = sb + S::BAR, empty0 = full0 + 8 * NST, barV = full0 + 16 * NST, barS = barV + 8,
                   sready = barV + 16, vready = barV + 24, dready = barV + 32, oready0 = barV + 40;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::ABORT);
    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1 + kBcEpiWarps);
        }
        mbar_init(barV, 1);
        mbar_init(barS, 1);
        mbar_init(sready, kBcEpiWarps);
        mbar_init(vready, kBcEpiWarps);
        mbar_init(dready, kBcEpiWarps);
        mbar_init(oready0, kBcEpiWarps);
        mbar_init(oready0 + 8, kBcEpiWarps);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kBcEpiWarps + 1) tc_alloc(sb + S::TMEM_SLOT, BC_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // All 512 columns are allocated, so the allocation starts at lane 0, column 0.
    const uint32_t tmem_alloc = *reinterpret_cast<volatile uint32_t *>(sm + S::TMEM_SLOT);
    auto fail = [&](unsigned code) {
        atomicOr(p.err, code);
        *abort_flag = 1;
    };
    if (tmem_alloc != 0) {
        if (tid == 0) fail(ERR_TMEM_BASE);
        nck = 0;
    }

    if (warp == kBcEpiWarps) {
        // ---------------- producer: iteration it carries chunk nck - 1 - it ----------------
        if (lane == 0) {
            for (int it = 0; it < nck && !*abort_flag; ++it) {
                const int s = it % NST;
                if (it >= NST && !mbar_wait(empty0 + 8 * s, ((it / NST) - 1) & 1)) {
                    fail(ERR_PIPE_EMPTY_WAIT);
                    break;
                }
                const uint8_t *src = p.items + ((c_begin + nck - 1 - it) * p.HV + h) * ITEM_BYTES;
                mbar_expect_tx(full0 + 8 * s, S::PART + 512);
                bulk_load(sb + s * S::STAGE, src, S::PART, full0 + 8 * s);
                bulk_load(sb + s * S::STAGE + S::GLO, src + ITEM_GL, 512, full0 + 8 * s);
            }
        }
    } else if (warp == kBcEpiWarps + 1) {
        // ---------------- MMA issuer ----------------
        const uint32_t iv_k = bwd_idesc(128, 64, false, false);   // A TMEM, B K-major (Kg^T)
        const uint32_t iv_mm = bwd_idesc(128, 64, true, true);    // A dO^T MN-major, B Aqk MN-major
        const uint32_t is_mm = bwd_idesc(128, 128, true, true);   // A dO^T MN-major, B Qg MN-major
        const uint32_t is_tm = bwd_idesc(128, 128, false, true);  // A TMEM, B -W MN-major
        const uint64_t dk0 = sw128_desc(sb, 16, 1024), kk0 = sw128_desc(sb, 8192, 1024);
        const uint32_t dhi = static_cast<uint32_t>(dk0 >> 32), khi = static_cast<uint32_t>(kk0 >> 32);
        auto kstep = [](int ks) { return static_cast<uint32_t>((ks >> 2) * 512 + (ks & 3) * 2); };
        auto body = [&](int it, auto stage) -> bool {
            constexpr int st = decltype(stage)::value;
            constexpr uint32_t so = static_cast<uint32_t>(st * (S::STAGE >> 4));
            uint32_t dlo = static_cast<uint32_t>(dk0), klo = static_cast<uint32_t>(kk0);
            asm volatile("" : "+r"(dlo), "+r"(klo));
            auto dd = [&](uint32_t off) { return (static_cast<uint64_t>(dhi) << 32) | (dlo + off); };
            auto kd = [&](uint32_t off) { return (static_cast<uint64_t>(khi) << 32) | (klo + off); };
            const int b = it & 1;
            const uint32_t dob = static_cast<uint32_t>((S::DO + b * CH * DV * 2) >> 4);
            bool w = mbar_wait(full0 + 8 * st, (it / NST) & 1) && mbar_wait_spin(oready0 + 8 * b, (it >> 1) & 1) &&
                     mbar_wait_spin(sready, it & 1);
            if (!__all_sync(0xffffffffu, w)) return false;
            tc_fence_after();
            // groups 1 and 2: dVnew^T = dS'^T Kg^T + dO^T Aqk
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                tc_mma_ts_warp(BC_DV, BC_AS + 8 * ks, dd(so + (ITEM_KG >> 4) + kstep(ks)), iv_k, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                bwd_mma_ss_warp(BC_DV, kd(dob + 128 * ks), kd(so + (ITEM_AQK >> 4) + 128 * ks), iv_mm, 1);
            tc_commit_warp(barV);
            // group 3: dS^T += dO^T Qg, onto dS'^T diag(exp(G_L)) (the epilogue's decay)
            if (!__all_sync(0xffffffffu, mbar_wait_spin(dready, it & 1))) return false;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                bwd_mma_ss_warp(BC_DS, kd(dob + 128 * ks), kd(so + (ITEM_QG >> 4) + 128 * ks), is_mm, 1);
            // group 4: dS^T += dVnew^T (-W)
            if (!__all_sync(0xffffffffu, mbar_wait_spin(vready, it & 1))) return false;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc_mma_ts_warp(BC_DS, BC_AV + 8 * ks, kd(so + (ITEM_WN >> 4) + 128 * ks), is_tm, 1);
            tc_commit_warp(barS);
            tc_commit_warp(empty0 + 8 * st);
            return true;
        };
        for (int it = 0; it < nck; ++it) {
            if (__any_sync(0xffffffffu, *abort_flag)) break;
            const int st = it % NST;
            const bool ok = st == 0   ? body(it, std::integral_constant<int, 0>{})
                            : st == 1 ? body(it, std::integral_constant<int, 1>{})
                                      : body(it, std::integral_constant<int, 2>{});
            if (!ok) {
                if (lane == 0) fail(ERR_PIPE_FULL_WAIT);
                break;
            }
        }
    } else {
        // ---------------- epilogue: value column v, key quarter kq (keys 32kq..), token quarter (16kq..) ----------
        const int qd = warp & 3, kq = warp >> 2;
        const int v = 32 * qd + lane;
        const uint32_t lb = static_cast<uint32_t>(32 * qd) << 16;
        auto arrive = [&](uint32_t bar) {
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        // fp16 copy of dS'^T[v][32kq ..] -> the A operand of the next group 1
        auto pack_ds = [&](const uint32_t (&r)[32]) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = pack_f16(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
            tc_st16(lb + BC_AS + 16 * kq, w);
        };
        // dS' of chunk c (the gradient at its end state) -> dstates, bf16 [key][v]
        auto store_dstates = [&](const uint32_t (&r)[32], int c) {
            __nv_bfloat16 *dst = p.dstates + ((c_begin + c) * p.HV + h) * DK * DV + v;
#pragma unroll
            for (int j = 0; j < 32; ++j) dst[(32 * kq + j) * DV] = __float2bfloat16_rn(__uint_as_float(r[j]));
        };
        // dO rows of chunk c, fp16, into buffer b: thread's two 16-byte pieces (row t, v-chunk vc), zero past the end
        uint4 dov[2];
        auto load_do = [&](int c) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int idx = tid + k * (kBcEpiWarps * 32), t = idx >> 4, vc = idx & 15;
                dov[k] = make_uint4(0u, 0u, 0u, 0u);
                if (c >= 0 && t < min(CH, len - c * CH))
                    dov[k] = *reinterpret_cast<const uint4 *>(
                        p.dout + ((row0 + static_cast<int64_t>(c) * CH + t) * p.HV + h) * DV + 8 * vc);
            }
        };
        auto put_do = [&](int b) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int idx = tid + k * (kBcEpiWarps * 32), t = idx >> 4, vc = idx & 15;
                const uint4 raw = dov[k];
                const uint4 w = make_uint4(pack_f16(bf16lo(raw.x), bf16hi(raw.x)), pack_f16(bf16lo(raw.y), bf16hi(raw.y)),
                                           pack_f16(bf16lo(raw.z), bf16hi(raw.z)), pack_f16(bf16lo(raw.w), bf16hi(raw.w)));
                *reinterpret_cast<uint4 *>(sm + S::DO + b * CH * DV * 2 + (vc >> 3) * 8192 + t * 128 +
                                           (((vc & 7) ^ (t & 7)) << 4)) = w;
            }
            fence_proxy_async();
        };

        bool alive = tmem_alloc == 0;
        {
            // dS' of the last chunk = dht (or zero)
            uint32_t r[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                r[j] = __float_as_uint(p.dht ? p.dht[unit_off + (32 * kq + j) * DV + v] : 0.f);
            if (alive && nck > 0) {
                tc_st32(lb + BC_DS + 32 * kq, r);
                pack_ds(r);
                load_do(nck - 1);
                put_do(0);
                arrive(oready0);
                arrive(sready);
                store_dstates(r, nck - 1);
                load_do(nck - 2);
            } else if (alive && p.dh0) {
#pragma unroll
                for (int j = 0; j < 32; ++j) p.dh0[unit_off + (32 * kq + j) * DV + v] = __uint_as_float(r[j]);
            }
        }
        for (int it = 0; it < nck && alive && !*abort_flag; ++it) {
            const int c = nck - 1 - it, st = it % NST;
            const float2 *gl = reinterpret_cast<const float2 *>(sm + st * S::STAGE + S::GLO) + 16 * kq;
            if (!mbar_wait(full0 + 8 * st, (it / NST) & 1)) {
                fail(ERR_PIPE_FULL_WAIT);
                break;
            }
            // 1. decay dS'^T by exp(G_L) of chunk c (group 1 reads only the fp16 copy)
            {
                uint32_t r[32];
                tc_ld32(lb + BC_DS + 32 * kq, r);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float2 x = mul2(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), gl[j]);
                    r[2 * j] = __float_as_uint(x.x);
                    r[2 * j + 1] = __float_as_uint(x.y);
                }
                tc_st32(lb + BC_DS + 32 * kq, r);
            }
            arrive(dready);
            // 2. dO of chunk c - 1 into the other buffer (its last reader, chunk c + 1's MMAs, completed before the
            //    previous iteration's barS), then request chunk c - 2's rows
            if (c > 0) {
                put_do((it + 1) & 1);
                arrive(oready0 + 8 * ((it + 1) & 1));
                load_do(c - 2);
            }
            // 3. dVnew^T -> fp16 A operand of group 4
            if (!mbar_wait_spin(barV, it & 1)) {
                fail(ERR_PIPE_FULL_WAIT);
                break;
            }
            tc_fence_after();
            {
                uint32_t pr[16], w[8];
                tc_ld16(lb + BC_DV + 16 * kq, pr);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 8; ++j) w[j] = pack_f16(__uint_as_float(pr[2 * j]), __uint_as_float(pr[2 * j + 1]));
                tc_st8(lb + BC_AV + 8 * kq, w);
            }
            arrive(vready);
            // 4. dS^T is now dS' of chunk c - 1: its fp16 copy, then dstates (or dh0 after chunk 0)
            if (!mbar_wait_spin(barS, it & 1)) {
                fail(ERR_PIPE_FULL_WAIT);
                break;
            }
            tc_fence_after();
            {
                uint32_t r[32];
                tc_ld32(lb + BC_DS + 32 * kq, r);
                tc_wait_ld();
                if (c > 0) {
                    pack_ds(r);
                    arrive(sready);
                    store_dstates(r, c - 1);
                } else if (p.dh0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) p.dh0[unit_off + (32 * kq + j) * DV + v] = __uint_as_float(r[j]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * st);  // exp(G_L) of this stage is consumed
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBcEpiWarps + 1) {
        tc_fence_after();
        tc_dealloc(tmem_alloc, BC_COLS);
    }
}

// ---------------------------------------------------------------------------------------------------------
// Chunk gradients: one CTA of 512 threads (16 warps) per (chunk, value head); fp32 values.  The value-column
// passes multiply fp16 operands (fp16 mma.sync for D, Vnew, dVnew and dv; tcgen05 with fp32 accumulators in TMEM
// for their accumulations); the pairwise terms, whose gate factors reach exp(+-8 |g|max), use TF32 MMAs.  The MMA phases (the value-column passes and the pairwise terms) give each warp a
// row block and a quarter of the columns; the gate scan and the solve's 16 x 16 steps run on threads 0-255 while
// the rest wait at the next barrier.  One CTA per SM: 16 warps hide more of the MMA chains' latency than 8.
constexpr int kBwThreads = 512, kBwCols = 16;  // value columns per pass over the state
constexpr int kRow = 132;                      // padded row stride (floats) of the [64][128] operand tiles
constexpr int kRowC = 68;                      // padded row stride of the [64][64] tiles
// Byte offset of element (r, c) of a pass tile, fp16 [rows][16 value columns]: 8 x 8 core matrices of 128 bytes
// (8 rows of 16 bytes), the two column halves of an 8-row group side by side.  This is the K-major operand layout
// without swizzle, with the 16 columns as K: leading byte offset 128 (between the halves), stride byte offset 256
// (between 8-row groups).  Reads of one column from 8 rows by 4 lanes each, and stores of 4-byte column pairs,
// fall into distinct banks.
__device__ __forceinline__ int tofs(int r, int c) { return (r >> 3) * 256 + (c >> 3) * 128 + (r & 7) * 16 + (c & 7) * 2; }
__device__ __forceinline__ uint64_t bwd_tile_desc(uint32_t saddr)
{
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128 >> 4) << 16) |
           (static_cast<uint64_t>(256 >> 4) << 32) | (1ull << 46);
}
__device__ __forceinline__ void bwd_prefetch_l2(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bwd_ldsm_x2_t(uint32_t addr, uint32_t &r0, uint32_t &r1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// 16 TMEM lanes (the address's lane onwards) x 8 (16) columns.  Thread (g, t) = (lane / 4, lane % 4) receives, for
// each block j of 8 columns, rows g and g + 8 at columns 8 j + 2 t and 8 j + 2 t + 1: the accumulator fragment of
// an m16n8 MMA, in the order (g, 2t), (g, 2t + 1), (g + 8, 2t), (g + 8, 2t + 1).
__device__ __forceinline__ void bwd_ld_frag2(uint32_t taddr, float (&d)[2][4])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    tc_wait_ld();
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i >> 2][i & 3] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void bwd_ld_frag4(uint32_t taddr, float (&d)[4][4])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    tc_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) d[i >> 2][i & 3] = __uint_as_float(r[i]);
}
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
    // pass tiles (inside WK), two buffers, each of fp16 tiles in the layout of tofs(): S[:, cols] and dS'[:, cols]
    // (128 rows), dO, D = v - Kb S, Vnew, dVnew and -dv (64 rows)
    static constexpr int P_S = 0, P_DS = 4096, P_O = 8192, P_D = 10240, P_N = 12288, P_DN = 14336, P_V = 16384;
    static constexpr int PBUF = 18432;
    static constexpr int WK_END = WK + 2 * PBUF;
    // the TMEM base address and two mbarriers, in the padding columns 64..67 of row 0 of P and of T (no phase reads
    // or writes a column of P or T past 63)
    static constexpr int TMEM_SLOT = PP + CH * 4;
    static constexpr int MBAR = TT + CH * 4;
    // phase-3 use of WK: the solve's products, 3 x [16][16] then [32][33]
    // phase-6 use of WK: dA, then Y = T^T dA diag(beta)
    static constexpr int DA = WK;                         // [64][kRowC]
    static constexpr int TOTAL = (WK_END > DA + CH * kRowC * 4 ? WK_END : DA + CH * kRowC * 4);
};
static_assert(BwSmem::TOTAL <= 232448, "shared memory");
static_assert((kRowC - CH) * 4 >= 16 && BwSmem::MBAR % 8 == 0 && BwSmem::TMEM_SLOT % 4 == 0,
              "the TMEM address and the two mbarriers need 16 bytes of row padding, 8-byte aligned");
static_assert(BwSmem::WK % 16 == 0 && BwSmem::PBUF % 16 == 0 && BwSmem::WK_END < (1 << 18),
              "pass tiles: 16-byte aligned, inside the descriptors' 18-bit address range");

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
    // TMEM (all 512 columns: the pass accumulators) and the two mbarriers of the pass MMAs
    if (tid == 0) {
        mbar_init(smem_u32(sm + S::MBAR), 1);
        mbar_init(smem_u32(sm + S::MBAR) + 8, 1);
        fence_mbar_init();
    }
    if (warp == 0) tc_alloc(smem_u32(sm + S::TMEM_SLOT), 512);
    tc_fence_before();
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
    // the passes' inputs (S, dS', and the rows of dO and v), pulled into L2 now: the passes read them 16 columns
    // at a time, and each pass's registers would otherwise wait on HBM
    if (tid == 0) {
        bwd_prefetch_l2(p.states + item * DK * DV, DK * DV * 2);
        bwd_prefetch_l2(p.dstates + item * DK * DV, DK * DV * 2);
    }
    if (tid < nvalid) {
        bwd_prefetch_l2(p.dout + ((row0 + tid) * p.HV + h) * DV, DV * 2);
        bwd_prefetch_l2(p.v + ((row0 + tid) * p.HV + h) * DV, DV * 2);
    }

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

    // ---- 2. P (j < i) and Aqk (j <= i) on TF32 MMAs (m16n8k8, fp32 accumulate).  Task t < 20 is the 16 x 8 tile
    //         n8 = t % 2 of block pair (I, J <= I), the pairs in the order (0,0), (1,0), (1,1), (2,0), ...; warp w
    //         takes task w, warps 0-3 also task 16 + w (one of them on each SMSP).  B = KB_J exp(m_I - m_J) (J < I) ----
    {
        for (int e = tid; e < CH * CH; e += kBwThreads) {  // T = I; P and Aqk above the diagonal blocks = 0
            const int i = e >> 6, j = e & (CH - 1);
            TT[i][j] = i == j ? 1.f : 0.f;
            if ((j >> 4) > (i >> 4)) {
                PP[i][j] = 0.f;
                AQ[i][j] = 0.f;
            }
        }
        auto task = [&](int t) {
            const int gq = lane >> 2, tq = lane & 3, n8 = t & 1;
            int pr = t >> 1, I = 0;
            while (pr > I) pr -= ++I;
            const int J = pr;
            const float *cf = J < I ? CF[cf_index(I, J)] : nullptr;
            const int ra = 16 * I + gq, rb = 16 * J + 8 * n8 + gq;
            float cp[4] = {}, cq[4] = {};
#pragma unroll 4
            for (int ks = 0; ks < DK; ks += 8) {
                const int k0 = ks + tq, k1 = k0 + 4;
                const uint32_t ap[4] = {to_tf32(KA[ra][k0]), to_tf32(KA[ra + 8][k0]), to_tf32(KA[ra][k1]),
                                        to_tf32(KA[ra + 8][k1])};
                const uint32_t aq[4] = {to_tf32(QA[ra][k0]), to_tf32(QA[ra + 8][k0]), to_tf32(QA[ra][k1]),
                                        to_tf32(QA[ra + 8][k1])};
                float b0 = KB[rb][k0], b1 = KB[rb][k1];
                if (cf) {
                    b0 = __fmul_rn(b0, cf[k0]);
                    b1 = __fmul_rn(b1, cf[k1]);
                }
                const uint32_t u0 = to_tf32(b0), u1 = to_tf32(b1);
                mma_tf32(cp, ap, u0, u1);
                mma_tf32(cq, aq, u0, u1);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = ra + 8 * (q >> 1), j = 16 * J + 8 * n8 + 2 * tq + (q & 1);
                PP[i][j] = j < i ? cp[q] : 0.f;
                AQ[i][j] = j <= i ? __fmul_rn(s, cq[q]) : 0.f;
            }
        };
        task(warp);
        if (warp < 4) task(16 + warp);
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

    // ---- 4-5. passes over 16 value columns at a time.  (a)-(d) on fp16 mma.sync (m16n8k16, fp32 accumulate); the
    //      accumulations of (e) on tcgen05: five kind::f16 MMAs per pass (M = 64 tokens, K = the pass's 16
    //      columns) add dQg, dKb, dKg (N = 128 keys) and dAqk, dA (N = 64 tokens) into TMEM.  An M = 64 accumulator
    //      keeps rows 16 I .. 16 I + 15 in lanes 32 I .. 32 I + 15, the lane quarter of warps I, I + 4, ..., so
    //      after the last pass each warp loads its phase-6/7 fragments from there.  S, dS' and dO of pass p + 1
    //      are read into registers during pass p and stored as fp16 tiles into the other buffer once the MMAs of
    //      pass p - 1, that buffer's last readers, have completed. ----
    tc_fence_after();
    const uint32_t tm = *reinterpret_cast<volatile uint32_t *>(sm + S::TMEM_SLOT);  // dQg 0, dKb 128, dKg 256,
    if (tm != 0 && tid == 0) atomicOr(p.err, ERR_TMEM_BASE);                        // dAqk 384, dA 448
    auto tile = [&](int b, int off) { return sm + S::WK + b * S::PBUF + off; };
    const __nv_bfloat16 *Sg = p.states + item * DK * DV;
    const __nv_bfloat16 *dSg = p.dstates + item * DK * DV;
    // MMA fragment ownership (g = lane / 4, t4 = lane % 4): warp (mt, nh), nh = 0..3, holds rows 16 mt + g and + 8,
    // and key columns 32 nh + 8 j + 2 t4 (+1), j = 0..3 (dQg, dKb, dKg), or token columns 16 nh + 8 j + 2 t4 (+1),
    // j = 0..1 (dAqk, dA).  In steps (a)-(d) of a pass, warp (mt, role, ntw) = (warp % 4, warp / 4 % 2, warp / 8)
    // computes rows 16 mt of the ntw-th 8-column tile of D and Vnew (role 0) or dVnew and dv (role 1).
    const int g = lane >> 2, t4 = lane & 3, mt = warp & 3, nh = warp >> 2;
    const int role = (warp >> 2) & 1, ntw = warp >> 3;
    const int r0 = 16 * mt + g, r1 = r0 + 8;
    // the A operand of step (a) (role 0: Kb = KA exp(m_I)) or (c) (role 1: Kg = KB exp(G_L - m_I)), rows 16 mt ..
    // and all 128 keys, as fp16 m16n8k16 fragments (|Kb|, |Kg| <= |kn| <= 1): built once, used by every pass
    uint32_t fa[8][4];
    {
        const float(*X)[kRow] = role ? KB : KA;
        const float *e = role ? EGLM[mt] : EM[mt];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = (q & 1) ? r1 : r0, k = 16 * kk + 2 * t4 + 8 * (q >> 1);
                const float2 x = *reinterpret_cast<const float2 *>(&X[r][k]);
                const float2 m = *reinterpret_cast<const float2 *>(&e[k]);
                fa[kk][q] = pack_f16(__fmul_rn(x.x, m.x), __fmul_rn(x.y, m.y));
            }
    }
    // the other pass-invariant A operands, per 16-token K step s: role 0: T diag(beta) (step (b), tokens 16 s, s <= mt);
    // role 1: Aqk^T (step (c), fb) and T^T (step (d), fc), tokens 16 (mt + s), s < 4 - mt
    uint32_t fb[4][4], fc[4][4];
#pragma unroll
    for (int st = 0; st < 4; ++st)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = (q & 1) ? r1 : r0;
            if (role == 0) {
                const int k = 16 * st + 2 * t4 + 8 * (q >> 1);
                const float2 t = *reinterpret_cast<const float2 *>(&TT[r][k]);
                const float2 bb = *reinterpret_cast<const float2 *>(&beta[k]);
                fb[st][q] = st <= mt ? pack_f16(__fmul_rn(t.x, bb.x), __fmul_rn(t.y, bb.y)) : 0u;
                fc[st][q] = 0u;
            } else {
                const int k = min(16 * (mt + st), 48) + 2 * t4 + 8 * (q >> 1);
                fb[st][q] = st < 4 - mt ? pack_f16(AQ[k][r], AQ[k + 1][r]) : 0u;
                fc[st][q] = st < 4 - mt ? pack_f16(TT[k][r], TT[k + 1][r]) : 0u;
            }
        }
    // staging: a thread takes one 16-byte row half (8 columns) of S (tid < 256) or dS' (tid >= 256) and, for
    // tid < 128, one of dO; 8 consecutive threads take 8 rows of one half, so a quarter-warp's stores fill 128
    // contiguous bytes
    const int su = tid & 255, s_half = (su >> 3) & 1, s_row = (su & 7) | ((su >> 4) << 3);
    const int o_half = (tid >> 3) & 1, o_row = (tid & 7) | ((tid >> 4) << 3);
    uint4 rs, ro = make_uint4(0u, 0u, 0u, 0u);
    uint32_t rv[2] = {0u, 0u}, rv_next[2] = {0u, 0u};  // v of rows r0, r1 (role 0), this pass and the next
    auto load_v = [&](int vb, uint32_t (&x)[2]) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int i = hf ? r1 : r0;
            x[hf] = 0u;
            if (role == 0 && i < nvalid)
                x[hf] = __ldg(reinterpret_cast<const unsigned int *>(p.v + ((row0 + i) * p.HV + h) * DV + vb + 8 * ntw + 2 * t4));
        }
    };
    auto load_pass = [&](int vb) {
        rs = __ldg(reinterpret_cast<const uint4 *>((tid < 256 ? Sg : dSg) + s_row * DV + vb + 8 * s_half));
        if (tid < 128) {
            ro = make_uint4(0u, 0u, 0u, 0u);
            if (o_row < nvalid)
                ro = __ldg(reinterpret_cast<const uint4 *>(p.dout + ((row0 + o_row) * p.HV + h) * DV + vb + 8 * o_half));
        }
    };
    auto to_f16x8 = [](uint4 x) {
        return make_uint4(pack_f16(bf16lo(x.x), bf16hi(x.x)), pack_f16(bf16lo(x.y), bf16hi(x.y)),
                          pack_f16(bf16lo(x.z), bf16hi(x.z)), pack_f16(bf16lo(x.w), bf16hi(x.w)));
    };
    auto store_pass = [&](int b) {
        *reinterpret_cast<uint4 *>(tile(b, tid < 256 ? S::P_S : S::P_DS) + tofs(s_row, 8 * s_half)) = to_f16x8(rs);
        if (tid < 128) *reinterpret_cast<uint4 *>(tile(b, S::P_O) + tofs(o_row, 8 * o_half)) = to_f16x8(ro);
    };
    const uint32_t mb0 = smem_u32(sm + S::MBAR);
    auto wait_mma = [&](int pass) {  // the MMAs of `pass` (and of every pass before it) have completed
        if (!mbar_wait(mb0 + 8 * (pass & 1), (pass >> 1) & 1)) atomicOr(p.err, ERR_PIPE_FULL_WAIT);
    };
    const uint32_t id128 = bwd_idesc(64, 128, false, false), id64 = bwd_idesc(64, 64, false, false);
    load_pass(0);
    store_pass(0);
    load_v(0, rv);
    float gl_acc = 0.f;  // thread d < 128: sum over all columns of S[d][.] dS'[d][.]
    for (int vb = 0, pass = 0; vb < DV; vb += kBwCols, ++pass) {
        const int buf = pass & 1;
        if (vb + kBwCols < DV) {
            load_pass(vb + kBwCols);
            load_v(vb + kBwCols, rv_next);
        }
        __syncthreads();  // this pass's S, dS' and dO tiles are stored
        if (tid < DK) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint4 x = *reinterpret_cast<const uint4 *>(tile(buf, S::P_S) + tofs(tid, 8 * hh));
                const uint4 y = *reinterpret_cast<const uint4 *>(tile(buf, S::P_DS) + tofs(tid, 8 * hh));
                const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 a = unpack_f16(xs[e]), b = unpack_f16(ys[e]);
                    gl_acc = __fmaf_rn(a.y, b.y, __fmaf_rn(a.x, b.x, gl_acc));
                }
            }
        }
        // steps (a)-(d): fp16 m16n8k16 MMAs; B fragments from the tiles by ldmatrix.trans (8 rows of 16 bytes per
        // matrix: thread (g, t4) receives rows 2 t4, 2 t4 + 1 of column g of this warp's 8 columns)
        const uint32_t tb = smem_u32(tile(buf, 0)) + 128 * ntw;
        if (role == 0) {
            // (a) D = v - Kb S for rows 16 mt .., columns 8 ntw ..
            float c[4] = {};
#pragma unroll
            for (int kk = 0; kk < 8; kk += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(tb + S::P_S + tofs(16 * kk + lane, 0), b0, b1, b2, b3);
                mma_f16(c, fa[kk], b0, b1);
                mma_f16(c, fa[kk + 1], b2, b3);
            }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int i = hf ? r1 : r0, cc = 8 * ntw + 2 * t4;
                const float2 vv = unpack_bf16(rv[hf]);
                *reinterpret_cast<uint32_t *>(tile(buf, S::P_D) + tofs(i, cc)) =
                    pack_f16(__fsub_rn(vv.x, c[2 * hf]), __fsub_rn(vv.y, c[2 * hf + 1]));
            }
        } else {
            // (c) dVnew = Kg dS' + Aqk^T dO for rows 16 mt .., columns 8 ntw ..
            float c[4] = {};
#pragma unroll
            for (int kk = 0; kk < 8; kk += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(tb + S::P_DS + tofs(16 * kk + lane, 0), b0, b1, b2, b3);
                mma_f16(c, fa[kk], b0, b1);
                mma_f16(c, fa[kk + 1], b2, b3);
            }
#pragma unroll
            for (int st = 0; st < 4; ++st)  // Aqk^T[i][j] = Aqk[j][i], nonzero for j >= i
                if (st < 4 - mt) {
                    uint32_t b0, b1;
                    bwd_ldsm_x2_t(tb + S::P_O + tofs(16 * (mt + st) + (lane & 15), 0), b0, b1);
                    mma_f16(c, fb[st], b0, b1);
                }
            *reinterpret_cast<uint32_t *>(tile(buf, S::P_DN) + tofs(r0, 8 * ntw + 2 * t4)) = pack_f16(c[0], c[1]);
            *reinterpret_cast<uint32_t *>(tile(buf, S::P_DN) + tofs(r1, 8 * ntw + 2 * t4)) = pack_f16(c[2], c[3]);
        }
        __syncthreads();
        if (role == 0) {
            // (b) Vnew = T diag(beta) D (T lower triangular: j < 16 (mt + 1))
            float c[4] = {};
#pragma unroll
            for (int st = 0; st < 4; ++st)
                if (st <= mt) {
                    uint32_t b0, b1;
                    bwd_ldsm_x2_t(tb + S::P_D + tofs(16 * st + (lane & 15), 0), b0, b1);
                    mma_f16(c, fb[st], b0, b1);
                }
            *reinterpret_cast<uint32_t *>(tile(buf, S::P_N) + tofs(r0, 8 * ntw + 2 * t4)) = pack_f16(c[0], c[1]);
            *reinterpret_cast<uint32_t *>(tile(buf, S::P_N) + tofs(r1, 8 * ntw + 2 * t4)) = pack_f16(c[2], c[3]);
        } else {
            // (d) dv = diag(beta) T^T dVnew (j >= i)
            float c[4] = {};
#pragma unroll
            for (int st = 0; st < 4; ++st)
                if (st < 4 - mt) {
                    uint32_t b0, b1;
                    bwd_ldsm_x2_t(tb + S::P_DN + tofs(16 * (mt + st) + (lane & 15), 0), b0, b1);
                    mma_f16(c, fc[st], b0, b1);
                }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int i = hf ? r1 : r0, cc = 8 * ntw + 2 * t4;
                const float x0 = __fmul_rn(beta[i], c[2 * hf]), x1 = __fmul_rn(beta[i], c[2 * hf + 1]);
                *reinterpret_cast<uint32_t *>(tile(buf, S::P_V) + tofs(i, cc)) = pack_f16(-x0, -x1);
                if (i < nvalid)
                    *reinterpret_cast<__nv_bfloat162 *>(p.dv + ((row0 + i) * p.HV + h) * DV + vb + cc) =
                        __floats2bfloat162_rn(x0, x1);
            }
        }
        fence_proxy_async();  // this thread's tile stores, visible to the tensor cores
        __syncthreads();      // the pass's seven tiles are complete
        if (warp == 0) {
            // (e) dQg += dO S^T, dKb += (-dv) S^T, dKg += Vnew dS'^T, dAqk += dO Vnew^T, dA += dVnew D^T
            tc_fence_after();
            const uint32_t t0 = smem_u32(tile(buf, 0)), acc = vb > 0;
            const uint64_t dS = bwd_tile_desc(t0 + S::P_S), dDS = bwd_tile_desc(t0 + S::P_DS),
                           dO = bwd_tile_desc(t0 + S::P_O), dD = bwd_tile_desc(t0 + S::P_D),
                           dN = bwd_tile_desc(t0 + S::P_N), dDN = bwd_tile_desc(t0 + S::P_DN),
                           dV = bwd_tile_desc(t0 + S::P_V);
            bwd_mma_ss_warp(tm + 0, dO, dS, id128, acc);
            bwd_mma_ss_warp(tm + 128, dV, dS, id128, acc);
            bwd_mma_ss_warp(tm + 256, dN, dDS, id128, acc);
            bwd_mma_ss_warp(tm + 384, dO, dN, id64, acc);
            bwd_mma_ss_warp(tm + 448, dDN, dD, id64, acc);
            tc_commit_warp(mb0 + 8 * buf);
        }
        if (vb + kBwCols < DV) {
            if (pass > 0) wait_mma(pass - 1);  // the other buffer's last readers are done
            store_pass(buf ^ 1);
            rv[0] = rv_next[0];
            rv[1] = rv_next[1];
        }
    }
    wait_mma(DV / kBwCols - 1);  // the last pass's MMAs, and with them every earlier one
    tc_fence_after();
    const uint32_t tl = tm + (static_cast<uint32_t>(32 * mt) << 16);  // this warp's lane quarter
    float aAq[2][4], aA[2][4];
    bwd_ld_frag2(tl + 384 + 16 * nh, aAq);
    bwd_ld_frag2(tl + 448 + 16 * nh, aA);

    if (tid < DK) dgl[tid] = __fmaf_rn(egl[tid], gl_acc, dgl[tid]);  // the exp(G_L) S dS' term of dG_L

    // the raw q/k pairs of the phase-7 elements (the element terms rebuild qn/kn from them; the normalisation's
    // Jacobian reads them at the end), requested here so that their latency hides behind phase 6
    uint32_t xq[2][4] = {}, xk[2][4] = {};
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
    // Y = T^T dA diag(beta), Y[a][e] = beta_e sum_{c >= a} T[c][a] dA[c][e], then dL = -Y T^T (a > b), both on TF32
    // MMAs (m16n8k8): warp (mt, nh) holds rows 16 mt + g (+ 8) of the 8-column tiles nb = nh and nh + 4.
    float y[2][4] = {};
    for (int ks = 16 * mt; ks < CH; ks += 8) {  // T[c][a] = 0 for c < a
        const uint32_t a[4] = {to_tf32(TT[ks + t4][r0]), to_tf32(TT[ks + t4][r1]), to_tf32(TT[ks + t4 + 4][r0]),
                               to_tf32(TT[ks + t4 + 4][r1])};
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int cn = 8 * (nh + 4 * jj) + g;
            mma_tf32(y[jj], a, to_tf32(DA[ks + t4][cn]), to_tf32(DA[ks + t4 + 4][cn]));
        }
    }
    __syncthreads();  // every read of dA is done
#pragma unroll
    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int col = 8 * (nh + 4 * jj) + 2 * t4 + (q & 1);
            DA[(q >> 1) ? r1 : r0][col] = __fmul_rn(beta[col], y[jj][q]);
        }
    __syncthreads();
    // dL[a][b] = -sum_{e <= b} Y[a][e] T[b][e] (a > b); dbeta_a += sum_b dL_ab P_ab; M = diag(beta) dL
    {
        float *rowp4 = reinterpret_cast<float *>(sm + S::DA + CH * kRowC * 4);  // [4 column quarters][64 rows]
        float dl[2][4] = {};
        const int kend = 8 * (nh + 4) + 8;  // tile nh + 4 needs e < kend, tile nh e < 8 nh + 8
        const bool live0 = 8 * nh < 16 * mt + 16, live1 = 8 * (nh + 4) < 16 * mt + 16;  // some a > b in the tile
        if (live0 || live1) {
            for (int ks = 0; ks < kend; ks += 8) {
                const uint32_t a[4] = {to_tf32(DA[r0][ks + t4]), to_tf32(DA[r1][ks + t4]), to_tf32(DA[r0][ks + t4 + 4]),
                                       to_tf32(DA[r1][ks + t4 + 4])};
                if (live0 && ks < 8 * nh + 8)
                    mma_tf32(dl[0], a, to_tf32(TT[8 * nh + g][ks + t4]), to_tf32(TT[8 * nh + g][ks + t4 + 4]));
                if (live1)
                    mma_tf32(dl[1], a, to_tf32(TT[8 * (nh + 4) + g][ks + t4]), to_tf32(TT[8 * (nh + 4) + g][ks + t4 + 4]));
            }
        }
        float rowp[2] = {};
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int a = (q >> 1) ? r1 : r0, b = 8 * (nh + 4 * jj) + 2 * t4 + (q & 1);
                float v = -dl[jj][q];
                if (b < a) rowp[q >> 1] = __fmaf_rn(v, PP[a][b], rowp[q >> 1]);
                else v = 0.f;
                dl[jj][q] = v;
            }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {  // the four lanes of a row, then (after the barrier) the four column quarters
            rowp[hf] = __fadd_rn(rowp[hf], __shfl_xor_sync(0xffffffffu, rowp[hf], 1));
            rowp[hf] = __fadd_rn(rowp[hf], __shfl_xor_sync(0xffffffffu, rowp[hf], 2));
        }
        if (t4 == 0) {
            rowp4[nh * CH + r0] = rowp[0];
            rowp4[nh * CH + r1] = rowp[1];
        }
        __syncthreads();  // every read of P and T is done (dbeta's column sums above included); quarters stored
        if (tid < CH)
            dbeta[tid] = __fadd_rn(dbeta[tid], __fadd_rn(__fadd_rn(rowp4[tid], rowp4[CH + tid]),
                                                         __fadd_rn(rowp4[2 * CH + tid], rowp4[3 * CH + tid])));
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int a = (q >> 1) ? r1 : r0, b = 8 * (nh + 4 * jj) + 2 * t4 + (q & 1);
                PP[a][b] = __fmul_rn(beta[a], dl[jj][q]);
            }
    }
    __syncthreads();
    float(*MM)[kRowC] = PP;
    float(*NN)[kRowC] = AQ;

    // ---- 7. element terms and pairwise terms, in the fragment ownership of phase 5 ----
    float aQ[4][4], aB[4][4], aG[4][4];
    bwd_ld_frag4(tl + 0 + 32 * nh, aQ);
    bwd_ld_frag4(tl + 128 + 32 * nh, aB);
    bwd_ld_frag4(tl + 256 + 32 * nh, aG);
    tc_fence_before();  // every TMEM read of this thread is done (TMEM is freed after the next barrier)
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
                const uint32_t wq = xq[hf][j], wk = xk[hf][j];
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
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tm, 512);
    }
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
