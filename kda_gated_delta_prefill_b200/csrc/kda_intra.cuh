// kda_intra.cuh -- intra-chunk kernel: everything of the chunk construction
// that does not depend on the carried state, for one (chunk, value head)
// item per CTA, fully parallel over items, with its contractions on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
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
// Gate references.  exp(G_i - G_j) is split into a row factor and a column
// factor that the tensor core multiplies over d.  The chunk is cut into two
// 32-token halves; inside half h the reference is the midpoint
// m_h = (G at the half's start + G at its end) / 2, so both factors stay
// within exp(+-|half's gate sum| / 2); across the halves (rows of the second,
// columns of the first) the reference is G_31 and both factors are <= 1.
// With per-channel half sums >= -170 every factor the method needs stays a
// normal bf16 number (per-token g >= -5 suffices).  All exponents are formed
// in base 2: G2 = log2(e) G, factors 2^(G2 - m).
//
// A CTA (256 threads, two per SM) is persistent: it takes items from a
// counter and, for each, runs
//   1. Rows past the end of the sequence are zeroed (the page's zero padding
//      of a partial chunk); q, k (Q/K head h / (HV/H)) and v arrived by TMA
//      tile loads issued during the previous item, g and beta by plain loads
//      into registers.
//   2. L2 normalisation of q and k in place (l2norm_half_row, the routine of
//      the standalone kda_l2norm_bf16 kernel).
//   3. Gate sums and the operands: A1 = [k exp(G - m); K^-0.5 q exp(G - m)]
//      (128 rows), B1 = k exp(m - G) (64 rows), A2 = the second half's k and q
//      rows against G_31, B2 = the first half's k rows against G_31 (bf16),
//      exp(G) k (fp16, W's operand), Qg and Kg (fp16, to the item block).
//   4. MMA1 on tcgen05: D1 = A1 B1^T (128 x 64), D2 = A2 B2^T (128 x 32).  Once
//      it completes, the next item's q/k tiles are requested into A1's place
//      and its g values into registers.  Epilogue: L (beta-scaled, strictly
//      lower) transposed into shared memory, Aqk (causal) to the item block.
//   5. A: exact float32 forward substitution for the two diagonal 32 x 32
//      blocks (one warp each, lane = column) while the other warps store Aqk,
//      then the lower-left block -X_1 (L_10 X_0) on tf32 mma.sync, scaled by
//      beta into fp16 A.
//   6. MMA2 on tcgen05: W = A (exp(G) k) (M = 128 with 64 rows used) and
//      U^T = v^T A^T; once it completes the next item's v tile is requested,
//      and -W and U^T go from the accumulators straight to the item block.
// One warp polls each tensor-core completion while the others wait at a
// hardware barrier.  Every wait is bounded; a wait that gives up sets the
// device error word and the CTA finishes its steps on whatever shared memory
// holds.
#pragma once
#include "kda_common.cuh"
#include "kda_norm.cuh"
#include "ptx.cuh"
#include "tc.cuh"

namespace kda {

struct IntraSmem {
    static constexpr int A1 = 0;          // bf16 [2 K-halves, 16384 apart][128 rows][128 B]: rows 0-63 k, 64-127 q
    static constexpr int V = 32768;       // [2 value halves][64 tok][128 B]: v bf16, then fp16 in place
    static constexpr int B1 = 49152;      // bf16 [2 K-halves, 8192 apart][64 tok][128 B]
    static constexpr int A2 = 65536;      // bf16 [2 K-halves, 8192 apart][64 rows][128 B]: k (rows 0-31), q (32-63)
    static constexpr int B2 = 81920;      // bf16 [2 K-halves, 4096 apart][32 tok][128 B]
    static constexpr int KEXP = 90112;    // fp16 [2 K-halves, 8192 apart][64 tok][128 B]: exp(G) k
    // once MMA1 has completed (B1's second K-half, A2 and B2 are free; A1 takes the next item's q and k)
    static constexpr int ASOL = B1;       // fp16 [64 i][64 j] SW128: A = (I + L)^-1 diag(beta)
    static constexpr int LD0 = 57344;     // fp32 [32 j][32]: column j of L_00, row i at (i % 4) * 8 + i / 4
    static constexpr int LD1 = 61440;     // fp32 [32 j][32]: column j of L_11, the same order
    static constexpr int L10T = 65536;    // fp32 [32 k][40]: L_10 transposed
    static constexpr int X0 = 70656;      // fp32 [32][40]: (I + L_00)^-1
    static constexpr int X1 = 75776;      // fp32 [32][36]: (I + L_11)^-1
    static constexpr int Y = 80384;       // fp32 [32][40]: L_10 X_0
    // once MMA2 has completed: the images of -W and U^T, stored by two bulk copies (read before the next
    // item writes B1 and A2 again)
    static constexpr int WST = B1;
    static constexpr int UST = A2;
    static constexpr int BETA = 106496;   // fp32 [64]
    static constexpr int OT = 106752;     // fp32 [8 octets][128 channels]: gate sums of 8-token octets (base 2)
    static constexpr int BAR = 110848;    // mbarriers: q/k tiles, v tile, MMA1, MMA2
    static constexpr int TSLOT = BAR + 32;   // tensor-memory base address
    static constexpr int NEXT = TSLOT + 4;   // the next item this CTA takes
    static constexpr int TOTAL = NEXT + 12;
};
static_assert(IntraSmem::Y + 32 * 40 * 4 <= IntraSmem::KEXP, "solve scratch overlaps exp(G) k");
static_assert(IntraSmem::LD0 == IntraSmem::B1 + 8192, "the solve scratch starts after A");
static_assert(IntraSmem::UST + 16384 <= IntraSmem::KEXP, "the U^T image overlaps exp(G) k");

struct IntraParams {
    const float *g;            // [rows][HV][128]
    const float *beta;
    const int32_t *cu;         // [N+1] or null
    const int32_t *chunk_off;  // [N+1] chunk offsets of the packed sequences, or null
    uint8_t *items;            // [num_chunks][HV] item blocks
    unsigned *err;
    int B, T, H, HV, N;
    int chunks_per_seq;        // ceil(T/64) when cu is null
    int chunk_begin;           // cu null: this launch covers chunks [chunk_begin, chunk_begin + chunk_count)
    int chunk_count;           //   of every sequence (cu given: all chunks, chunk_begin = 0)
    int *counter;              // persistent launch: items taken so far beyond the first gridDim.x (zero before
                               //   the launch); null: one item per CTA
    int n_items;               // (chunk, value head) items of this launch
    int prefetch_stride;       // one item per CTA: CTAs resident at once (the item whose inputs to pull into L2)
};

constexpr int kIntraCtasPerSm = 2;           // the shared-memory footprint lets two CTAs share an SM
constexpr uint32_t kIntraTmemCols = 256;     // D1 + D2 (96 columns), later W (128) + U^T (64)

__device__ __forceinline__ void intra_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }

__device__ __forceinline__ float4 f4add(float4 a, float4 b)
{
    const float2 lo = add2(make_float2(a.x, a.y), make_float2(b.x, b.y));
    const float2 hi = add2(make_float2(a.z, a.w), make_float2(b.z, b.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// 16-byte chunk c of row r in a 128-byte-swizzled tile of 128-byte rows
__device__ __forceinline__ uint32_t sw_chunk(int r, int c) { return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4)); }

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

    // ---- item -> (item chunk index, value head, row of the chunk start, valid rows); false past the end ----
    const int nchunks = p.cu ? p.chunk_off[p.N] : p.B * p.chunk_count;
    struct Item {
        int ci, h, hq, nvalid;
        int64_t row0;
    };
    auto locate = [&](int item, Item &it) {
        if (item >= p.n_items) return false;
        const int local = item / p.HV;
        if (local >= nchunks) return false;
        it.h = item % p.HV;
        it.hq = it.h / (p.HV / p.H);
        if (p.cu) {
            it.ci = local;
            int lo = 0, hi = p.N - 1;  // last n with chunk_off[n] <= ci
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (p.chunk_off[mid] <= local) lo = mid; else hi = mid - 1;
            }
            const int c = local - p.chunk_off[lo];
            const int len = p.cu[lo + 1] - p.cu[lo];
            it.row0 = p.cu[lo] + static_cast<int64_t>(c) * CH;
            it.nvalid = min(CH, len - c * CH);
        } else {
            const int b = local / p.chunk_count, c = p.chunk_begin + local % p.chunk_count;
            it.ci = b * p.chunks_per_seq + c;
            it.row0 = static_cast<int64_t>(b) * p.T + static_cast<int64_t>(c) * CH;
            it.nvalid = min(CH, p.T - c * CH);
        }
        return true;
    };
    // this thread's gate values: tokens 8*warp .. 8*warp+7, channels 4*lane .. 4*lane+3 (zero past the valid
    // rows), and the item's beta (threads 0-63)
    auto load_g = [&](const Item &it, float4 (&gv)[8], float &bt) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = 8 * warp + u;
            gv[u] = i < it.nvalid
                        ? __ldg(reinterpret_cast<const float4 *>(p.g + ((it.row0 + i) * p.HV + it.h) * DK) + lane)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        bt = (tid < it.nvalid) ? __ldg(p.beta + (it.row0 + tid) * p.HV + it.h) : 0.f;
    };
    const uint32_t bar_qk = sb + S::BAR, bar_v = bar_qk + 8, bar_m1 = bar_qk + 16, bar_m2 = bar_qk + 24;
    auto load_qk = [&](const Item &it) {  // thread 0
        mbar_expect_tx(bar_qk, 32768);
        const int z = static_cast<int>(it.row0);
        tma_load_3d(sb + S::A1, &tk, 0, it.hq, z, bar_qk);           // k, channels 0-63: rows 0-63 of K-half 0
        tma_load_3d(sb + S::A1 + 16384, &tk, 64, it.hq, z, bar_qk);  // k, channels 64-127: rows 0-63 of K-half 1
        tma_load_3d(sb + S::A1 + 8192, &tq, 0, it.hq, z, bar_qk);    // q: rows 64-127
        tma_load_3d(sb + S::A1 + 24576, &tq, 64, it.hq, z, bar_qk);
    };
    auto load_v = [&](const Item &it) {  // thread 0
        mbar_expect_tx(bar_v, 16384);
        const int z = static_cast<int>(it.row0);
        tma_load_3d(sb + S::V, &tv, 0, it.h, z, bar_v);
        tma_load_3d(sb + S::V + 8192, &tv, 64, it.h, z, bar_v);
    };
    auto prefetch = [&](const Item &it) {  // thread 0: the item's inputs into L2
        const int z = static_cast<int>(it.row0);
        tma_prefetch_3d(&tq, 0, it.hq, z);
        tma_prefetch_3d(&tq, 64, it.hq, z);
        tma_prefetch_3d(&tk, 0, it.hq, z);
        tma_prefetch_3d(&tk, 64, it.hq, z);
        tma_prefetch_3d(&tv, 0, it.h, z);
        tma_prefetch_3d(&tv, 64, it.h, z);
        tma_prefetch_3d(&tg, 0, it.h, z);
    };

    Item cur;
    if (!locate(blockIdx.x, cur)) return;
    if (tid == 0) {
        mbar_init(bar_qk, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_m1, 1);
        mbar_init(bar_m2, 1);
        fence_mbar_init();
        load_qk(cur);
        load_v(cur);
    }
    if (warp == 0) tc_alloc(sb + S::TSLOT, kIntraTmemCols);
    float4 gv[8];
    float bt;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + S::TSLOT);
    float *sbeta = reinterpret_cast<float *>(sm + S::BETA);
    volatile int *snext = reinterpret_cast<volatile int *>(sm + S::NEXT);

    for (int iter = 0;; ++iter) {
        const uint32_t par = iter & 1;
        uint8_t *out = p.items + (static_cast<int64_t>(cur.ci) * p.HV + cur.h) * ITEM_BYTES;  // item block (global)
        // this item's gate values and beta into registers (used after the normalisation); the next item: in a
        // persistent launch claimed now and published (its inputs pulled into L2) after the normalisation, so
        // that the atomic's latency is off the path; otherwise none
        load_g(cur, gv, bt);
        int claim = p.n_items;
        if (tid == 0 && p.counter) claim = static_cast<int>(gridDim.x) + atomicAdd(p.counter, 1);
        if (!mbar_wait(bar_qk, par)) atomicOr(p.err, ERR_TMA_WAIT);
        if (cur.nvalid < CH) {  // zero the rows past the sequence's end (another sequence's or batch row's tokens)
            for (int idx = tid; idx < (CH - cur.nvalid) * 32; idx += 256) {
                const int r = cur.nvalid + idx / 32, w = idx % 32;  // 16-byte words of the row: k and q, two K-halves
                const int isq = w >> 4, kh = (w >> 3) & 1, c = w & 7;
                *reinterpret_cast<uint4 *>(sm + S::A1 + kh * 16384 + (64 * isq + r) * 128 + c * 16) =
                    make_uint4(0, 0, 0, 0);
            }
        }
        intra_sync();

        // ---- 2. normalise k (rows 0-63) and q (rows 64-127): thread = row half, the partner lane holds the rest ----
        {
            const int r = tid >> 1, kh = tid & 1;
            uint8_t *row = sm + S::A1 + kh * 16384 + r * 128;
            uint4 raw[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) raw[c] = *reinterpret_cast<const uint4 *>(row + ((c ^ (r & 7)) << 4));
            l2norm_half_row(raw);  // the routine the standalone kda_l2norm_bf16 kernel runs
#pragma unroll
            for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(row + ((c ^ (r & 7)) << 4)) = raw[c];
        }

        // ---- 3. gate sums (base 2) and the operands: warp = token octet, lane = channel quad ----
        {
            const float2 l2e = make_float2(1.4426950408889634f, 1.4426950408889634f);
            float4 *ot = reinterpret_cast<float4 *>(sm + S::OT);
            {
                float2 lo = make_float2(0.f, 0.f), hi = lo;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    lo = add2(lo, mul2(make_float2(gv[u].x, gv[u].y), l2e));
                    hi = add2(hi, mul2(make_float2(gv[u].z, gv[u].w), l2e));
                }
                ot[warp * 32 + lane] = make_float4(lo.x, lo.y, hi.x, hi.y);
            }
            if (tid == 0) {
                *snext = claim;
                Item ni;
                // the item a later CTA (or this one next) takes: its inputs into L2
                if (locate(p.counter ? claim : static_cast<int>(blockIdx.x) + p.prefetch_stride, ni)) prefetch(ni);
                bulk_wait_read();  // the previous item's -W and U^T images (over B1 and A2) have been read
            }
            if (tid < CH) sbeta[tid] = bt;
            intra_sync();  // also: every row is normalised
            float4 before = make_float4(0.f, 0.f, 0.f, 0.f), g31 = before, g63 = before;
#pragma unroll
            for (int o = 0; o < 8; ++o) {
                const float4 t = ot[o * 32 + lane];
                if (o < warp) before = f4add(before, t);
                if (o < 4) g31 = f4add(g31, t);
                g63 = f4add(g63, t);
            }
            const int half = warp >> 2;
            // reference of this half: m0 = G31 / 2, m1 = (G31 + G63) / 2
            const float4 m = half == 0 ? make_float4(0.5f * g31.x, 0.5f * g31.y, 0.5f * g31.z, 0.5f * g31.w)
                                       : make_float4(0.5f * (g31.x + g63.x), 0.5f * (g31.y + g63.y),
                                                     0.5f * (g31.z + g63.z), 0.5f * (g31.w + g63.w));
            // per-channel factors: 2^m (exp(G) = f 2^m), 2^(G63 - m) (exp(G_last - G) = fi 2^(G63 - m)), and the
            // change to the reference G31: 2^(G31 / 2) for the first half's key rows (G31 - m0), 2^((G63 - G31) / 2)
            // for the second half's rows (m1 - G31)
            const float4 eM = make_float4(ex2(m.x), ex2(m.y), ex2(m.z), ex2(m.w));
            const float4 eL = make_float4(ex2(g63.x - m.x), ex2(g63.y - m.y), ex2(g63.z - m.z), ex2(g63.w - m.w));
            const float4 cx = half == 0 ? make_float4(ex2(0.5f * g31.x), ex2(0.5f * g31.y), ex2(0.5f * g31.z),
                                                      ex2(0.5f * g31.w))
                                        : make_float4(ex2(0.5f * (g63.x - g31.x)), ex2(0.5f * (g63.y - g31.y)),
                                                      ex2(0.5f * (g63.z - g31.z)), ex2(0.5f * (g63.w - g31.w)));
            if (warp == 0)
                *reinterpret_cast<float4 *>(out + ITEM_GL + 16 * lane) =
                    make_float4(ex2(g63.x), ex2(g63.y), ex2(g63.z), ex2(g63.w));
            // K^-0.5 = 128^-0.5 in float32 is applied to Qg here and to Aqk in its epilogue
            const float sc = 0.08838834764831845f;
            const float2 eM01 = make_float2(eM.x, eM.y), eM23 = make_float2(eM.z, eM.w);
            const float2 eQ01 = make_float2(eM.x * sc, eM.y * sc), eQ23 = make_float2(eM.z * sc, eM.w * sc);
            const float2 eL01 = make_float2(eL.x, eL.y), eL23 = make_float2(eL.z, eL.w);
            const float2 cx01 = make_float2(cx.x, cx.y), cx23 = make_float2(cx.z, cx.w);
            const float2 mlo = make_float2(m.x, m.y), mhi = make_float2(m.z, m.w);
            const int kh = lane >> 4, cq = (lane & 15) >> 1, sub = (lane & 1) * 8;  // K-half, 16-byte chunk, offset
            float2 Glo = make_float2(before.x, before.y), Ghi = make_float2(before.z, before.w);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = 8 * warp + u;  // token; i % 8 == u
                Glo = add2(Glo, mul2(make_float2(gv[u].x, gv[u].y), l2e));  // inclusive cumulative gate (base 2)
                Ghi = add2(Ghi, mul2(make_float2(gv[u].z, gv[u].w), l2e));
                const float2 x01 = make_float2(Glo.x - mlo.x, Glo.y - mlo.y), x23 = make_float2(Ghi.x - mhi.x, Ghi.y - mhi.y);
                const float2 f01 = make_float2(ex2_ftz(x01.x), ex2_ftz(x01.y)), f23 = make_float2(ex2_ftz(x23.x), ex2_ftz(x23.y));
                const float2 fi01 = make_float2(ex2_ftz(-x01.x), ex2_ftz(-x01.y));
                const float2 fi23 = make_float2(ex2_ftz(-x23.x), ex2_ftz(-x23.y));
                const uint32_t o1 = kh * 16384 + ((cq ^ u) << 4) + sub;  // in A1 (row offset added below)
                const uint32_t o2 = kh * 8192 + ((cq ^ u) << 4) + sub;   // in the [2][rows][128 B] tiles
                const uint2 kr = *reinterpret_cast<const uint2 *>(sm + S::A1 + i * 128 + o1);
                const uint2 qr = *reinterpret_cast<const uint2 *>(sm + S::A1 + (64 + i) * 128 + o1);
                const float2 k01 = unpack_bf16(kr.x), k23 = unpack_bf16(kr.y);
                const float2 q01 = unpack_bf16(qr.x), q23 = unpack_bf16(qr.y);
                const float2 ak01 = mul2(k01, f01), ak23 = mul2(k23, f23);
                const float2 aq01 = mul2(q01, f01), aq23 = mul2(q23, f23);
                const float2 bk01 = mul2(k01, fi01), bk23 = mul2(k23, fi23);
                *reinterpret_cast<uint2 *>(sm + S::A1 + i * 128 + o1) =
                    make_uint2(pack_bf16(ak01.x, ak01.y), pack_bf16(ak23.x, ak23.y));
                *reinterpret_cast<uint2 *>(sm + S::A1 + (64 + i) * 128 + o1) =
                    make_uint2(pack_bf16(aq01.x, aq01.y), pack_bf16(aq23.x, aq23.y));
                *reinterpret_cast<uint2 *>(sm + S::B1 + i * 128 + o2) =
                    make_uint2(pack_bf16(bk01.x, bk01.y), pack_bf16(bk23.x, bk23.y));
                const float2 ke01 = mul2(ak01, eM01), ke23 = mul2(ak23, eM23);
                *reinterpret_cast<uint2 *>(sm + S::KEXP + i * 128 + o2) =
                    make_uint2(pack_f16(ke01.x, ke01.y), pack_f16(ke23.x, ke23.y));
                const float2 qg01 = mul2(aq01, eQ01), qg23 = mul2(aq23, eQ23);
                *reinterpret_cast<uint2 *>(out + ITEM_QG + i * 128 + o2) =
                    make_uint2(pack_f16(qg01.x, qg01.y), pack_f16(qg23.x, qg23.y));
                const float2 kg01 = mul2(bk01, eL01), kg23 = mul2(bk23, eL23);
                *reinterpret_cast<uint2 *>(out + ITEM_KG + i * 128 + o2) =
                    make_uint2(pack_f16(kg01.x, kg01.y), pack_f16(kg23.x, kg23.y));
                if (half == 0) {  // B2 row i: k exp(G31 - G)
                    const float2 b01 = mul2(bk01, cx01), b23 = mul2(bk23, cx23);
                    *reinterpret_cast<uint2 *>(sm + S::B2 + kh * 4096 + i * 128 + ((cq ^ u) << 4) + sub) =
                        make_uint2(pack_bf16(b01.x, b01.y), pack_bf16(b23.x, b23.y));
                } else {          // A2 rows i - 32 (k) and i (q): exp(G - G31)
                    const float2 a01 = mul2(ak01, cx01), a23 = mul2(ak23, cx23);
                    const float2 c01 = mul2(aq01, cx01), c23 = mul2(aq23, cx23);
                    *reinterpret_cast<uint2 *>(sm + S::A2 + (i - 32) * 128 + o2) =
                        make_uint2(pack_bf16(a01.x, a01.y), pack_bf16(a23.x, a23.y));
                    *reinterpret_cast<uint2 *>(sm + S::A2 + i * 128 + o2) =
                        make_uint2(pack_bf16(c01.x, c01.y), pack_bf16(c23.x, c23.y));
                }
            }
        }
        fence_proxy_async();  // the operands are read by the tensor core (async proxy)
        tc_fence_before();
        intra_sync();

        // ---- 4. MMA1: D1 = A1 B1^T (TMEM columns 0-63), D2 = A2 B2^T (columns 64-95) ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t i1 = idesc_kind_f16(128, 64, true, false, false);
            const uint32_t i2 = idesc_kind_f16(128, 32, true, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kb = (ks & 3) * 32;
                tc_mma_ss(tmem, sw128_desc(sb + S::A1 + (ks >> 2) * 16384 + kb, 16, 1024),
                          sw128_desc(sb + S::B1 + (ks >> 2) * 8192 + kb, 16, 1024), i1, ks > 0);
            }
            // A2 spans 128 rows of which 64 are used: its rows 64-127 read the next 8 KB (the other K-half, or B2)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kb = (ks & 3) * 32;
                tc_mma_ss(tmem + 64, sw128_desc(sb + S::A2 + (ks >> 2) * 8192 + kb, 16, 1024),
                          sw128_desc(sb + S::B2 + (ks >> 2) * 4096 + kb, 16, 1024), i2, ks > 0);
            }
            tc_commit(bar_m1);
        }
        // v (its copy overlapped the steps above): zero the padding rows, bf16 -> fp16 in place
        if (!mbar_wait(bar_v, par)) atomicOr(p.err, ERR_TMA_WAIT);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int idx = tid + 256 * k;  // 16-byte chunk: half (idx >> 9), row ((idx >> 3) & 63)
            uint4 *pv = reinterpret_cast<uint4 *>(sm + S::V) + idx;
            const uint4 uu = *pv;
            uint32_t w[4] = {uu.x, uu.y, uu.z, uu.w};
            const bool pad = ((idx >> 3) & 63) >= cur.nvalid;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 xv = unpack_bf16(w[j]);
                w[j] = pad ? 0u : pack_f16(xv.x, xv.y);
            }
            *pv = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (warp == 0 && !mbar_wait_spin(bar_m1, par) && lane == 0) atomicOr(p.err, ERR_PIPE_FULL_WAIT);
        intra_sync();
        tc_fence_after();
        // A1 is free: the next item's q and k tiles
        Item nxt;
        const bool more = locate(*snext, nxt);
        if (more && tid == 0) load_qk(nxt);

        // ---- 4b. MMA1 epilogue: warp = TMEM lane quarter (warp & 3) x role ----
        {
            float *LD0 = reinterpret_cast<float *>(sm + S::LD0);
            float *LD1 = reinterpret_cast<float *>(sm + S::LD1);
            float *L10T = reinterpret_cast<float *>(sm + S::L10T);
            const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
            const int perm = (lane & 3) * 8 + (lane >> 2);  // where row `lane` of a diagonal block sits in LD
            uint32_t r[32];
            // Aqk row i (times K^-0.5), 16-byte chunks c0 .. c0+3 from 32 accumulator columns; j <= jmax kept
            auto aqk_row = [&](int i, int c0, int jmax) {
                const float sc = 0.08838834764831845f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 8 * c + 2 * e;
                        w[e] = pack_f16(j <= jmax ? sc * __uint_as_float(r[j]) : 0.f,
                                        j + 1 <= jmax ? sc * __uint_as_float(r[j + 1]) : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(out + ITEM_AQK + sw_chunk(i, c0 + c)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            };
            switch (warp) {
            case 0: {  // L_00, rows i = lane (D1 lanes 0-31, columns 0-31)
                tc_ld32(tl, r);
                tc_wait_ld();
                const float bi = sbeta[lane];
#pragma unroll
                for (int j = 0; j < 32; ++j) LD0[j * 32 + perm] = j < lane ? bi * __uint_as_float(r[j]) : 0.f;
                break;
            }
            case 1: {  // L_11, rows 32 + lane (D1 lanes 32-63, columns 32-63)
                tc_ld32(tl + 32, r);
                tc_wait_ld();
                const float bi = sbeta[32 + lane];
#pragma unroll
                for (int j = 0; j < 32; ++j) LD1[j * 32 + perm] = j < lane ? bi * __uint_as_float(r[j]) : 0.f;
                break;
            }
            case 4: {  // L_10, rows 32 + lane (D2 lanes 0-31): every column j < 32 is below the diagonal
                tc_ld32(tl + 64, r);
                tc_wait_ld();
                const float bi = sbeta[32 + lane];
#pragma unroll
                for (int j = 0; j < 32; ++j) L10T[j * 40 + lane] = bi * __uint_as_float(r[j]);
                break;
            }
            case 5:  // Aqk_10: rows 32 + lane (D2 lanes 32-63), columns 0-31
                tc_ld32(tl + 64, r);
                tc_wait_ld();
                aqk_row(32 + lane, 0, 31);
                break;
            case 2:  // Aqk_00: rows lane (D1 lanes 64-95), columns 0-31, causal
                tc_ld32(tl, r);
                tc_wait_ld();
                aqk_row(lane, 0, lane);
                break;
            case 3:  // Aqk_11: rows 32 + lane (D1 lanes 96-127), columns 32-63, causal
                tc_ld32(tl + 32, r);
                tc_wait_ld();
                aqk_row(32 + lane, 4, lane);
                break;
            case 6:  // Aqk rows 0-31, columns 32-63: above the diagonal
#pragma unroll
                for (int c = 4; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(out + ITEM_AQK + sw_chunk(lane, c)) = make_uint4(0, 0, 0, 0);
                break;
            default:  // A rows 0-31, columns 32-63: above the diagonal
#pragma unroll
                for (int c = 4; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(sm + S::ASOL + sw_chunk(lane, c)) = make_uint4(0, 0, 0, 0);
                break;
            }
        }
        tc_fence_before();
        intra_sync();

        // ---- 5. A = (I + L)^-1 diag(beta) ----
        {  // diagonal blocks: exact float32 substitution on all 256 threads.  Thread = (block, column c, row group
           // r4 holding rows r4, r4 + 4, ..., r4 + 28); the four threads of a column are adjacent lanes.
           // Right-looking: row j, once final, is broadcast to its column's lanes and updates every later row,
           // each row taking its terms in the order j = 0, 1, ...; L's zeros above the diagonal make the
           // updates of earlier rows no-ops.
            const int blk = warp >> 2, c = (warp & 3) * 8 + (lane >> 2), r4 = lane & 3;
            const float *LD = reinterpret_cast<const float *>(sm + (blk ? S::LD1 : S::LD0));
            float x[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) x[q] = 4 * q + r4 == c ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < 31; ++j) {
                const float xj = __shfl_sync(0xffffffffu, x[j >> 2], (lane & ~3) | (j & 3));
                const float4 *col = reinterpret_cast<const float4 *>(LD + j * 32 + r4 * 8);  // L[4q + r4][j], q = 0..7
                float l[8];
                if (j < 16) {
                    const float4 lo = col[0];
                    l[0] = lo.x; l[1] = lo.y; l[2] = lo.z; l[3] = lo.w;
                }
                const float4 hi = col[1];
                l[4] = hi.x; l[5] = hi.y; l[6] = hi.z; l[7] = hi.w;
#pragma unroll
                for (int q = j >> 2; q < 8; ++q)
                    if (j < 16 || q >= 4) x[q] = __fmaf_rn(-l[q], xj, x[q]);
            }
            float *Xs = reinterpret_cast<float *>(sm + (blk ? S::X1 : S::X0));
            const int xs = blk ? 36 : 40, o = 32 * blk;
            const float bc = sbeta[o + c];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int i = 4 * q + r4;
                Xs[i * xs + c] = x[q];
                *reinterpret_cast<__half *>(sm + S::ASOL + sw_chunk(o + i, (o + c) >> 3) + ((o + c) & 7) * 2) =
                    __float2half_rn(x[q] * bc);
            }
        }
        intra_sync();
        {  // Y = L_10 X_0 (tf32, warp = 16 x 8 tile)
            const int mt = warp >> 2, nt = warp & 3;
            const float *L10T = reinterpret_cast<const float *>(sm + S::L10T);
            const float *X0 = reinterpret_cast<const float *>(sm + S::X0);
            float d[4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int kb = 8 * ks, m0 = 16 * mt + g8;  // L_10[m][k] = L10T[k][m]
                uint32_t a[4];
                a[0] = to_tf32(L10T[(kb + t4) * 40 + m0]);
                a[1] = to_tf32(L10T[(kb + t4) * 40 + m0 + 8]);
                a[2] = to_tf32(L10T[(kb + t4 + 4) * 40 + m0]);
                a[3] = to_tf32(L10T[(kb + t4 + 4) * 40 + m0 + 8]);
                mma_tf32(d, a, to_tf32(X0[(kb + t4) * 40 + 8 * nt + g8]), to_tf32(X0[(kb + t4 + 4) * 40 + 8 * nt + g8]));
            }
            float *Yf = reinterpret_cast<float *>(sm + S::Y);
            *reinterpret_cast<float2 *>(Yf + (16 * mt + g8) * 40 + 8 * nt + 2 * t4) = make_float2(d[0], d[1]);
            *reinterpret_cast<float2 *>(Yf + (16 * mt + g8 + 8) * 40 + 8 * nt + 2 * t4) = make_float2(d[2], d[3]);
        }
        intra_sync();
        {  // A_10 = -(X_1 Y) diag(beta_0..31) (tf32; X_1 rows 0-15 are zero beyond column 15)
            const int mt = warp >> 2, nt = warp & 3;
            const float *X1 = reinterpret_cast<const float *>(sm + S::X1);
            const float *Yf = reinterpret_cast<const float *>(sm + S::Y);
            float d[4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                if (mt == 0 && ks >= 2) continue;
                const int kb = 8 * ks, m0 = 16 * mt + g8;
                uint32_t a[4];
                a[0] = to_tf32(X1[m0 * 36 + kb + t4]);
                a[1] = to_tf32(X1[(m0 + 8) * 36 + kb + t4]);
                a[2] = to_tf32(X1[m0 * 36 + kb + t4 + 4]);
                a[3] = to_tf32(X1[(m0 + 8) * 36 + kb + t4 + 4]);
                mma_tf32(d, a, to_tf32(Yf[(kb + t4) * 40 + 8 * nt + g8]), to_tf32(Yf[(kb + t4 + 4) * 40 + 8 * nt + g8]));
            }
            const int cc = 8 * nt + 2 * t4, r0 = 32 + 16 * mt + g8;
            const float b0 = sbeta[cc], b1 = sbeta[cc + 1];
            *reinterpret_cast<uint32_t *>(sm + S::ASOL + sw_chunk(r0, cc >> 3) + (cc & 7) * 2) =
                pack_f16(-d[0] * b0, -d[1] * b1);
            *reinterpret_cast<uint32_t *>(sm + S::ASOL + sw_chunk(r0 + 8, cc >> 3) + (cc & 7) * 2) =
                pack_f16(-d[2] * b0, -d[3] * b1);
        }
        fence_proxy_async();  // A and the fp16 v are read by the tensor core
        intra_sync();

        // ---- 6. MMA2: W = A (exp(G) k) into columns 0-127 (rows 0-63 used), U^T = v^T A^T into 128-191 ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t iw = idesc_kind_f16(128, 128, false, false, true);  // A K-major, exp(G) k MN-major
            const uint32_t iu = idesc_kind_f16(128, 64, false, true, false);   // v^T MN-major, A^T K-major
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)  // A's rows 64-127 read the next 8 KB of shared memory (unused rows)
                tc_mma_ss(tmem, sw128_desc(sb + S::ASOL + ks * 32, 16, 1024),
                          sw128_desc(sb + S::KEXP + ks * 2048, 8192, 1024), iw, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc_mma_ss(tmem + 128, sw128_desc(sb + S::V + ks * 2048, 8192, 1024),
                          sw128_desc(sb + S::ASOL + ks * 32, 16, 1024), iu, ks > 0);
            tc_commit(bar_m2);
        }
        if (warp == 0 && !mbar_wait_spin(bar_m2, par) && lane == 0) atomicOr(p.err, ERR_PIPE_FULL_WAIT);
        intra_sync();
        tc_fence_after();
        if (more && tid == 0) load_v(nxt);  // v's place is free
        {  // epilogue: -W (lanes 0-63 = tokens) and U^T (lanes = value rows) into their item images
            const int qd = warp & 3, ch = warp >> 2;
            const uint32_t tl = tmem + (static_cast<uint32_t>(32 * qd) << 16);
            uint32_t r[32];
            if (qd < 2) {  // -W row i, keys 64 ch .. 64 ch + 63 (K-half ch of the item's [64 tok][128 key] tile)
                const int i = 32 * qd + lane;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    tc_ld32(tl + 64 * ch + 32 * hh, r);
                    tc_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = pack_f16(-__uint_as_float(r[8 * c4 + 2 * e]), -__uint_as_float(r[8 * c4 + 2 * e + 1]));
                        *reinterpret_cast<uint4 *>(sm + S::WST + ch * 8192 + sw_chunk(i, 4 * hh + c4)) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            {  // U^T row vv, tokens 32 ch .. 32 ch + 31
                const int vv = 32 * qd + lane;
                tc_ld32(tl + 128 + 32 * ch, r);
                tc_wait_ld();
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = pack_f16(__uint_as_float(r[8 * c4 + 2 * e]), __uint_as_float(r[8 * c4 + 2 * e + 1]));
                    *reinterpret_cast<uint4 *>(sm + S::UST + sw_chunk(vv, 4 * ch + c4)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        fence_proxy_async();  // the images are read by the bulk copies
        tc_fence_before();
        intra_sync();  // every TMEM read is done before the next MMA1 writes
        if (tid == 0) {
            bulk_store(out + ITEM_WN, sb + S::WST, 16384);
            bulk_store(out + ITEM_U, sb + S::UST, 16384);
            bulk_commit();
        }
        if (!more) break;
        cur = nxt;
    }
    if (tid == 0) bulk_wait_read();  // shared memory must outlive the last images' reads
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tmem, kIntraTmemCols);
    }
}

}  // namespace kda
