// kda_carry.cuh -- inter-chunk state carry on the 5th-generation tensor cores
// ("KDA Chunk Prefill on Ascend A3", section "Mathematical definition", last
// three formulas), written transposed so that the value dimension (128) is
// the MMA's M dimension:
//   Vnew^T = U^T - S_in^T W^T
//   O^T    = S_in^T Qg^T + Vnew^T Aqk^T
//   S_out^T = S_in^T diag(exp(G_last)) + Vnew^T Kg
// One CTA per (sequence, value head).  Warps 0-15 (epilogue) own TMEM lane
// v = 32*(warp%4) + lane, i.e. value column v, and a quarter of the key and
// token columns (warp/4); they keep the float32 master state S^T[v][:] in registers and
// write its fp16 copy into TMEM, where it is the A operand of the next
// chunk's MMAs.  Warp 16 streams the per-chunk blocks written by the
// intra-chunk kernel into a three-stage shared-memory ring (one bulk copy per
// chunk); the last warp allocates TMEM and issues the MMAs.  Every wait is
// bounded.
#pragma once
#include <type_traits>

#include "kda_common.cuh"
#include "ptx.cuh"
#include "tc.cuh"

namespace kda {

struct CarrySmem {
    static constexpr int STAGE = ((ITEM_BYTES + 1023) / 1024) * 1024;  // 75776
    // Three stages (222 KB): a chunk block is requested two chunk periods before it is needed, which covers
    // the copy latency while the intra-chunk kernel loads HBM on the other SMs.
    static constexpr int NST = 3;
    static constexpr int BAR = NST * STAGE;   // mbarriers: full[NST] empty[NST] barP barS sready vready barO
    static constexpr int TMEM_SLOT = BAR + (2 * NST + 5) * 8;
    static constexpr int ABORT = TMEM_SLOT + 4;
    static constexpr int TOTAL = ABORT + 12;
};

constexpr int kCarryEpiWarps = 16;  // 4 or 8 or 16: warps per TMEM lane quarter x 4
static_assert(kCarryEpiWarps == 4 || kCarryEpiWarps == 8 || kCarryEpiWarps == 16, "epilogue warps");
constexpr int kCarryThreads = (kCarryEpiWarps + 2) * 32;

// TMEM column map (512 allocated): P^T (64), O^T x2 (64 each), S^T fp32 master (128), S^T fp16 (64), Vnew^T fp16 (32).
constexpr uint32_t TM_P = 0, TM_O0 = 64, TM_S = 192, TA_S = 320, TA_V = 384, TM_COLS = 512;

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
    int chunk_begin;           // this launch carries chunks [chunk_begin, chunk_begin + chunk_count) of every
    int chunk_count;           //   sequence, from s0 (cu given: clipped to the sequence's own chunks)
    // Segmented carry of plain batches (seg_phase != 0): the chunks of every sequence are split into seg_count
    // segments [nck*p/seg_count, nck*(p+1)/seg_count), unit = (sequence, value head) = blockIdx % units.
    //  seg_phase 1, j = blockIdx / units: j = 0 carries segment 0 from s0 and stores its end state, which is the
    //    start of segment 1, in seg_S[unit][1]; j = 2p-1 carries segment p from zero into seg_B[unit][p]; j = 2p
    //    carries segment p from the identity with U taken as zero (the segment's linear map) into seg_M[unit][p].
    //    No o is written.
    //    CTA j = 0 also copies the initial state (s0, or zeros) into seg_S[unit][0].
    //  seg_phase 2, p = blockIdx / units: segment p from seg_S[unit][p], writing o; the last segment writes sN
    //    (which may be the buffer s0 points to).
    int seg_phase;
    int seg_count;
    float *seg_S, *seg_M, *seg_B;  // [units][seg_count][K][V]
    // When set (not in the segment-map pass), the state at the start of every chunk is also stored, bf16
    // [K][V] (nearest even) at states + (global chunk * HV + h) * K * V (the item's index), for the backward.
    __nv_bfloat16 *states;
    int no_o;                      // unsegmented launches: skip o (the O products and stores)
    int h_begin, h_count;          // plain batches, optional: only value heads [h_begin, h_begin + h_count)
};

// kDump: the backward's instantiation, which also stores every chunk's start state (p.states)
template <bool kDump>
__global__ void __launch_bounds__(kCarryThreads, 1) kda_carry_kernel(const CarryParams p)
{
    using S = CarrySmem;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // A launch that the host made a programmatic dependent of this one (the next chunk window's intra-chunk
    // work, which reads nothing this kernel writes) may start once every CTA of this grid is resident.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int nh = p.h_count ? p.h_count : p.HV;  // value heads this launch covers, from h_begin
    int h = p.h_begin + static_cast<int>(blockIdx.x % nh);
    int n = p.order ? p.order[blockIdx.x / nh] : blockIdx.x / nh;
    int64_t c_begin, tok0;
    int nck, len;
    // where the state starts and ends, and what the chunk loop produces
    enum { FROM_S0, FROM_ZERO, FROM_IDENTITY };
    int from = FROM_S0;
    const float *s_in = p.s0 ? p.s0 + (static_cast<int64_t>(n) * p.HV + h) * DK * DV : nullptr;
    float *s_out = p.sN + (static_cast<int64_t>(n) * p.HV + h) * DK * DV;
    float *s_copy = nullptr;  // where the initial state is also stored (segmented first pass only)
    bool with_o = true, homogeneous = false;
    if (p.seg_phase != 0) {
        const int units = p.N * p.HV, unit = blockIdx.x % units, j = blockIdx.x / units;
        n = unit / p.HV;
        h = unit % p.HV;
        const int seg = p.seg_phase == 1 ? (j + 1) / 2 : j;
        const int cb = static_cast<int>(static_cast<int64_t>(p.chunks_per_seq) * seg / p.seg_count);
        const int ce = static_cast<int>(static_cast<int64_t>(p.chunks_per_seq) * (seg + 1) / p.seg_count);
        c_begin = static_cast<int64_t>(n) * p.chunks_per_seq + cb;
        nck = ce - cb;
        tok0 = static_cast<int64_t>(n) * p.T + static_cast<int64_t>(cb) * CH;
        len = p.T - cb * CH;
        const int64_t slot = (static_cast<int64_t>(unit) * p.seg_count + seg) * DK * DV;
        s_in = p.s0 ? p.s0 + (static_cast<int64_t>(n) * p.HV + h) * DK * DV : nullptr;
        if (p.seg_phase == 1) {
            with_o = false;
            if (j == 0) {  // also keeps a copy of the initial state for the second pass (final_state may alias it)
                s_copy = p.seg_S + slot;
                s_out = p.seg_S + (static_cast<int64_t>(unit) * p.seg_count + 1) * DK * DV;
            } else if (j & 1) {
                from = FROM_ZERO;
                s_out = p.seg_B + slot;
            } else {
                from = FROM_IDENTITY;
                homogeneous = true;
                s_out = p.seg_M + slot;
            }
        } else {
            s_in = p.seg_S + slot;
            s_out = seg + 1 == p.seg_count ? p.sN + (static_cast<int64_t>(n) * p.HV + h) * DK * DV : nullptr;
        }
    } else if (p.cu) {
        with_o = !p.no_o;
        const int all = p.chunk_off[n + 1] - p.chunk_off[n], a = min(p.chunk_begin, all);
        c_begin = p.chunk_off[n] + a;
        nck = min(all - a, p.chunk_count);
        tok0 = p.cu[n] + static_cast<int64_t>(a) * CH;
        len = p.cu[n + 1] - p.cu[n] - a * CH;
        // A window past this sequence's end, with the state carried in place: nothing to do.
        if (nck == 0 && s_in == s_out) return;
    } else {
        with_o = !p.no_o;
        c_begin = static_cast<int64_t>(n) * p.chunks_per_seq + p.chunk_begin;
        nck = p.chunk_count;
        tok0 = static_cast<int64_t>(n) * p.T + static_cast<int64_t>(p.chunk_begin) * CH;
        len = p.T - p.chunk_begin * CH;
    }

    const uint32_t full0 = sb + S::BAR, empty0 = full0 + 8 * S::NST, barP = full0 + 16 * S::NST, barS = barP + 8,
                   sready = barP + 16, vready = barP + 24, barO = barP + 32;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S::ABORT);
    if (tid == 0) {
        for (int s = 0; s < S::NST; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1 + kCarryEpiWarps);
        }
        mbar_init(barP, 1);
        mbar_init(barS, 1);
        mbar_init(barO, 1);
        mbar_init(sready, kCarryEpiWarps);
        mbar_init(vready, kCarryEpiWarps);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kCarryEpiWarps + 1) tc_alloc(sb + S::TMEM_SLOT, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The CTA allocates all 512 columns, so the allocation can only start at lane 0, column 0: every TMEM
    // address below is a compile-time constant (fewer instructions per MMA issue and per tcgen05.ld/st).
    const uint32_t tmem_alloc = *reinterpret_cast<volatile uint32_t *>(sm + S::TMEM_SLOT);
    constexpr uint32_t tmem = 0;

    auto fail = [&](unsigned code) {
        atomicOr(p.err, code);
        *abort_flag = 1;
    };
    if (tmem_alloc != 0) {
        if (tid == 0) fail(ERR_TMEM_BASE);
        nck = 0;
    }

    if (warp == kCarryEpiWarps) {
        // ---------------- producer: one bulk copy per chunk block ----------------
        if (lane == 0) {
            for (int c = 0; c < nck && !*abort_flag; ++c) {
                const int s = c % S::NST;
                if (c >= S::NST && !mbar_wait(empty0 + 8 * s, ((c / S::NST) - 1) & 1)) {
                    fail(ERR_PIPE_EMPTY_WAIT);
                    break;
                }
                mbar_expect_tx(full0 + 8 * s, ITEM_BYTES);
                bulk_load(sb + s * S::STAGE, p.items + ((c_begin + c) * p.HV + h) * ITEM_BYTES, ITEM_BYTES,
                          full0 + 8 * s);
            }
        }
    } else if (warp == kCarryEpiWarps + 1) {
        // ---------------- MMA issuer: the whole warp walks the chunks, one elected lane issues ----------------
        // The body is instantiated once per ring stage, so every descriptor is a constant offset from the
        // shared-memory base.
        // Descriptor = high word (strides, swizzle) : low word (start address >> 4, leading offset).  Start
        // addresses stay below 2^18 bytes, so offsets only ever touch the low word.
        const uint32_t i64 = idesc_f16(128, 64, false), i128mn = idesc_f16(128, 128, true);
        const uint64_t dk0 = sw128_desc(sb, 16, 1024), kk0 = sw128_desc(sb, 8192, 1024);
        const uint32_t dhi = static_cast<uint32_t>(dk0 >> 32), khi = static_cast<uint32_t>(kk0 >> 32);
        auto chunk = [&](int c, auto stage) -> bool {
            constexpr int st = decltype(stage)::value;
            constexpr uint32_t so = static_cast<uint32_t>(st * (S::STAGE >> 4));
            // opaque per chunk, so the compiler forms each descriptor next to its MMA instead of keeping
            // all of them live across the loop
            uint32_t dlo = static_cast<uint32_t>(dk0), klo = static_cast<uint32_t>(kk0);
            asm volatile("" : "+r"(dlo), "+r"(klo));
            auto dbase = [&](uint32_t off) { return (static_cast<uint64_t>(dhi) << 32) | (dlo + off); };
            auto kbase = [&](uint32_t off) { return (static_cast<uint64_t>(khi) << 32) | (klo + off); };
            const bool ok = mbar_wait(full0 + 8 * st, (c / S::NST) & 1) && mbar_wait_spin(sready, c & 1);
            if (!__all_sync(0xffffffffu, ok)) return false;
            tc_fence_after();
            const uint32_t tmo = tmem + TM_O0 + 64 * (c & 1);
            // P^T = S^T W^T (K = 128 keys, 8 steps); W is stored negated, so P^T = -(S^T W^T)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                tc_mma_ts_warp(tmem + TM_P, tmem + TA_S + 8 * ks,
                               dbase(so + (ITEM_WN >> 4) + (ks >> 2) * 512 + (ks & 3) * 2), i64, ks > 0);
            tc_commit_warp(barP);
            // O^T = S^T Qg^T
            if (with_o) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma_ts_warp(tmo, tmem + TA_S + 8 * ks,
                                   dbase(so + (ITEM_QG >> 4) + (ks >> 2) * 512 + (ks & 3) * 2), i64, ks > 0);
            }
            if (!__all_sync(0xffffffffu, mbar_wait_spin(vready, c & 1))) return false;
            tc_fence_after();
            // S^T += Vnew^T Kg onto the decayed master state (on the chain to the next chunk, so first).
            // Kg is MN-major: 64-key blocks 8192 bytes apart, token groups of 8 rows 1024 bytes apart.
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc_mma_ts_warp(tmem + TM_S, tmem + TA_V + 8 * ks, kbase(so + (ITEM_KG >> 4) + ks * 128), i128mn, 1);
            tc_commit_warp(barS);
            // O^T += Vnew^T Aqk^T (K = 64 tokens)
            if (with_o) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc_mma_ts_warp(tmo, tmem + TA_V + 8 * ks, dbase(so + (ITEM_AQK >> 4) + ks * 2), i64, 1);
                tc_commit_warp(barO);
            }
            tc_commit_warp(empty0 + 8 * st);
            return true;
        };
        static_assert(S::NST == 3, "the issuer body is instantiated for three stages");
        for (int c = 0; c < nck; ++c) {
            if (__any_sync(0xffffffffu, *abort_flag)) break;
            const int st = c % S::NST;
            const bool ok = st == 0   ? chunk(c, std::integral_constant<int, 0>{})
                            : st == 1 ? chunk(c, std::integral_constant<int, 1>{})
                                      : chunk(c, std::integral_constant<int, 2>{});
            if (!ok) {
                if (lane == 0) fail(ERR_PIPE_FULL_WAIT);
                break;
            }
        }
    } else {
        // ---------------- epilogue: value column v, key/token quarter kq ----------------
        // Sub-block kq (0..3) = key columns 32kq..32kq+31 of the state and token columns 16kq..16kq+15; a warp
        // owns kSub consecutive sub-blocks of its lane quarter.
        constexpr int kSub = 16 / kCarryEpiWarps;
        const int qd = warp & 3, kq0 = (warp >> 2) * kSub;
        const int v = 32 * qd + lane;
        const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
        auto tS = [&](int kq) { return tmem + lane_base + TM_S + 32 * kq; };  // fp32 master S^T[v][32kq .. 32kq+31]
        auto tA = [&](int kq) { return tmem + lane_base + TA_S + 16 * kq; };  // its fp16 copy (A operand)
        const int64_t ostride = static_cast<int64_t>(p.HV) * DV;
        // S^T[v][32kq ..] (32 master-state values) -> fp16 A operand of the next chunk's MMAs.
        auto pack_state = [&](const uint32_t (&r)[32], int kq) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    w[j] = pack_f16(__uint_as_float(r[16 * hf + 2 * j]), __uint_as_float(r[16 * hf + 2 * j + 1]));
                tc_st8(tA(kq) + 8 * hf, w);
            }
        };
        auto arrive = [&](uint32_t bar) {
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        // the state at the start of chunk c (S^T[v][32kq + j] in r) -> states, rows kd = 32kq + j, column v
        __nv_bfloat16 *dump = kDump && p.seg_phase != 1 ? p.states : nullptr;
        auto dump_state = [&](const uint32_t (&r)[32], int kq, int c) {
            __nv_bfloat16 *dst = dump + ((c_begin + c) * p.HV + h) * DK * DV + v;
#pragma unroll
            for (int j = 0; j < 32; ++j) dst[(32 * kq + j) * DV] = __float2bfloat16_rn(__uint_as_float(r[j]));
        };
        bool alive = tmem_alloc == 0;
        if (alive) {
            const float *s0 = from == FROM_S0 ? s_in : nullptr;
#pragma unroll
            for (int i = 0; i < kSub; ++i) {
                const int kq = kq0 + i;
                uint32_t r[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    r[j] = __float_as_uint(s0 ? s0[(32 * kq + j) * DV + v]
                                              : (from == FROM_IDENTITY && 32 * kq + j == v ? 1.f : 0.f));
                if (s_copy) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) s_copy[(32 * kq + j) * DV + v] = __uint_as_float(r[j]);
                }
                tc_st32(tS(kq), r);
                pack_state(r, kq);
                if (kDump && dump && nck > 0) dump_state(r, kq, 0);
            }
            arrive(sready);
        }
        // o rows of chunk c: O^T[v][tok], tok in [16*kq, 16*kq+16); a warp writes 64 contiguous bytes per token
        auto store_o = [&](int c) {
#pragma unroll
            for (int i = 0; i < kSub; ++i) {
                const int kq = kq0 + i;
                uint32_t orr[16];
                tc_ld16(tmem + lane_base + TM_O0 + 64 * (c & 1) + 16 * kq, orr);
                tc_wait_ld();
                __nv_bfloat16 *ob = p.o + ((tok0 + static_cast<int64_t>(c) * CH + 16 * kq) * p.HV + h) * DV + v;
                const int nrows = min(CH, len - c * CH) - 16 * kq;
                if (nrows >= 16) {
#pragma unroll
                    for (int t = 0; t < 16; ++t) ob[t * ostride] = __float2bfloat16_rn(__uint_as_float(orr[t]));
                } else {
#pragma unroll
                    for (int t = 0; t < 16; ++t)
                        if (t < nrows) ob[t * ostride] = __float2bfloat16_rn(__uint_as_float(orr[t]));
                }
            }
        };

        for (int c = 0; c < nck && alive && !*abort_flag; ++c) {
            const int s = c % S::NST;
            const uint8_t *st = sm + s * S::STAGE;
            // --- while MMA1/O1 of chunk c run: S^T <- S^T diag(exp(G_last)) ---
            if (!mbar_wait(full0 + 8 * s, (c / S::NST) & 1)) {
                fail(ERR_PIPE_FULL_WAIT);
                break;
            }
#pragma unroll
            for (int i = 0; i < kSub; ++i) {
                const int kq = kq0 + i;
                const float2 *gl = reinterpret_cast<const float2 *>(st + ITEM_GL) + 16 * kq;
                uint32_t r[32];
                tc_ld32(tS(kq), r);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float2 x = mul2(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), gl[j]);
                    r[2 * j] = __float_as_uint(x.x);
                    r[2 * j + 1] = __float_as_uint(x.y);
                }
                tc_st32(tS(kq), r);
            }
            // --- Vnew^T[v][tok] = U^T[v][tok] + P^T[v][tok], tok in [16*kq, 16*kq+16) ---
            if (!mbar_wait_spin(barP, c & 1)) {
                fail(ERR_PIPE_FULL_WAIT);
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int i = 0; i < kSub; ++i) {
                const int kq = kq0 + i;
                uint32_t pr[16];
                tc_ld16(tmem + lane_base + TM_P + 16 * kq, pr);
                uint4 ur[2];
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    ur[q] = *reinterpret_cast<const uint4 *>(st + ITEM_U + v * 128 + (((2 * kq + q) ^ (v & 7)) << 4));
                tc_wait_ld();
                uint32_t w[8];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint32_t uw[4] = {ur[q].x, ur[q].y, ur[q].z, ur[q].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = 8 * q + 2 * e;
                        const float2 pv = make_float2(__uint_as_float(pr[t]), __uint_as_float(pr[t + 1]));
                        const float2 x = homogeneous ? pv : add2(unpack_f16(uw[e]), pv);
                        w[4 * q + e] = pack_f16(x.x, x.y);
                    }
                }
                tc_st8(tmem + lane_base + TA_V + 8 * kq, w);
            }
            // O of the previous chunk must be observed complete BEFORE this warp arrives on vready: after the
            // arrival, the issuer may finish chunk c's O as well, and a parity wait on barO would then see
            // the barrier two phases on and never return.  (O2 of chunk c-1 ran ahead of MMA1 of chunk c,
            // so this wait normally passes at once.)
            if (with_o && c > 0 && !mbar_wait_spin(barO, (c - 1) & 1)) {
                fail(ERR_PIPE_FULL_WAIT);
                break;
            }
            arrive(vready);  // the wait also covers the decayed master state
            if (lane == 0) mbar_arrive(empty0 + 8 * s);  // U and exp(G_last) of this stage are consumed
            if (with_o && c > 0) {  // the previous chunk's o rows, while MMA2 runs
                tc_fence_after();
                store_o(c - 1);
            }
            // --- S^T (master, now S_out^T) -> fp16 A operand for the next chunk ---
            if (!mbar_wait_spin(barS, c & 1)) {
                fail(ERR_PIPE_FULL_WAIT);
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int i = 0; i < kSub; ++i) {
                const int kq = kq0 + i;
                uint32_t r[32];
                tc_ld32(tS(kq), r);
                tc_wait_ld();
                pack_state(r, kq);
                if (kDump && dump && c + 1 < nck) dump_state(r, kq, c + 1);
            }
            arrive(sready);
        }
        if (with_o && nck > 0 && !*abort_flag) {
            if (mbar_wait(barO, (nck - 1) & 1)) {
                tc_fence_after();
                store_o(nck - 1);
            } else {
                fail(ERR_PIPE_FULL_WAIT);
            }
        }
        // final state (S^T[v][kd] -> final_state[kd][v]); skipped when the TMEM allocation was unusable
        if (tmem_alloc == 0 && s_out) {
            float *sN = s_out;
#pragma unroll
            for (int i = 0; i < kSub; ++i) {
                const int kq = kq0 + i;
                uint32_t r[32];
                tc_ld32(tS(kq), r);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) sN[(32 * kq + j) * DV + v] = __uint_as_float(r[j]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kCarryEpiWarps + 1) {
        tc_fence_after();
        tc_dealloc(tmem_alloc, TM_COLS);
    }
}

}  // namespace kda
