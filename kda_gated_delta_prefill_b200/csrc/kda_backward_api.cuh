// kda_backward_api.cuh -- host side of the backward (included at the end of kda_prefill.cu, whose argument
// checks, workspace helpers, tensor-map encoding and carry launch it uses).
#pragma once

namespace {

// Backward workspace (also the buffer a forward saves for the backward): the forward's own workspace (chunk
// offsets and order for packed batches, the per-chunk blocks, segment scratch), then the chunk start states and
// the gradients at the chunk end states (bf16), the final state of a recomputed forward, and the per-value-head
// gradients at the normalised q/k rows.
struct BwdWorkspace {
    size_t chunk_off = 0, items = 0, fwd_total = 0, states = 0, dstates = 0, final_state = 0, dqn = 0, dkn = 0,
           total = 0;
    int64_t max_chunks = 0;
};

BwdWorkspace bwd_workspace_layout(int B, int T, int HV, int num_seqs)
{
    BwdWorkspace w;
    const bool varlen = num_seqs > 0;
    const int64_t N = varlen ? num_seqs : B;
    const Workspace f = workspace_layout(B, T, HV, num_seqs);
    w.max_chunks = f.max_chunks;
    w.chunk_off = f.chunk_off;
    w.items = f.items;
    w.fwd_total = f.total;
    const size_t rows = static_cast<size_t>(B) * T, state = static_cast<size_t>(DK) * DV * sizeof(float);
    const size_t state16 = static_cast<size_t>(DK) * DV * 2;  // the per-chunk states and gradients are bf16
    size_t off = round_up(f.total, kAlign);
    w.states = off;
    off = round_up(off + static_cast<size_t>(w.max_chunks) * HV * state16, kAlign);
    w.dstates = off;
    off = round_up(off + static_cast<size_t>(w.max_chunks) * HV * state16, kAlign);
    w.final_state = off;
    off = round_up(off + static_cast<size_t>(N) * HV * state, kAlign);
    w.dqn = off;
    off = round_up(off + rows * HV * DK * sizeof(float), kAlign);
    w.dkn = off;
    off = round_up(off + rows * HV * DK * sizeof(float), kAlign);
    w.total = off;
    return w;
}

kda_status_t backward_impl(const void *q, const void *k, const void *v, const float *g, const float *beta,
                           const float *initial_state, const int32_t *cu_seqlens, int num_seqs, int B, int T, int H,
                           int HV, int K, int V, const void *dout, const float *dht, void *dq, void *dk, void *dv,
                           float *dg, float *dbeta, float *dh0, void *workspace, size_t workspace_bytes, void *stream,
                           bool recompute);

}  // namespace

extern "C" size_t kda_prefill_backward_workspace_size(int B, int T, int H, int HV, int K, int V, int num_seqs)
{
    Dims d;
    if (check_dims(B, T, H, HV, K, V, num_seqs > 0, num_seqs, d) != KDA_OK) return 0;
    return bwd_workspace_layout(B, T, HV, num_seqs > 0 ? num_seqs : 0).total;
}

extern "C" int kda_prefill_backward_kernel_launches(int B, int T, int H, int HV, int K, int V, int num_seqs)
{
    Dims d;
    const bool varlen = num_seqs > 0;
    if (check_dims(B, T, H, HV, K, V, varlen, num_seqs, d) != KDA_OK) return 0;
    const int with_tokens = static_cast<int64_t>(B) * T > 0 ? 1 : 0;
    // the forward's cut into parts (it depends on the SM count only for sequences long enough to be cut)
    int parts = 1;
    if (!varlen && with_tokens && (T + CH - 1) / CH / kMinChunksPerPart >= 2) {
        DeviceInfo info;
        if (device_info(info) != cudaSuccess) return 0;
        parts = pipeline_parts(B, T, HV, false, info.sms);
    }
    // chunk offsets (packed), intra-chunk and carry with the start states per part, reverse carry, chunk
    // gradients, and the Q/K normalisation's Jacobian (inside the chunk kernel when H == HV)
    return (varlen ? 1 : 0) + (with_tokens + 1) * parts + 1 + with_tokens * (H == HV ? 1 : 2);
}

extern "C" kda_status_t kda_prefill_backward(const void *q, const void *k, const void *v, const float *g,
                                             const float *beta, const float *initial_state,
                                             const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int HV,
                                             int K, int V, const void *dout, const float *dht, void *dq, void *dk,
                                             void *dv, float *dg, float *dbeta, float *dh0, void *workspace,
                                             size_t workspace_bytes, void *stream)
{
    return backward_impl(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, B, T, H, HV, K, V, dout, dht, dq, dk,
                         dv, dg, dbeta, dh0, workspace, workspace_bytes, stream, true);
}

extern "C" kda_status_t kda_prefill_backward_saved(const void *q, const void *k, const void *v, const float *g,
                                                   const float *beta, const float *initial_state,
                                                   const int32_t *cu_seqlens, int num_seqs, int B, int T, int H,
                                                   int HV, int K, int V, const void *dout, const float *dht, void *dq,
                                                   void *dk, void *dv, float *dg, float *dbeta, float *dh0,
                                                   void *saved, size_t saved_bytes, void *stream)
{
    return backward_impl(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, B, T, H, HV, K, V, dout, dht, dq, dk,
                         dv, dg, dbeta, dh0, saved, saved_bytes, stream, false);
}

extern "C" kda_status_t kda_prefill_forward_save(const void *q, const void *k, const void *v, const float *g,
                                                 const float *beta, const float *initial_state,
                                                 const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int HV,
                                                 int K, int V, void *o, float *final_state, void *saved,
                                                 size_t saved_bytes, void *stream)
{
    Dims d;
    const bool varlen = cu_seqlens != nullptr;
    kda_status_t st = check_dims(B, T, H, HV, K, V, varlen, num_seqs, d);
    if (st != KDA_OK) return st;
    const BwdWorkspace ws = bwd_workspace_layout(B, T, HV, varlen ? num_seqs : 0);
    if (!saved || saved_bytes < ws.total) return KDA_ERR_WORKSPACE;
    if (!aligned(saved, kAlign)) return KDA_ERR_MISALIGNED;
    const int64_t tokens = static_cast<int64_t>(B) * T;
    const size_t nq = static_cast<size_t>(tokens) * H * K * 2, nvb = static_cast<size_t>(tokens) * HV * V * 2;
    const size_t ng = static_cast<size_t>(tokens) * HV * K * 4, nb = static_cast<size_t>(tokens) * HV * 4;
    const size_t ns = static_cast<size_t>(d.N) * HV * K * V * 4;
    const void *ext[] = {q, k, v, g, beta, initial_state, cu_seqlens, o, final_state};
    const size_t ext_n[] = {nq, nq, nvb, ng, nb, initial_state ? ns : 0,
                            varlen ? static_cast<size_t>(num_seqs + 1) * 4 : 0, nvb, ns};
    for (int i = 0; i < 9; ++i)
        if (overlaps(saved, ws.total, ext[i], ext_n[i])) return KDA_ERR_INVALID_ARG;
    uint8_t *sb = static_cast<uint8_t *>(saved);
    return forward_impl(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, B, T, H, HV, K, V, o, final_state, sb,
                        ws.fwd_total, stream, reinterpret_cast<__nv_bfloat16 *>(sb + ws.states));
}

namespace {
kda_status_t backward_impl(const void *q, const void *k, const void *v, const float *g, const float *beta,
                           const float *initial_state, const int32_t *cu_seqlens, int num_seqs, int B, int T, int H,
                           int HV, int K, int V, const void *dout, const float *dht, void *dq, void *dk, void *dv,
                           float *dg, float *dbeta, float *dh0, void *workspace, size_t workspace_bytes, void *stream,
                           bool recompute)
{
    Dims d;
    const bool varlen = cu_seqlens != nullptr;
    kda_status_t st = check_dims(B, T, H, HV, K, V, varlen, num_seqs, d);
    if (st != KDA_OK) return st;
    const int64_t tokens = static_cast<int64_t>(B) * T;
    if (tokens > 0 && (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta))
        return KDA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) || !aligned(dout, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(dg, 16) || !aligned(dbeta, 4) ||
        !aligned(beta, 4) || !aligned(initial_state, 16) || !aligned(dht, 16) || !aligned(dh0, 16) ||
        !aligned(cu_seqlens, 4))
        return KDA_ERR_MISALIGNED;
    const size_t nq = static_cast<size_t>(tokens) * H * K * 2, nvb = static_cast<size_t>(tokens) * HV * V * 2;
    const size_t ng = static_cast<size_t>(tokens) * HV * K * 4, nb = static_cast<size_t>(tokens) * HV * 4;
    const size_t ns = static_cast<size_t>(d.N) * HV * K * V * 4;
    const void *ins[] = {q, k, v, g, beta, initial_state, cu_seqlens, dout, dht};
    const size_t in_n[] = {nq, nq, nvb, ng, nb, initial_state ? ns : 0,
                           varlen ? static_cast<size_t>(num_seqs + 1) * 4 : 0, nvb, dht ? ns : 0};
    const void *outs[] = {dq, dk, dv, dg, dbeta, dh0};
    const size_t out_n[] = {nq, nq, nvb, ng, nb, dh0 ? ns : 0};
    for (int o = 0; o < 6; ++o) {
        for (int i = 0; i < 9; ++i)
            if (overlaps(outs[o], out_n[o], ins[i], in_n[i])) return KDA_ERR_INVALID_ARG;
        for (int o2 = o + 1; o2 < 6; ++o2)
            if (overlaps(outs[o], out_n[o], outs[o2], out_n[o2])) return KDA_ERR_INVALID_ARG;
    }
    const BwdWorkspace ws = bwd_workspace_layout(B, T, HV, varlen ? num_seqs : 0);
    if (!workspace || workspace_bytes < ws.total) return KDA_ERR_WORKSPACE;
    if (!aligned(workspace, kAlign)) return KDA_ERR_MISALIGNED;
    for (int i = 0; i < 9; ++i)
        if (overlaps(workspace, ws.total, ins[i], in_n[i])) return KDA_ERR_INVALID_ARG;
    for (int o = 0; o < 6; ++o)
        if (overlaps(workspace, ws.total, outs[o], out_n[o])) return KDA_ERR_INVALID_ARG;

    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return KDA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    int32_t *chunk_off = varlen ? reinterpret_cast<int32_t *>(wsb + ws.chunk_off) : nullptr;
    uint8_t *items = wsb + ws.items;
    __nv_bfloat16 *states = reinterpret_cast<__nv_bfloat16 *>(wsb + ws.states);
    __nv_bfloat16 *dstates = reinterpret_cast<__nv_bfloat16 *>(wsb + ws.dstates);
    if (varlen && recompute) {
        kda::chunk_offsets_kernel<<<1, 1024, 0, s>>>(cu_seqlens, num_seqs, chunk_off);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    }
    // 1. the forward's per-chunk blocks, then its carry storing every chunk's start state (no o); a saved
    //    forward left both (and the chunk offsets) in the workspace
    CUtensorMap tq, tk, tv, tg;
    kda::IntraParams ip{};
    if (tokens > 0 && recompute) {
        if (!make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, tokens, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, tokens, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HV, tokens, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&tg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, HV, tokens, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
            return KDA_ERR_CUDA;
        ip.beta = beta;
        ip.cu = cu_seqlens;
        ip.chunk_off = chunk_off;
        ip.items = items;
        ip.err = info.err;
        ip.B = B;
        ip.T = T;
        ip.H = H;
        ip.HV = HV;
        ip.N = d.N;
        ip.chunks_per_seq = (T + CH - 1) / CH;
        ip.prefetch_stride = info.sms * kda::kIntraCtasPerSm;
        if (cudaFuncSetAttribute(kda::kda_intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kda::IntraSmem::TOTAL) != cudaSuccess)
            return KDA_ERR_CUDA;
    }
    auto launch_intra = [&](int chunk_begin, int chunk_count, int64_t grid_chunks) {
        ip.chunk_begin = chunk_begin;
        ip.chunk_count = chunk_count;
        kda::kda_intra_kernel<<<static_cast<int>(grid_chunks * HV), 256, kda::IntraSmem::TOTAL, s>>>(tq, tk, tv, tg,
                                                                                                      ip);
        return cudaGetLastError();
    };
    kda::CarryParams cp{};
    cp.items = items;
    cp.s0 = initial_state;
    cp.cu = cu_seqlens;
    cp.chunk_off = chunk_off;
    cp.sN = reinterpret_cast<float *>(wsb + ws.final_state);
    cp.err = info.err;
    cp.T = T;
    cp.HV = HV;
    cp.N = d.N;
    cp.chunks_per_seq = (T + CH - 1) / CH;
    cp.chunk_begin = 0;
    cp.chunk_count = cp.chunks_per_seq;
    cp.states = states;
    cp.no_o = 1;
    // The forward carry runs on the high-priority side stream, joined before the chunk kernel.  A sequence long
    // enough for the forward's cut into parts is cut the same way here: the carry of part j beside the
    // intra-chunk work of part j + 1 (each part's carry starting from the previous part's fp32 end state, so
    // the stored start states are the ones one launch gives).  The reverse carry reads only the blocks, so it
    // follows the last intra-chunk part on the main stream, beside the last forward-carry parts.
    CarryLane *lane = nullptr;
    std::unique_lock<std::mutex> lane_lock;
    if (recompute) {
        if (carry_lane(info.dev, lane, lane_lock) != cudaSuccess) return KDA_ERR_CUDA;
        const int parts = tokens > 0 ? pipeline_parts(B, T, HV, varlen, info.sms) : 1;
        const int nck = cp.chunks_per_seq;
        const int64_t den = 4 * parts - 3;  // the last part a quarter of the others, as in the forward
        for (int j = 0; j < parts; ++j) {
            const int c0 = parts == 1 ? 0 : static_cast<int>(static_cast<int64_t>(nck) * 4 * j / den);
            const int c1 = j + 1 == parts ? nck : static_cast<int>(static_cast<int64_t>(nck) * 4 * (j + 1) / den);
            if (tokens > 0) {
                const int64_t grid = parts == 1 ? ws.max_chunks : static_cast<int64_t>(B) * (c1 - c0);
                if (launch_intra(c0, c1 - c0, grid) != cudaSuccess) return KDA_ERR_CUDA;
            }
            if (cudaEventRecord(lane->fork, s) != cudaSuccess ||
                cudaStreamWaitEvent(lane->stream, lane->fork, 0) != cudaSuccess)
                return KDA_ERR_CUDA;
            cp.s0 = j == 0 ? initial_state : cp.sN;
            cp.chunk_begin = c0;
            cp.chunk_count = c1 - c0;
            if (launch_carry(cp, d.N * HV, lane->stream) != cudaSuccess) return KDA_ERR_CUDA;
        }
        if (cudaEventRecord(lane->join, lane->stream) != cudaSuccess) return KDA_ERR_CUDA;
    }

    // 2. reverse carry: the gradient at every chunk's end state, and at the initial state
    kda::BwdParams bp{};
    bp.q = static_cast<const __nv_bfloat16 *>(q);
    bp.k = static_cast<const __nv_bfloat16 *>(k);
    bp.v = static_cast<const __nv_bfloat16 *>(v);
    bp.dout = static_cast<const __nv_bfloat16 *>(dout);
    bp.g = g;
    bp.beta = beta;
    bp.items = items;
    bp.states = states;
    bp.dstates = dstates;
    bp.dht = dht;
    bp.dh0 = dh0;
    bp.dqn = reinterpret_cast<float *>(wsb + ws.dqn);
    bp.dkn = reinterpret_cast<float *>(wsb + ws.dkn);
    bp.dq = static_cast<__nv_bfloat16 *>(dq);
    bp.dk = static_cast<__nv_bfloat16 *>(dk);
    bp.fuse_norm = H == HV;
    bp.dv = static_cast<__nv_bfloat16 *>(dv);
    bp.dg = dg;
    bp.dbeta = dbeta;
    bp.cu = cu_seqlens;
    bp.chunk_off = chunk_off;
    bp.err = info.err;
    bp.T = T;
    bp.H = H;
    bp.HV = HV;
    bp.N = d.N;
    bp.chunks_per_seq = (T + CH - 1) / CH;
    if (cudaFuncSetAttribute(kda::kda_bwd_carry_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kda::BcSmem::TOTAL) != cudaSuccess)
        return KDA_ERR_CUDA;
    kda::kda_bwd_carry_kernel<<<d.N * HV, kda::kBcThreads, kda::BcSmem::TOTAL, s>>>(bp);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    if (recompute && cudaStreamWaitEvent(s, lane->join, 0) != cudaSuccess) return KDA_ERR_CUDA;
    if (tokens == 0) return KDA_OK;

    // 3. every chunk's gradients, 4. the Q/K groups through the normalisation
    if (cudaFuncSetAttribute(kda::kda_bwd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kda::BwSmem::TOTAL) != cudaSuccess)
        return KDA_ERR_CUDA;
    kda::kda_bwd_chunk_kernel<<<static_cast<int>(ws.max_chunks * HV), kda::kBwThreads, kda::BwSmem::TOTAL, s>>>(bp);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    if (bp.fuse_norm) return KDA_OK;  // the chunk kernel wrote dq and dk
    const int64_t warps = (tokens * H * 2 + kda::kNormUnits - 1) / kda::kNormUnits;
    kda::kda_bwd_norm_kernel<<<static_cast<int>((warps + 7) / 8), 256, 0, s>>>(bp, tokens);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
}  // namespace
