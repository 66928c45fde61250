// kda_prefill.cu -- C ABI of the KDA chunk-prefill forward (declared in
// include/kda_prefill.h): host-side argument checks and kernel launches.
// No numeric work happens on the host; every step of the forward runs in
// the kernels of kda_fused.cuh / kda_norm.cuh.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "kda_fused.cuh"
#include "kda_norm.cuh"
#include "kda_prefill.h"

namespace {

using kda::CH;
using kda::DK;
using kda::DV;

constexpr size_t kAlign = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

int num_sms(int dev)
{
    static int cached[64] = {0};
    if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

template <int NW>
cudaError_t launch_fused(const kda::FwdParams &p, int units, cudaStream_t stream)
{
    using S = kda::Smem<NW>;
    cudaError_t err = cudaFuncSetAttribute(kda::kda_fused_fwd_kernel<NW>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL);
    if (err != cudaSuccess) return err;
    kda::FwdParams q = p;
    q.nslices = DV / S::VS;
    const int grid = units * q.nslices;
    kda::kda_fused_fwd_kernel<NW><<<grid, NW * 32, S::TOTAL, stream>>>(q);
    return cudaGetLastError();
}

struct Dims {
    int B, T, H, HV, K, V, N;
    bool varlen;
};

kda_status_t check_dims(int B, int T, int H, int HV, int K, int V, bool varlen, int num_seqs, Dims &d)
{
    if (B <= 0 || H <= 0 || HV <= 0 || K <= 0 || V <= 0) return KDA_ERR_INVALID_ARG;
    if (T < 0 || (T == 0 && !varlen)) return KDA_ERR_INVALID_ARG;
    if (HV % H != 0) return KDA_ERR_INVALID_ARG;
    if (K != DK || V != DV) return KDA_ERR_UNSUPPORTED;
    if (varlen && (B != 1 || num_seqs <= 0)) return KDA_ERR_INVALID_ARG;
    const int64_t units = static_cast<int64_t>(varlen ? num_seqs : B) * HV;
    if (units * 2 > INT32_MAX) return KDA_ERR_UNSUPPORTED;
    d = Dims{B, T, H, HV, K, V, varlen ? num_seqs : B, varlen};
    return KDA_OK;
}

}  // namespace

extern "C" const char *kda_status_string(kda_status_t s)
{
    switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    }
    return "KDA_ERR_UNKNOWN";
}

extern "C" size_t kda_prefill_workspace_size(int B, int T, int H, int HV, int K, int V, int num_seqs)
{
    (void)B; (void)T; (void)H; (void)HV; (void)K; (void)V;
    if (num_seqs <= 0) return 0;
    return round_up(static_cast<size_t>(num_seqs) * sizeof(int32_t), kAlign);
}

extern "C" kda_status_t kda_prefill_forward(const void *q, const void *k, const void *v, const float *g,
                                            const float *beta, const float *initial_state,
                                            const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int HV,
                                            int K, int V, void *o, float *final_state, void *workspace,
                                            size_t workspace_bytes, void *stream)
{
    Dims d;
    const bool varlen = cu_seqlens != nullptr;
    kda_status_t st = check_dims(B, T, H, HV, K, V, varlen, num_seqs, d);
    if (st != KDA_OK) return st;
    const int64_t tokens = static_cast<int64_t>(B) * T;
    if (tokens > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    if (!final_state) return KDA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) || !aligned(o, 16) ||
        !aligned(beta, 4) || !aligned(final_state, 4) || !aligned(initial_state, 4) || !aligned(cu_seqlens, 4))
        return KDA_ERR_MISALIGNED;

    const size_t nq = static_cast<size_t>(tokens) * H * K * 2, nvb = static_cast<size_t>(tokens) * HV * V * 2;
    const size_t ng = static_cast<size_t>(tokens) * HV * K * 4, nb = static_cast<size_t>(tokens) * HV * 4;
    const size_t ns = static_cast<size_t>(d.N) * HV * K * V * 4;
    // Outputs may not overlap any input, except final_state == initial_state exactly.
    const void *ins[] = {q, k, v, g, beta, cu_seqlens};
    const size_t in_n[] = {nq, nq, nvb, ng, nb, varlen ? static_cast<size_t>(num_seqs + 1) * 4 : 0};
    for (int i = 0; i < 6; ++i)
        if (overlaps(o, nvb, ins[i], in_n[i]) || overlaps(final_state, ns, ins[i], in_n[i]))
            return KDA_ERR_INVALID_ARG;
    if (overlaps(o, nvb, final_state, ns) || overlaps(o, nvb, initial_state, ns)) return KDA_ERR_INVALID_ARG;
    if (initial_state && initial_state != final_state && overlaps(initial_state, ns, final_state, ns))
        return KDA_ERR_INVALID_ARG;

    const size_t need = kda_prefill_workspace_size(B, T, H, HV, K, V, varlen ? num_seqs : 0);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
        if (!aligned(workspace, kAlign)) return KDA_ERR_MISALIGNED;
        if (overlaps(workspace, need, o, nvb) || overlaps(workspace, need, final_state, ns))
            return KDA_ERR_INVALID_ARG;
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;

    kda::FwdParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.g = g;
    p.beta = beta;
    p.s0 = initial_state;
    p.cu = cu_seqlens;
    p.order = nullptr;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.sN = final_state;
    p.B = B;
    p.T = T;
    p.H = H;
    p.HV = HV;
    p.N = d.N;

    if (varlen) {
        int32_t *order = static_cast<int32_t *>(workspace);
        const int threads = 256;
        const int blocks = (num_seqs + threads - 1) / threads;
        kda::seq_order_kernel<<<blocks, threads, 0, s>>>(cu_seqlens, num_seqs, order);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
        p.order = order;
    }

    // Two value-column slices (4 warps each) when the (sequence, head) units
    // alone would leave SMs idle; otherwise one slice of 8 warps per unit.
    const int units = d.N * HV;
    cudaError_t err;
    if (units * 2 <= num_sms(dev))
        err = launch_fused<4>(p, units, s);
    else
        err = launch_fused<8>(p, units, s);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" size_t kda_prefill_host_staging_size(int B, int T, int H, int HV, int K, int V, int num_seqs,
                                                int has_initial_state, int has_cu_seqlens)
{
    const size_t tokens = static_cast<size_t>(B > 0 ? B : 0) * (T > 0 ? T : 0);
    const size_t N = has_cu_seqlens ? static_cast<size_t>(num_seqs > 0 ? num_seqs : 0) : static_cast<size_t>(B > 0 ? B : 0);
    size_t total = 0;
    total += round_up(tokens * H * K * 2, kAlign) * 2;          // q, k
    total += round_up(tokens * HV * V * 2, kAlign);             // v
    total += round_up(tokens * HV * K * 4, kAlign);             // g
    total += round_up(tokens * HV * 4, kAlign);                 // beta
    if (has_initial_state) total += round_up(N * HV * K * V * 4, kAlign);
    if (has_cu_seqlens) total += round_up((N + 1) * 4, kAlign);
    total += round_up(tokens * HV * V * 2, kAlign);             // o
    total += round_up(N * HV * K * V * 4, kAlign);              // final_state
    total += kda_prefill_workspace_size(B, T, H, HV, K, V, has_cu_seqlens ? num_seqs : 0);
    return total;
}

extern "C" kda_status_t kda_prefill_forward_host(const void *q_h, const void *k_h, const void *v_h, const float *g_h,
                                                 const float *beta_h, const float *s0_h, const int32_t *cu_h,
                                                 int num_seqs, int B, int T, int H, int HV, int K, int V, void *o_h,
                                                 float *sN_h, void *staging, size_t staging_bytes, void *stream)
{
    Dims d;
    const bool varlen = cu_h != nullptr;
    kda_status_t st = check_dims(B, T, H, HV, K, V, varlen, num_seqs, d);
    if (st != KDA_OK) return st;
    const size_t tokens = static_cast<size_t>(B) * T;
    if (tokens > 0 && (!q_h || !k_h || !v_h || !g_h || !beta_h || !o_h)) return KDA_ERR_INVALID_ARG;
    if (!sN_h || !staging) return KDA_ERR_INVALID_ARG;
    const size_t need = kda_prefill_host_staging_size(B, T, H, HV, K, V, num_seqs, s0_h != nullptr, varlen);
    if (staging_bytes < need) return KDA_ERR_WORKSPACE;
    if (!aligned(staging, kAlign)) return KDA_ERR_MISALIGNED;

    const size_t nq = tokens * H * K * 2, nvb = tokens * HV * V * 2, ng = tokens * HV * K * 4, nb = tokens * HV * 4;
    const size_t ns = static_cast<size_t>(d.N) * HV * K * V * 4, ncu = varlen ? (static_cast<size_t>(d.N) + 1) * 4 : 0;
    char *base = static_cast<char *>(staging);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base + off;
        off += round_up(bytes, kAlign);
        return p;
    };
    char *dq = take(nq), *dk = take(nq), *dv = take(nvb), *dg = take(ng), *db = take(nb);
    char *ds0 = s0_h ? take(ns) : nullptr;
    char *dcu = varlen ? take(ncu) : nullptr;
    char *dO = take(nvb), *dsN = take(ns);
    const size_t ws = kda_prefill_workspace_size(B, T, H, HV, K, V, varlen ? num_seqs : 0);
    char *dws = ws ? take(ws) : nullptr;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    struct Cp {
        void *dst;
        const void *src;
        size_t n;
    } ins[] = {{dq, q_h, nq}, {dk, k_h, nq}, {dv, v_h, nvb}, {dg, g_h, ng}, {db, beta_h, nb},
               {ds0, s0_h, ns}, {dcu, cu_h, ncu}};
    for (const Cp &c : ins)
        if (c.dst && c.n && cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return KDA_ERR_CUDA;
    st = kda_prefill_forward(dq, dk, dv, reinterpret_cast<float *>(dg), reinterpret_cast<float *>(db),
                             reinterpret_cast<float *>(ds0), reinterpret_cast<int32_t *>(dcu), num_seqs, B, T, H, HV,
                             K, V, dO, reinterpret_cast<float *>(dsN), dws, ws, stream);
    if (st != KDA_OK) return st;
    if (nvb && cudaMemcpyAsync(o_h, dO, nvb, cudaMemcpyDeviceToHost, s) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemcpyAsync(sN_h, dsN, ns, cudaMemcpyDeviceToHost, s) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

extern "C" kda_status_t kda_l2norm_bf16(const void *x, int64_t rows, int K, void *out, void *stream)
{
    if (rows < 0) return KDA_ERR_INVALID_ARG;
    if (K != DK) return KDA_ERR_UNSUPPORTED;
    if (rows == 0) return KDA_OK;
    if (!x || !out) return KDA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16)) return KDA_ERR_MISALIGNED;
    const size_t n = static_cast<size_t>(rows) * K * 2;
    if (x != out && overlaps(x, n, out, n)) return KDA_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    const int64_t blocks_needed = (rows + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms(dev)) * 8;
    const int blocks = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    kda::l2norm_bf16_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(x), rows, static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
