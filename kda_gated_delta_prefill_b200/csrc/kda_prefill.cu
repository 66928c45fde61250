// kda_prefill.cu -- C ABI of the KDA chunk-prefill forward (declared in
// include/kda_prefill.h): host-side argument checks, workspace layout,
// tensor maps and kernel launches.  No numeric work happens on the host;
// every step of the forward runs in the kernels of kda_intra.cuh,
// kda_carry.cuh, kda_sched.cuh and kda_norm.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "kda_backward.cuh"
#include "kda_carry.cuh"
#include "kda_decode.cuh"
#include "kda_intra.cuh"
#include "kda_norm.cuh"
#include "kda_prefill.h"
#include "kda_scan.cuh"
#include "kda_sched.cuh"

// Bits set by kernels whose bounded waits gave up (see ptx.cuh).  Host code
// reaches it only through the address cudaGetSymbolAddress returns.
static __device__ unsigned g_kda_device_error;

namespace {

using kda::CH;
using kda::DK;
using kda::DV;

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

// Per-device facts: the SM count (looked up once; it belongs to the device, not to a context) and the error
// word's device address, looked up on every call so that a recreated context (after cudaDeviceReset) never
// receives a stale address.
struct DeviceInfo {
    bool ready = false;
    int dev = 0;
    int sms = 148;
    unsigned *err = nullptr;
};
std::mutex g_info_mu;
DeviceInfo g_info[kMaxDevices];

cudaError_t device_info(DeviceInfo &out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(g_info_mu);
        DeviceInfo &d = g_info[dev];
        if (!d.ready) {
            d.dev = dev;
            e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            d.ready = true;
        }
        out = d;
    }
    return cudaGetSymbolAddress(reinterpret_cast<void **>(&out.err), g_kda_device_error);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [rows][heads][128] tensor as a 3D tiled map; one TMA box = 64 rows of one head.
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, int heads, int64_t rows,
              int box_inner, CUtensorMapSwizzle sw)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(128) * elem_bytes, static_cast<cuuint64_t>(heads) * 128 * elem_bytes};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 1, static_cast<cuuint32_t>(CH)};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
    // token rows are TMA coordinates (int32); grids stay below 2^31 blocks
    if (static_cast<int64_t>(B) * T > INT_MAX - CH) return KDA_ERR_UNSUPPORTED;
    const int64_t N = varlen ? num_seqs : B;
    const int64_t max_chunks = varlen ? (static_cast<int64_t>(T) + CH - 1) / CH + N
                                      : static_cast<int64_t>(B) * ((T + CH - 1) / CH);
    if (max_chunks * HV > INT_MAX || N * HV * 4 > INT_MAX) return KDA_ERR_UNSUPPORTED;
    d = Dims{B, T, H, HV, K, V, static_cast<int>(N), varlen};
    return KDA_OK;
}

// Workspace: [chunk_off (N+1) | order (N) | window offsets (4 x (N+1))] for packed batches, then the
// item blocks.
// Plain batches with few (sequence, value head) units and long sequences: one carry CTA per unit would run far
// longer than everything else, so the carry can run on segments of every sequence at once (segment maps, a
// scan of the start states, then the segments with outputs).  The workspace reserves room for up to
// max_carry_segments segments (a bound that does not depend on the device: segments of 16 chunks or more, at
// most 1024 first-pass CTAs, units <= 48); the forward picks the count on the device.
int max_carry_segments(int B, int T, int HV, bool varlen)
{
    const int64_t units = static_cast<int64_t>(B) * HV;
    if (varlen || units > 48) return 1;
    const int64_t by_ctas = 1024 / (2 * units + 1);
    const int64_t by_len = ((static_cast<int64_t>(T) + CH - 1) / CH) / 16;
    const int64_t segs = by_ctas < by_len ? by_ctas : by_len;
    return segs >= 3 ? static_cast<int>(segs) : 1;
}

// Segment count for this device, from a cost model in carry chunk periods fitted to measurements on B200
// (intra-chunk work of one (chunk, head) item is about 1/32 of a period):
//   segmented = intra + (waves of the first pass + waves of the second) x (chunks per segment + 3) + 4 per
//               scan step (the +3: pipeline fill and the state's load and store in each pass),
//   otherwise = max(5/4 carry + intra / 4, 27/20 intra) (the carry overlapping the intra-chunk work).
// Picks the cheapest count, and segments only when that is under 90 % of the alternative.  1 = no segments.
int carry_segments(int B, int T, int HV, bool varlen, int sms)
{
    const int smax = max_carry_segments(B, T, HV, varlen);
    if (smax < 3) return 1;
    const int64_t units = static_cast<int64_t>(B) * HV, nck = (static_cast<int64_t>(T) + CH - 1) / CH;
    const int64_t intra = units * nck / 32;
    const int64_t a = 5 * nck / 4 + intra / 4, b = 27 * intra / 20;
    int best = 1;
    int64_t best_cost = (a > b ? a : b) * 9 / 10;
    for (int sg = 3; sg <= smax; ++sg) {
        const int64_t w1 = (units * (2 * sg - 1) + sms - 1) / sms, w2 = (units * sg + sms - 1) / sms;
        const int64_t cost = intra + (w1 + w2) * ((nck + sg - 1) / sg + 3) + 4 * sg;
        if (cost < best_cost) {
            best_cost = cost;
            best = sg;
        }
    }
    return best;
}

struct Workspace {
    size_t chunk_off = 0, order = 0, win_off = 0, items = 0, seg = 0, total = 0;
    int64_t max_chunks = 0;
    int segments = 1;
};

Workspace workspace_layout(int B, int T, int HV, int num_seqs)
{
    Workspace w;
    const bool varlen = num_seqs > 0;
    w.max_chunks = varlen ? (static_cast<int64_t>(T) + CH - 1) / CH + num_seqs
                          : static_cast<int64_t>(B) * ((T + CH - 1) / CH);
    size_t off = 0;
    if (varlen) {
        w.chunk_off = off;
        off += round_up((static_cast<size_t>(num_seqs) + 1) * 4, kAlign);
        w.order = off;
        off += round_up(static_cast<size_t>(num_seqs) * 4, kAlign);
        w.win_off = off;
        off += round_up(static_cast<size_t>(kda::kMaxWindows) * (num_seqs + 1) * 4, kAlign);
    }
    w.items = off;
    off += static_cast<size_t>(w.max_chunks) * HV * kda::ITEM_BYTES;
    w.segments = max_carry_segments(B, T, HV, varlen);
    if (w.segments > 1) {  // start states, maps and zero-start images: 3 x units x segments fp32 [K][V]
        off = round_up(off, kAlign);
        w.seg = off;
        off += 3 * static_cast<size_t>(B) * HV * w.segments * DK * DV * sizeof(float);
    }
    w.total = round_up(off, kAlign);
    return w;
}

// Fixed-length batches with fewer (sequence, value head) units than SMs leave most of the GPU idle while the
// state carry runs.  Such a forward is cut into parts along the sequence (whole chunks): the carry of part j
// runs on a high-priority side stream, one CTA per unit, while the intra-chunk kernel of part j+1 fills the
// remaining SMs.  The carry of part j starts from the state part j-1 left in final_state.
constexpr int kMaxParts = 8;
constexpr int kMinChunksPerPart = 16;

int pipeline_parts(int B, int T, int HV, bool varlen, int sms)
{
    if (varlen || static_cast<int64_t>(B) * HV >= sms) return 1;
    const int chunks = (T + CH - 1) / CH;
    const int parts = chunks / kMinChunksPerPart;
    return parts < 2 ? 1 : (parts < kMaxParts ? parts : kMaxParts);
}

// Plain batches with more (sequence, value head) units than SMs but fewer than twice as many carry in two waves,
// and the second, partial wave runs alone.  Such a batch is instead split by value heads into two groups: the
// last group is as many heads as make one full wave of carry CTAs (floor(SMs / B) heads), the first the rest.
// The first group's carry then runs beside the last group's intra-chunk work, and the last group's carry is one
// full wave at the end.  (More groups would not help: a carry costs more SM-time beside intra-chunk work than in
// a full last wave.)  Returns the heads of the last group, or 0 for no split.
int head_group_split(int B, int T, int HV, int sms)
{
    const int64_t units = static_cast<int64_t>(B) * HV;
    const int chunks = (T + CH - 1) / CH;
    if (units <= sms || units >= 2 * static_cast<int64_t>(sms) || chunks < kMinChunksPerPart) return 0;
    const int last = sms / B;
    return last > 0 && last < HV ? last : 0;
}

// Packed batches whose lengths the host knows: when the longest sequence is long and the units carried past its
// first window fit beside the intra-chunk work, the batch is cut into windows of chunk index within each
// sequence, the longest sequence's chunks split like a plain sequence into parts (the last a quarter of the
// others).  The carry of window j (every sequence with chunks in it, longest first) runs while the intra-chunk
// kernel works on window j+1.  Window 0 holds every sequence's first chunks; later windows only the longer
// sequences.  At most kMaxWindows (4) windows: each intra-chunk launch ends in a partly filled wave of CTAs,
// which short windows cannot amortise (on the packed GQA workload 4 windows beat 2, 3, 6 and 8).
struct WindowPlan {
    kda::ChunkWindows win{};
    int64_t items[kda::kMaxWindows] = {};  // chunks in each window
    int seqs[kda::kMaxWindows] = {};       // sequences with chunks in each window (window 0: all)
};

int plan_windows(const int32_t *cu_host, int N, int HV, int sms, WindowPlan &pl)
{
    if (!cu_host || N <= 0) return 1;
    int longest = 0;
    for (int n = 0; n < N; ++n) {
        const int64_t len = static_cast<int64_t>(cu_host[n + 1]) - cu_host[n];
        const int nck = len > 0 ? static_cast<int>((len + CH - 1) / CH) : 0;
        longest = nck > longest ? nck : longest;
    }
    int parts = longest / kMinChunksPerPart;
    parts = parts < 2 ? 1 : (parts < kda::kMaxWindows ? parts : kda::kMaxWindows);
    if (parts == 1) return 1;
    const int64_t den = 4 * parts - 3;  // the last window a quarter of the others, as for plain batches
    for (int j = 0; j <= parts; ++j) {
        const int a = j == parts ? longest : static_cast<int>(static_cast<int64_t>(longest) * 4 * j / den);
        if (j < parts) pl.win.a[j] = a;
        if (j > 0) pl.win.w[j - 1] = a - pl.win.a[j - 1];
    }
    pl.win.count = parts;
    for (int j = 0; j < parts; ++j) {
        pl.items[j] = 0;
        pl.seqs[j] = j == 0 ? N : 0;
        for (int n = 0; n < N; ++n) {
            const int64_t len = static_cast<int64_t>(cu_host[n + 1]) - cu_host[n];
            const int nck = len > 0 ? static_cast<int>((len + CH - 1) / CH) : 0;
            const int in = nck - pl.win.a[j];
            if (in > 0) {
                pl.items[j] += in < pl.win.w[j] ? in : pl.win.w[j];
                if (j > 0) ++pl.seqs[j];
            }
        }
    }
    // the later windows' carries must leave room for the intra-chunk work beside them
    return static_cast<int64_t>(pl.seqs[1]) * HV < sms ? parts : 1;
}

// A lane: a side stream for the carry and its fork/join events, created on first use.  A forward that cuts its
// sequence into parts holds one lane (its mutex) while it enqueues, so that one forward's launches and event
// records stay together.  Each device has several lanes and a call takes a free one, so forwards that host
// threads issue at the same time on different streams get different side streams and their carries overlap.
struct CarryLane {
    bool ready = false;
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    // the host-buffer forward: an upload stream (inputs, part by part), a download stream (o, part by part)
    bool io_ready = false;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, down_done = nullptr, up_done[8] = {}, part_done[8] = {};
    std::mutex mu;
};
constexpr int kLanesPerDevice = 4;
CarryLane g_lane[kMaxDevices][kLanesPerDevice];
std::mutex g_lane_mu;

// Takes a lane of device `dev` (a free one if any, else waits for the first) and returns it locked.
cudaError_t carry_lane(int dev, CarryLane *&out, std::unique_lock<std::mutex> &held)
{
    CarryLane *pick = nullptr;
    for (int i = 0; i < kLanesPerDevice && !pick; ++i) {
        std::unique_lock<std::mutex> trial(g_lane[dev][i].mu, std::try_to_lock);
        if (trial.owns_lock()) {
            pick = &g_lane[dev][i];
            held = std::move(trial);
        }
    }
    if (!pick) {
        pick = &g_lane[dev][0];
        held = std::unique_lock<std::mutex>(pick->mu);
    }
    std::lock_guard<std::mutex> lock(g_lane_mu);
    CarryLane &l = *pick;
    if (!l.ready) {
        int least = 0, greatest = 0;
        cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        if (e != cudaSuccess) return e;
        e = cudaStreamCreateWithPriority(&l.stream, cudaStreamNonBlocking, greatest);
        if (e != cudaSuccess) return e;
        e = cudaEventCreateWithFlags(&l.fork, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        e = cudaEventCreateWithFlags(&l.join, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        l.ready = true;
    }
    out = &l;
    return cudaSuccess;
}

static_assert(kMaxParts <= 8, "a lane holds one upload and one download event per part");

// The host-buffer forward's copy streams and events of a lane, created on first use.
cudaError_t host_io_lane(CarryLane &l)
{
    std::lock_guard<std::mutex> lock(g_lane_mu);
    if (l.io_ready) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&l.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&l.down, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&l.start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&l.down_done, cudaEventDisableTiming);
    for (int j = 0; j < 8 && e == cudaSuccess; ++j) {
        e = cudaEventCreateWithFlags(&l.up_done[j], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&l.part_done[j], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) l.io_ready = true;
    return e;
}

// Host buffers of the host-buffer forward when it runs part by part: each part's input rows are uploaded on
// their own stream while the previous parts compute, and each part's o rows are downloaded as soon as its
// carry has run, so the two copy directions overlap each other and the kernels.
struct HostIO {
    const void *src[5];     // q, k, v, g, beta on the host ([B, T, heads, width] rows)
    void *dst[5];           // their device copies (the same layout)
    size_t row_bytes[5];    // bytes of one token row of each
    const float *s0_host;   // initial state on the host, or null
    float *s0_dev;          // its device copy
    void *o_host;           // o on the host
    size_t o_row_bytes;
    float *sN_host;         // final state on the host
    size_t state_bytes;
};

// Rows [t0, t1) of every batch row of a [B, T, ...] tensor: one strided copy.
cudaError_t copy_rows(void *dst, const void *src, size_t row_bytes, int B, int T, int t0, int t1, cudaMemcpyKind kind,
                      cudaStream_t st)
{
    if (t1 <= t0 || B <= 0) return cudaSuccess;
    const size_t pitch = static_cast<size_t>(T) * row_bytes, off = static_cast<size_t>(t0) * row_bytes;
    return cudaMemcpy2DAsync(static_cast<char *>(dst) + off, pitch, static_cast<const char *>(src) + off, pitch,
                             static_cast<size_t>(t1 - t0) * row_bytes, B, kind, st);
}

cudaError_t launch_carry(const kda::CarryParams &p, int units, cudaStream_t stream)
{
    auto kern = p.states ? kda::kda_carry_kernel<true> : kda::kda_carry_kernel<false>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kda::CarrySmem::TOTAL);
    if (err != cudaSuccess) return err;
    kern<<<units, kda::kCarryThreads, kda::CarrySmem::TOTAL, stream>>>(p);
    return cudaGetLastError();
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
    Dims d;
    if (check_dims(B, T, H, HV, K, V, num_seqs > 0, num_seqs, d) != KDA_OK) return 0;
    return workspace_layout(B, T, HV, num_seqs > 0 ? num_seqs : 0).total;
}

extern "C" int kda_prefill_kernel_launches(int B, int T, int H, int HV, int K, int V, int num_seqs)
{
    Dims d;
    const bool varlen = num_seqs > 0;
    if (check_dims(B, T, H, HV, K, V, varlen, num_seqs, d) != KDA_OK) return 0;
    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return 0;
    if (varlen) return 2 + (T > 0 ? 1 : 0) + 1;  // chunk offsets, order, intra (if any token), carry
    if (carry_segments(B, T, HV, false, info.sms) > 1) return 4;  // intra, segment maps, scan, segments with outputs
    if (pipeline_parts(B, T, HV, false, info.sms) == 1 && head_group_split(B, T, HV, info.sms) > 0)
        return 4;  // intra and carry of each head group
    return 2 * pipeline_parts(B, T, HV, false, info.sms);
}

extern "C" kda_status_t kda_prefill_device_error(unsigned *word, int clear)
{
    if (!word) return KDA_ERR_INVALID_ARG;
    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemcpy(word, info.err, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    if (clear && cudaMemset(info.err, 0, sizeof(unsigned)) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

namespace {
// The forward; `states` (optional): also store every chunk's start state, bf16 [chunks][HV][K][V] (the
// backward's saved form).
kda_status_t forward_impl(const void *q, const void *k, const void *v, const float *g, const float *beta,
                          const float *initial_state, const int32_t *cu_seqlens, int num_seqs, int B, int T, int H,
                          int HV, int K, int V, void *o, float *final_state, void *workspace, size_t workspace_bytes,
                          void *stream, __nv_bfloat16 *states, const HostIO *hio = nullptr,
                          const int32_t *cu_host = nullptr);
}  // namespace

extern "C" kda_status_t kda_prefill_forward(const void *q, const void *k, const void *v, const float *g,
                                            const float *beta, const float *initial_state,
                                            const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int HV,
                                            int K, int V, void *o, float *final_state, void *workspace,
                                            size_t workspace_bytes, void *stream)
{
    return forward_impl(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, B, T, H, HV, K, V, o, final_state,
                        workspace, workspace_bytes, stream, nullptr);
}

namespace {
// A host copy of cu_seqlens: 0 first, T last, non-decreasing.
bool host_cu_ok(const int32_t *cu, int N, int T)
{
    if (!cu || N <= 0 || cu[0] != 0 || cu[N] != T) return false;
    for (int n = 0; n < N; ++n)
        if (cu[n + 1] < cu[n]) return false;
    return true;
}
}  // namespace

extern "C" kda_status_t kda_prefill_forward_varlen(const void *q, const void *k, const void *v, const float *g,
                                                   const float *beta, const float *initial_state,
                                                   const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                                   int num_seqs, int T, int H, int HV, int K, int V, void *o,
                                                   float *final_state, void *workspace, size_t workspace_bytes,
                                                   void *stream)
{
    if (!cu_seqlens || !host_cu_ok(cu_seqlens_host, num_seqs, T)) return KDA_ERR_INVALID_ARG;
    return forward_impl(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, 1, T, H, HV, K, V, o, final_state,
                        workspace, workspace_bytes, stream, nullptr, nullptr, cu_seqlens_host);
}

extern "C" int kda_prefill_varlen_kernel_launches(int T, int H, int HV, int K, int V, int num_seqs,
                                                  const int32_t *cu_seqlens_host)
{
    Dims d;
    if (check_dims(1, T, H, HV, K, V, true, num_seqs, d) != KDA_OK || !host_cu_ok(cu_seqlens_host, num_seqs, T))
        return 0;
    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return 0;
    WindowPlan wp;
    const int windows = T > 0 ? plan_windows(cu_seqlens_host, num_seqs, HV, info.sms, wp) : 1;
    if (windows > 1) return 3 + 2 * windows;  // chunk offsets, order, window offsets; intra and carry per window
    return 2 + (T > 0 ? 1 : 0) + 1;
}

namespace {
kda_status_t forward_impl(const void *q, const void *k, const void *v, const float *g, const float *beta,
                          const float *initial_state, const int32_t *cu_seqlens, int num_seqs, int B, int T, int H,
                          int HV, int K, int V, void *o, float *final_state, void *workspace, size_t workspace_bytes,
                          void *stream, __nv_bfloat16 *states, const HostIO *hio, const int32_t *cu_host)
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

    const Workspace ws = workspace_layout(B, T, HV, varlen ? num_seqs : 0);
    if (!workspace || workspace_bytes < ws.total) return KDA_ERR_WORKSPACE;
    if (!aligned(workspace, kAlign)) return KDA_ERR_MISALIGNED;
    for (int i = 0; i < 6; ++i)
        if (overlaps(workspace, ws.total, ins[i], in_n[i])) return KDA_ERR_INVALID_ARG;
    if (overlaps(workspace, ws.total, o, nvb) || overlaps(workspace, ws.total, final_state, ns) ||
        overlaps(workspace, ws.total, initial_state, ns))
        return KDA_ERR_INVALID_ARG;

    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return KDA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    int32_t *chunk_off = varlen ? reinterpret_cast<int32_t *>(wsb + ws.chunk_off) : nullptr;
    int32_t *order = varlen ? reinterpret_cast<int32_t *>(wsb + ws.order) : nullptr;
    uint8_t *items = wsb + ws.items;

    if (varlen) {
        kda::chunk_offsets_kernel<<<1, 1024, 0, s>>>(cu_seqlens, num_seqs, chunk_off);
        kda::seq_order_kernel<<<(num_seqs + 255) / 256, 256, 0, s>>>(cu_seqlens, num_seqs, order);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    }

    CUtensorMap tq, tk, tv, tg;
    kda::IntraParams ip{};
    if (tokens > 0) {
        const int64_t rows = tokens;
        if (!make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, rows, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, rows, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HV, rows, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&tg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, HV, rows, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
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
    cp.order = order;
    cp.o = static_cast<__nv_bfloat16 *>(o);
    cp.sN = final_state;
    cp.err = info.err;
    cp.T = T;
    cp.HV = HV;
    cp.N = d.N;
    cp.chunks_per_seq = (T + CH - 1) / CH;
    cp.states = states;

    const int segments = ws.segments > 1 ? carry_segments(B, T, HV, varlen, info.sms) : 1;
    if (segments > 1) {
        if (launch_intra(0, cp.chunks_per_seq, ws.max_chunks) != cudaSuccess) return KDA_ERR_CUDA;
        const int units = d.N * HV;
        float *seg = reinterpret_cast<float *>(wsb + ws.seg);
        const size_t per = static_cast<size_t>(units) * ws.segments * DK * DV;  // reserved for the maximum count
        cp.seg_count = segments;
        cp.seg_S = seg;
        cp.seg_M = seg + per;
        cp.seg_B = seg + 2 * per;
        cp.seg_phase = 1;
        if (launch_carry(cp, units * (2 * segments - 1), s) != cudaSuccess) return KDA_ERR_CUDA;
        kda::kda_seg_scan_kernel<<<units * kda::kScanCtasPerUnit, 256, 0, s>>>(cp.seg_S, cp.seg_M, cp.seg_B,
                                                                             segments);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
        cp.seg_phase = 2;
        return launch_carry(cp, units * segments, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    WindowPlan wp;
    const int windows = varlen && tokens > 0 && !hio ? plan_windows(cu_host, d.N, HV, info.sms, wp) : 1;
    if (windows > 1) {
        int32_t *woff = reinterpret_cast<int32_t *>(wsb + ws.win_off);
        kda::window_offsets_kernel<<<windows, 1024, 0, s>>>(chunk_off, d.N, wp.win, woff);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
        // All on `stream`.  Each window's carry is launched right after its intra-chunk kernel and signals on
        // entry (griddepcontrol.launch_dependents) once its CTAs are resident; the next window's intra-chunk kernel
        // is a programmatic dependent launch of that carry, so it fills the SMs the carry left free instead of
        // racing it for them.  It reads nothing the carry writes.  Every later launch in the stream is ordered as
        // usual: window j+1's carry starts after both window j+1's intra-chunk kernel and window j's carry.
        for (int j = 0; j < windows; ++j) {
            ip.win_off = woff + static_cast<int64_t>(j) * (d.N + 1);
            ip.win_begin = wp.win.a[j];
            ip.chunk_begin = 0;
            ip.chunk_count = 0;
            cudaLaunchConfig_t cfg{};
            cudaLaunchAttribute attr[1]{};
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.gridDim = dim3(static_cast<unsigned>(wp.items[j] * HV));
            cfg.blockDim = dim3(256);
            cfg.dynamicSmemBytes = kda::IntraSmem::TOTAL;
            cfg.stream = s;
            cfg.attrs = attr;
            cfg.numAttrs = j > 0 ? 1 : 0;
            if (cudaLaunchKernelEx(&cfg, kda::kda_intra_kernel, tq, tk, tv, tg, ip) != cudaSuccess)
                return KDA_ERR_CUDA;
            cp.s0 = j == 0 ? initial_state : final_state;
            cp.chunk_begin = wp.win.a[j];
            cp.chunk_count = wp.win.w[j];
            if (launch_carry(cp, wp.seqs[j] * HV, s) != cudaSuccess) return KDA_ERR_CUDA;
        }
        return KDA_OK;
    }
    const int parts = pipeline_parts(B, T, HV, varlen, info.sms);
    if (hio && parts == 1) return KDA_ERR_INVALID_ARG;  // the host-buffer forward copies part by part only here
    if (parts == 1) {
        cp.chunk_begin = 0;
        cp.chunk_count = cp.chunks_per_seq;
        const int last = varlen || tokens == 0 || hio ? 0 : head_group_split(B, T, HV, info.sms);
        if (last > 0) {
            // Two head groups on `stream`: the first group's carry is followed by the last group's intra-chunk
            // kernel as a programmatic dependent launch (it starts once every carry CTA is resident and reads
            // nothing the carry writes), then the last group's carry, an ordinary launch after both.
            const int first = HV - last;
            for (int grp = 0; grp < 2; ++grp) {
                const int h0 = grp == 0 ? 0 : first, nh = grp == 0 ? first : last;
                ip.h_begin = h0;
                ip.h_count = nh;
                ip.chunk_begin = 0;
                ip.chunk_count = cp.chunks_per_seq;
                cudaLaunchConfig_t cfg{};
                cudaLaunchAttribute attr[1]{};
                attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                attr[0].val.programmaticStreamSerializationAllowed = 1;
                cfg.gridDim = dim3(static_cast<unsigned>(static_cast<int64_t>(B) * cp.chunks_per_seq * nh));
                cfg.blockDim = dim3(256);
                cfg.dynamicSmemBytes = kda::IntraSmem::TOTAL;
                cfg.stream = s;
                cfg.attrs = attr;
                cfg.numAttrs = grp > 0 ? 1 : 0;
                if (cudaLaunchKernelEx(&cfg, kda::kda_intra_kernel, tq, tk, tv, tg, ip) != cudaSuccess)
                    return KDA_ERR_CUDA;
                cp.h_begin = h0;
                cp.h_count = nh;
                if (launch_carry(cp, B * nh, s) != cudaSuccess) return KDA_ERR_CUDA;
            }
            return KDA_OK;
        }
        if (tokens > 0 && launch_intra(0, cp.chunks_per_seq, ws.max_chunks) != cudaSuccess) return KDA_ERR_CUDA;
        return launch_carry(cp, d.N * HV, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }

    CarryLane *lane = nullptr;
    std::unique_lock<std::mutex> lane_lock;
    if (carry_lane(info.dev, lane, lane_lock) != cudaSuccess) return KDA_ERR_CUDA;
    // The last part's carry has nothing left to overlap with, so it is a quarter of the size of the others:
    // part j starts at chunk nck * 4j / (4 parts - 3).
    const int nck = cp.chunks_per_seq;
    const int64_t den = 4 * parts - 3;
    auto chunk_at = [&](int j) { return j >= parts ? nck : static_cast<int>(static_cast<int64_t>(nck) * 4 * j / den); };
    auto tok = [&](int c) { return c * CH < T ? c * CH : T; };
    if (hio) {  // uploads: the initial state, then every part's rows, in order, after the stream's earlier work
        if (host_io_lane(*lane) != cudaSuccess || cudaEventRecord(lane->start, s) != cudaSuccess ||
            cudaStreamWaitEvent(lane->up, lane->start, 0) != cudaSuccess ||
            cudaStreamWaitEvent(lane->down, lane->start, 0) != cudaSuccess)
            return KDA_ERR_CUDA;
        if (hio->s0_host && cudaMemcpyAsync(hio->s0_dev, hio->s0_host, hio->state_bytes, cudaMemcpyHostToDevice,
                                            lane->up) != cudaSuccess)
            return KDA_ERR_CUDA;
        for (int j = 0; j < parts; ++j) {
            for (int t = 0; t < 5; ++t)
                if (copy_rows(hio->dst[t], hio->src[t], hio->row_bytes[t], B, T, tok(chunk_at(j)), tok(chunk_at(j + 1)),
                              cudaMemcpyHostToDevice, lane->up) != cudaSuccess)
                    return KDA_ERR_CUDA;
            if (cudaEventRecord(lane->up_done[j], lane->up) != cudaSuccess) return KDA_ERR_CUDA;
        }
    }
    for (int j = 0; j < parts; ++j) {
        const int c0 = chunk_at(j), c1 = chunk_at(j + 1);
        if (hio && cudaStreamWaitEvent(s, lane->up_done[j], 0) != cudaSuccess) return KDA_ERR_CUDA;
        if (launch_intra(c0, c1 - c0, static_cast<int64_t>(B) * (c1 - c0)) != cudaSuccess) return KDA_ERR_CUDA;
        if (cudaEventRecord(lane->fork, s) != cudaSuccess || cudaStreamWaitEvent(lane->stream, lane->fork, 0) != cudaSuccess)
            return KDA_ERR_CUDA;
        cp.s0 = j == 0 ? initial_state : final_state;
        cp.chunk_begin = c0;
        cp.chunk_count = c1 - c0;
        if (launch_carry(cp, d.N * HV, lane->stream) != cudaSuccess) return KDA_ERR_CUDA;
        if (hio) {  // this part's o rows are final: download them beside the next parts
            if (cudaEventRecord(lane->part_done[j], lane->stream) != cudaSuccess ||
                cudaStreamWaitEvent(lane->down, lane->part_done[j], 0) != cudaSuccess ||
                copy_rows(hio->o_host, o, hio->o_row_bytes, B, T, tok(c0), tok(c1), cudaMemcpyDeviceToHost,
                          lane->down) != cudaSuccess)
                return KDA_ERR_CUDA;
        }
    }
    if (cudaEventRecord(lane->join, lane->stream) != cudaSuccess || cudaStreamWaitEvent(s, lane->join, 0) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (hio) {  // the final state after the last carry, then the caller's stream waits for every download
        if (cudaMemcpyAsync(hio->sN_host, final_state, hio->state_bytes, cudaMemcpyDeviceToHost, lane->down) !=
                cudaSuccess ||
            cudaEventRecord(lane->down_done, lane->down) != cudaSuccess ||
            cudaStreamWaitEvent(s, lane->down_done, 0) != cudaSuccess)
            return KDA_ERR_CUDA;
    }
    return KDA_OK;
}
}  // namespace

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
    // A plain batch that the forward cuts into parts: uploads and downloads part by part beside the kernels.
    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return KDA_ERR_CUDA;
    if (!varlen && tokens > 0 && carry_segments(B, T, HV, false, info.sms) == 1 &&
        pipeline_parts(B, T, HV, false, info.sms) > 1) {
        HostIO io{};
        const void *srcs[5] = {q_h, k_h, v_h, g_h, beta_h};
        void *dsts[5] = {dq, dk, dv, dg, db};
        const size_t rows[5] = {static_cast<size_t>(H) * K * 2, static_cast<size_t>(H) * K * 2,
                                static_cast<size_t>(HV) * V * 2, static_cast<size_t>(HV) * K * 4,
                                static_cast<size_t>(HV) * 4};
        for (int t = 0; t < 5; ++t) {
            io.src[t] = srcs[t];
            io.dst[t] = dsts[t];
            io.row_bytes[t] = rows[t];
        }
        io.s0_host = s0_h;
        io.s0_dev = reinterpret_cast<float *>(ds0);
        io.o_host = o_h;
        io.o_row_bytes = static_cast<size_t>(HV) * V * 2;
        io.sN_host = sN_h;
        io.state_bytes = ns;
        return forward_impl(dq, dk, dv, reinterpret_cast<float *>(dg), reinterpret_cast<float *>(db),
                            reinterpret_cast<float *>(ds0), nullptr, 0, B, T, H, HV, K, V, dO,
                            reinterpret_cast<float *>(dsN), dws, ws, stream, nullptr, &io);
    }
    struct Cp {
        void *dst;
        const void *src;
        size_t n;
    } ins[] = {{dq, q_h, nq}, {dk, k_h, nq}, {dv, v_h, nvb}, {dg, g_h, ng}, {db, beta_h, nb},
               {ds0, s0_h, ns}, {dcu, cu_h, ncu}};
    for (const Cp &c : ins)
        if (c.dst && c.n && cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return KDA_ERR_CUDA;
    st = varlen ? kda_prefill_forward_varlen(dq, dk, dv, reinterpret_cast<float *>(dg), reinterpret_cast<float *>(db),
                                             reinterpret_cast<float *>(ds0), reinterpret_cast<int32_t *>(dcu), cu_h,
                                             num_seqs, T, H, HV, K, V, dO, reinterpret_cast<float *>(dsN), dws, ws,
                                             stream)
                : kda_prefill_forward(dq, dk, dv, reinterpret_cast<float *>(dg), reinterpret_cast<float *>(db),
                                      reinterpret_cast<float *>(ds0), nullptr, 0, B, T, H, HV, K, V, dO,
                                      reinterpret_cast<float *>(dsN), dws, ws, stream);
    if (st != KDA_OK) return st;
    if (nvb && cudaMemcpyAsync(o_h, dO, nvb, cudaMemcpyDeviceToHost, s) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemcpyAsync(sN_h, dsN, ns, cudaMemcpyDeviceToHost, s) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

extern "C" kda_status_t kda_decode_step(const void *q, int64_t q_row_stride, const void *k, int64_t k_row_stride,
                                        const void *v, int64_t v_row_stride, const float *g, const float *beta,
                                        void *state, int64_t slot_stride, int num_slots, const int32_t *state_indices,
                                        int B, int H, int HV, int K, int V, void *o, void *stream)
{
    if (B < 0 || H <= 0 || HV <= 0 || num_slots <= 0 || HV % H != 0) return KDA_ERR_INVALID_ARG;
    if (K != DK || V != DV) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    if (static_cast<int64_t>(B) * HV > INT_MAX) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !beta || !state || !state_indices || !o) return KDA_ERR_INVALID_ARG;
    if (q_row_stride < static_cast<int64_t>(H) * K || k_row_stride < static_cast<int64_t>(H) * K ||
        v_row_stride < static_cast<int64_t>(HV) * V || slot_stride < static_cast<int64_t>(HV) * K * V)
        return KDA_ERR_INVALID_ARG;
    if (!aligned(q, 8) || !aligned(k, 8) || !aligned(v, 2) || !aligned(g, 4) || !aligned(beta, 4) ||
        !aligned(state, 16) || !aligned(state_indices, 4) || !aligned(o, 4) || q_row_stride % 4 || k_row_stride % 4 ||
        slot_stride % 8)
        return KDA_ERR_MISALIGNED;
    const size_t nq = static_cast<size_t>(B - 1) * q_row_stride * 2 + static_cast<size_t>(H) * K * 2;
    const size_t nk = static_cast<size_t>(B - 1) * k_row_stride * 2 + static_cast<size_t>(H) * K * 2;
    const size_t nv = static_cast<size_t>(B - 1) * v_row_stride * 2 + static_cast<size_t>(HV) * V * 2;
    const size_t ng = static_cast<size_t>(B) * HV * K * 4, nb = static_cast<size_t>(B) * HV * 4;
    const size_t ns = static_cast<size_t>(num_slots - 1) * slot_stride * 2 + static_cast<size_t>(HV) * K * V * 2;
    const size_t no = static_cast<size_t>(B) * HV * V * 2, ni = static_cast<size_t>(B) * 4;
    // o overlaps nothing; the pool overlaps no input
    const void *ins[] = {q, k, v, g, beta, state_indices};
    const size_t in_n[] = {nq, nk, nv, ng, nb, ni};
    for (int i = 0; i < 6; ++i)
        if (overlaps(o, no, ins[i], in_n[i]) || overlaps(state, ns, ins[i], in_n[i])) return KDA_ERR_INVALID_ARG;
    if (overlaps(o, no, state, ns)) return KDA_ERR_INVALID_ARG;

    kda::DecodeParams dp{};
    dp.q = static_cast<const __nv_bfloat16 *>(q);
    dp.k = static_cast<const __nv_bfloat16 *>(k);
    dp.v = static_cast<const __nv_bfloat16 *>(v);
    dp.q_stride = q_row_stride;
    dp.k_stride = k_row_stride;
    dp.v_stride = v_row_stride;
    dp.g = g;
    dp.beta = beta;
    dp.state = static_cast<__nv_bfloat16 *>(state);
    dp.slot_stride = slot_stride;
    dp.state_indices = state_indices;
    dp.o = static_cast<__nv_bfloat16 *>(o);
    dp.B = B;
    dp.H = H;
    dp.HV = HV;
    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return KDA_ERR_CUDA;
    dp.err = info.err;
    using namespace kda;
    auto kern = kda_decode_kernel<kDecodeThreads, kDecodeStages>;
    constexpr int smem = DecodeSmem<kDecodeThreads, kDecodeStages>::TOTAL;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return KDA_ERR_CUDA;
    const int64_t units = static_cast<int64_t>(B) * HV, cap = static_cast<int64_t>(info.sms) * kDecodeCtasPerSm;
    const int grid = static_cast<int>(units < cap ? units : cap);
    kern<<<grid, kDecodeThreads, smem, static_cast<cudaStream_t>(stream)>>>(dp);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
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
    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return KDA_ERR_CUDA;
    const int64_t blocks_needed = (rows + 127) / 128;  // 8 warps of 16 rows
    const int64_t cap = static_cast<int64_t>(info.sms) * 8;
    const int blocks = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    kda::l2norm_bf16_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(x), rows, static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Allocation-free variant of kda_prefill_forward.
//
// Some callers cannot hand the library a workspace: an inference runtime that
// freezes its device memory after warm-up (a cudaMalloc would synchronise the
// whole device and stall every other stream), or a plugin host that gives its
// plugins no allocator at all.  For them the workspace lives in a fixed
// file-scope device array that every GPU loading this library reserves until
// the process exits.  Host code must not use the array's name as an address:
// on the host it is only a stand-in symbol, so its device address is looked
// up once per device with cudaGetSymbolAddress and cached for the life of the
// process (so a context destroyed by cudaDeviceReset leaves a stale address:
// the header tells callers not to use this entry point after a reset).
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
static __device__ __align__(256) uint8_t g_kda_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

extern "C" kda_status_t kda_prefill_forward_noalloc(const void *q, const void *k, const void *v, const float *g,
                                                    const float *beta, const float *initial_state,
                                                    const int32_t *cu_seqlens, int num_seqs, int B, int T, int H,
                                                    int HV, int K, int V, void *o, float *final_state, void *stream)
{
    Dims d;
    const bool varlen = cu_seqlens != nullptr;
    const kda_status_t st = check_dims(B, T, H, HV, K, V, varlen, num_seqs, d);
    if (st != KDA_OK) return st;
    const size_t need = workspace_layout(B, T, HV, varlen ? num_seqs : 0).total;
    if (need > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
            g_noalloc_ptr[dev] = p;
        }
        scratch = g_noalloc_ptr[dev];
    }
    // Everything the kernels read from the scratch is written earlier in the
    // same call (chunk offsets, sequence order, chunk blocks), so nothing
    // needs clearing between calls.
    return kda_prefill_forward(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, B, T, H, HV, K, V, o,
                               final_state, scratch, kNoAllocScratchBytes, stream);
}

// ---------------------------------------------------------------------------------------------------------
// bf16 state storage: the forward with a bf16 initial and final state.  The state is widened into fp32 scratch
// before the carry and rounded (nearest even) after it, so every mode of the forward applies unchanged.
namespace kda {
__global__ void __launch_bounds__(256) state_bf16_to_f32_kernel(const __nv_bfloat16 *__restrict__ in,
                                                                float *__restrict__ out, int64_t n8)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint4 r = reinterpret_cast<const uint4 *>(in)[i];
        float4 *o = reinterpret_cast<float4 *>(out) + 2 * i;
        o[0] = make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
        o[1] = make_float4(bf16lo(r.z), bf16hi(r.z), bf16lo(r.w), bf16hi(r.w));
    }
}
__global__ void __launch_bounds__(256) state_f32_to_bf16_kernel(const float *__restrict__ in,
                                                                __nv_bfloat16 *__restrict__ out, int64_t n8)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 a = reinterpret_cast<const float4 *>(in)[2 * i], b = reinterpret_cast<const float4 *>(in)[2 * i + 1];
        reinterpret_cast<uint4 *>(out)[i] =
            make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
    }
}
}  // namespace kda

extern "C" size_t kda_prefill_state_bf16_workspace_size(int B, int T, int H, int HV, int K, int V, int num_seqs)
{
    Dims d;
    if (check_dims(B, T, H, HV, K, V, num_seqs > 0, num_seqs, d) != KDA_OK) return 0;
    const size_t state = static_cast<size_t>(d.N) * HV * K * V * sizeof(float);
    return workspace_layout(B, T, HV, num_seqs > 0 ? num_seqs : 0).total + 2 * round_up(state, kAlign);
}

extern "C" kda_status_t kda_prefill_forward_state_bf16(const void *q, const void *k, const void *v, const float *g,
                                                       const float *beta, const void *initial_state,
                                                       const int32_t *cu_seqlens, int num_seqs, int B, int T, int H,
                                                       int HV, int K, int V, void *o, void *final_state,
                                                       void *workspace, size_t workspace_bytes, void *stream)
{
    Dims d;
    const bool varlen = cu_seqlens != nullptr;
    kda_status_t st = check_dims(B, T, H, HV, K, V, varlen, num_seqs, d);
    if (st != KDA_OK) return st;
    if (!final_state) return KDA_ERR_INVALID_ARG;
    if (!aligned(initial_state, 16) || !aligned(final_state, 16)) return KDA_ERR_MISALIGNED;
    const size_t nstate = static_cast<size_t>(d.N) * HV * K * V;
    const size_t fwd = workspace_layout(B, T, HV, varlen ? num_seqs : 0).total;
    const size_t need = fwd + 2 * round_up(nstate * sizeof(float), kAlign);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if (!aligned(workspace, kAlign)) return KDA_ERR_MISALIGNED;
    if (overlaps(workspace, need, initial_state, initial_state ? nstate * 2 : 0) ||
        overlaps(workspace, need, final_state, nstate * 2) ||
        (initial_state && initial_state != final_state && overlaps(initial_state, nstate * 2, final_state, nstate * 2)))
        return KDA_ERR_INVALID_ARG;
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    float *s0 = reinterpret_cast<float *>(wsb + fwd);
    float *sN = reinterpret_cast<float *>(wsb + fwd + round_up(nstate * sizeof(float), kAlign));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DeviceInfo info;
    if (device_info(info) != cudaSuccess) return KDA_ERR_CUDA;
    const int64_t n8 = static_cast<int64_t>(nstate / 8);
    const int grid = static_cast<int>(std::min<int64_t>((n8 + 255) / 256, static_cast<int64_t>(info.sms) * 8));
    if (initial_state) {
        kda::state_bf16_to_f32_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(initial_state), s0, n8);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    }
    st = kda_prefill_forward(q, k, v, g, beta, initial_state ? s0 : nullptr, cu_seqlens, num_seqs, B, T, H, HV, K, V, o,
                             sN, workspace, fwd, stream);
    if (st != KDA_OK) return st;
    kda::state_f32_to_bf16_kernel<<<grid, 256, 0, s>>>(sN, static_cast<__nv_bfloat16 *>(final_state), n8);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// The backward's entry points (they use the helpers above).
#include "kda_backward_api.cuh"
