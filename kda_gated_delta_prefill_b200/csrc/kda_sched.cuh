// kda_sched.cuh -- device-side chunk scheduler for packed varlen batches:
// chunk offsets of every sequence (exclusive scan of ceil(len/64)), the
// longest-first order in which the carry kernel takes the sequences, and the
// per-sequence offsets of chunk windows.
// cu_seqlens is read on the device only, so the host never synchronises.
#pragma once
#include <cstdint>

#include "kda_common.cuh"

namespace kda {

// One CTA of 1024 threads: chunk_off[n] = sum_{m<n} ceil(len_m / 64), chunk_off[N] = total.
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(const int32_t *__restrict__ cu, int N,
                                                             int32_t *__restrict__ chunk_off)
{
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int n = base + tid;
        int len = (n < N) ? cu[n + 1] - cu[n] : 0;
        if (len < 0) len = 0;
        const int nch = (len + CH - 1) / CH;
        int x = nch;  // inclusive warp scan
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, off);
                if (lane >= off) w += y;
            }
            warp_sums[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int before = carry + (warp ? warp_sums[warp - 1] : 0) + x - nch;
        if (n < N) chunk_off[n] = before;
        __syncthreads();
        if (tid == 1023) carry = before + nch;
        __syncthreads();
    }
    if (tid == 0) chunk_off[N] = carry;
}

// Windows of chunk index within each packed sequence: window j holds chunks [a[j], a[j] + w[j]) of every
// sequence, so the forward can carry window j while the intra-chunk kernel works on window j+1.
constexpr int kMaxWindows = 4;
struct ChunkWindows {
    int count;
    int a[kMaxWindows], w[kMaxWindows];
};

// One CTA of 1024 threads per window j: woff[j * (N + 1) + n] = number of window-j chunks of the sequences
// before n (exclusive scan of clamp(nck_n - a_j, 0, w_j), nck_n = chunk_off[n + 1] - chunk_off[n]), and
// woff[j * (N + 1) + N] = the window's total.
__global__ void __launch_bounds__(1024) window_offsets_kernel(const int32_t *__restrict__ chunk_off, int N,
                                                              ChunkWindows win, int32_t *__restrict__ woff)
{
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, j = blockIdx.x;
    if (j >= win.count || j >= kMaxWindows) return;
    const int a = win.a[j], w = win.w[j];
    int32_t *out = woff + static_cast<int64_t>(j) * (N + 1);
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int n = base + tid;
        int cnt = (n < N) ? chunk_off[n + 1] - chunk_off[n] - a : 0;
        cnt = cnt < 0 ? 0 : (cnt > w ? w : cnt);
        int x = cnt;  // inclusive warp scan
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int v = warp_sums[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, v, off);
                if (lane >= off) v += y;
            }
            warp_sums[lane] = v;
        }
        __syncthreads();
        const int before = carry + (warp ? warp_sums[warp - 1] : 0) + x - cnt;
        if (n < N) out[n] = before;
        __syncthreads();
        if (tid == 1023) carry = before + cnt;
        __syncthreads();
    }
    if (tid == 0) out[N] = carry;
}

// Longest-first order of packed sequences: order[rank] = n, ranks by
// descending length, ties by index.  One thread per sequence.
__global__ void __launch_bounds__(256) seq_order_kernel(const int32_t *__restrict__ cu, int N, int32_t *__restrict__ order)
{
    __shared__ int32_t len_tile[1024];
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int my = (n < N) ? cu[n + 1] - cu[n] : 0;
    int rank = 0;
    for (int base = 0; base < N; base += 1024) {
        __syncthreads();
        for (int i = threadIdx.x; i < 1024; i += blockDim.x)
            len_tile[i] = (base + i < N) ? cu[base + i + 1] - cu[base + i] : -1;
        __syncthreads();
        const int lim = (N - base) < 1024 ? (N - base) : 1024;
        for (int i = 0; i < lim; ++i) {
            const int l = len_tile[i];
            rank += (l > my) || (l == my && base + i < n);
        }
    }
    if (n < N) order[rank] = n;
}

}  // namespace kda
