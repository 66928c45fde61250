// kda_sched.cuh -- device-side chunk scheduler for packed varlen batches:
// chunk offsets of every sequence (exclusive scan of ceil(len/64)) and the
// longest-first order in which the carry kernel takes the sequences.
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
