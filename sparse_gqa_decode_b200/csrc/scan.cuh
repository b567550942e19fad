// scan.cuh -- block-wide exclusive prefix sum of one int32 per thread.
#pragma once

#include "common.cuh"

namespace sgd {

__device__ __forceinline__ int32_t warp_inclusive_scan(int32_t v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Every thread of the block must call this (blockDim.x a multiple of 32, <= 1024).
// `sm` is 33 int32 of shared memory.  Returns the exclusive prefix of v over the
// threads in order and the block total in `total`.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t &total, int32_t *sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int32_t inc = warp_inclusive_scan(v);
    if (lane == 31) sm[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int32_t s = (lane < nw) ? sm[lane] : 0;
        const int32_t si = warp_inclusive_scan(s);
        if (lane < nw) sm[lane] = si;
        const int32_t tot = __shfl_sync(0xffffffffu, si, nw - 1);
        if (lane == 0) sm[32] = tot;
    }
    __syncthreads();
    const int32_t base = warp ? sm[warp - 1] : 0;
    total = sm[32];
    __syncthreads();
    return base + inc - v;
}

// Two exclusive prefix sums at once (one per value), with their block totals; same rules as
// block_exclusive_scan.  `sm` is 33 int2 of shared memory.
__device__ __forceinline__ int2 block_exclusive_scan2(int32_t a, int32_t b, int2 &total, int2 *sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int32_t ia = warp_inclusive_scan(a), ib = warp_inclusive_scan(b);
    if (lane == 31) sm[warp] = make_int2(ia, ib);
    __syncthreads();
    if (warp == 0) {
        const int2 v = (lane < nw) ? sm[lane] : make_int2(0, 0);
        const int32_t sa = warp_inclusive_scan(v.x), sb = warp_inclusive_scan(v.y);
        if (lane < nw) sm[lane] = make_int2(sa, sb);
        const int32_t ta = __shfl_sync(0xffffffffu, sa, nw - 1), tb = __shfl_sync(0xffffffffu, sb, nw - 1);
        if (lane == 0) sm[32] = make_int2(ta, tb);
    }
    __syncthreads();
    const int2 base = warp ? sm[warp - 1] : make_int2(0, 0);
    total = sm[32];
    __syncthreads();
    return make_int2(base.x + ia - a, base.y + ib - b);
}

}  // namespace sgd
