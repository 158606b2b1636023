// block_scan.cuh -- warp-shuffle exclusive prefix sums over a thread block.
#pragma once

namespace hata {

__device__ __forceinline__ int warp_inclusive_scan(int v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Exclusive prefix sum of v over the block, in threadIdx.x order; *total gets
// the block sum.  scratch: >= NT/32 + 1 ints of shared memory.  Every thread
// of the block must call it; it synchronises the block twice.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int *scratch, int *total)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int inc = warp_inclusive_scan(v);
    if (lane == 31) scratch[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NW ? scratch[lane] : 0;
        const int winc = warp_inclusive_scan(w);
        if (lane < NW) scratch[lane] = winc - w;
        if (lane == NW - 1) scratch[NW] = winc;
    }
    __syncthreads();
    const int r = scratch[warp] + inc - v;
    *total = scratch[NW];
    __syncthreads();  // scratch may be reused right after
    return r;
}

}  // namespace hata

namespace hata {

// Exclusive prefix sums of two counters (a, b) over the first NT threads of
// the block at once, in threadIdx.x order; *ta / *tb get the sums.  scratch:
// >= NT/32 + 1 int2 of shared memory.  Every one of the NT threads must call
// it.  BAR = 0 synchronises with __syncthreads (NT = the block size); any
// other BAR with the named barrier BAR over those NT threads, so that other
// warps of the block may run unrelated work meanwhile.  Two barriers, plus
// one at the end so that scratch may be reused right after.
template <int NT, int BAR = 0>
__device__ __forceinline__ int2 block_exclusive_scan2(int a, int b, int2 *scratch, int *ta, int *tb)
{
    constexpr int NW = NT / 32;
    auto sync = [] {
        if constexpr (BAR == 0)
            __syncthreads();
        else
            asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
    };
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int na = __shfl_up_sync(0xffffffffu, ia, o);
        const int nb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) { ia += na; ib += nb; }
    }
    if (lane == 31) scratch[warp] = make_int2(ia, ib);
    sync();
    if (warp == 0) {
        const int2 w = lane < NW ? scratch[lane] : make_int2(0, 0);
        int wa = w.x, wb = w.y;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int na = __shfl_up_sync(0xffffffffu, wa, o);
            const int nb = __shfl_up_sync(0xffffffffu, wb, o);
            if (lane >= o) { wa += na; wb += nb; }
        }
        if (lane < NW) scratch[lane] = make_int2(wa - w.x, wb - w.y);
        if (lane == NW - 1) scratch[NW] = make_int2(wa, wb);
    }
    sync();
    const int2 base = scratch[warp];
    *ta = scratch[NW].x;
    *tb = scratch[NW].y;
    sync();
    return make_int2(base.x + ia - a, base.y + ib - b);
}

}  // namespace hata
