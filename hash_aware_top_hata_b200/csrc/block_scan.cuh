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
