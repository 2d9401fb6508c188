// Block-wide scans and the radix-digit search shared by the selection kernels
// (topk.cu, select.cu).  Device-only; internal to the li library.
#pragma once

#include <stdint.h>

namespace li {

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Block-wide inclusive scan with one __syncthreads: each warp scans its lanes,
// then every warp scans the NW warp totals in parallel (lane l holds warp l's).
// wsum must not be reused before every thread has passed the next block-wide
// barrier.
template <int NW>
__device__ __forceinline__ uint32_t block_scan1(uint32_t v, uint32_t* wsum, uint32_t* total) {
    static_assert(NW >= 1 && NW <= 32, "warps per block");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t incl = warp_incl_scan(v, lane);
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint32_t x = lane < NW ? wsum[lane] : 0u;
#pragma unroll
    for (int o = 1; o < NW; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
    }
    *total = __shfl_sync(0xffffffffu, x, NW - 1);
    const uint32_t before = __shfl_sync(0xffffffffu, x, (warp + 31) & 31);  // warps 0 .. warp-1
    return incl + (warp > 0 ? before : 0u);
}

// Digit of the krem-th largest key from a histogram h[NB] indexed by digit:
// bc[0] = digit, bc[1] = keys in higher digits, bc[2] = keys in that digit,
// bc[3] = total count.  Ends with a block-wide barrier; every thread may read
// bc afterwards.  (0, 0, 0) when the histogram holds fewer than krem keys.
template <int NT, int NB>
__device__ __forceinline__ void find_digit(const uint32_t* h, int krem, uint32_t* wsum, uint32_t* bc) {
    constexpr int OW = NB < NT ? NB : NT;
    constexpr int BPT = NB / OW;
    uint32_t tot[BPT];
    uint32_t s = 0u;
    const bool own = threadIdx.x < OW;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
        tot[i] = own ? h[NB - 1 - (BPT * threadIdx.x + i)] : 0u;
        s += tot[i];
    }
    if (threadIdx.x == 0) bc[0] = bc[1] = bc[2] = 0u;
    uint32_t total;
    const uint32_t incl = block_scan1<NT / 32>(s, wsum, &total);
    const uint32_t excl = incl - s;
    if (own && excl < (uint32_t)krem && incl >= (uint32_t)krem) {
        uint32_t run = excl;
#pragma unroll
        for (int i = 0; i < BPT; ++i) {
            if (run < (uint32_t)krem && run + tot[i] >= (uint32_t)krem) {
                bc[0] = (uint32_t)(NB - 1 - (BPT * threadIdx.x + i));
                bc[1] = run;
                bc[2] = tot[i];
            }
            run += tot[i];
        }
    }
    if (threadIdx.x == 0) bc[3] = total;
    __syncthreads();
}


}  // namespace li
