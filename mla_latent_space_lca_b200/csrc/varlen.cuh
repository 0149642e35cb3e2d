// varlen.cuh -- tile list of a ragged decode batch: sequence b holds lens[b]
// rows, and its tiles (history tiles of 4 groups, or stored-representative
// tiles, then window tiles; seq_geom) are tile_start[b] .. tile_start[b+1]-1
// of the batch's list, an exclusive prefix sum.  One CTA scans the batch
// in chunks of 1024 sequences.
#pragma once
#include "attn_decode.cuh"

namespace lca {

constexpr int VT_THREADS = 1024;

template <int MODE>
__global__ void __launch_bounds__(VT_THREADS)
    varlen_tiles_kernel(const int32_t *__restrict__ lens, int B, int64_t L_max, int w,
                        int32_t *__restrict__ tile_start)
{
    __shared__ int32_t wsum[32];
    __shared__ int32_t carry;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < B; base += VT_THREADS) {
        const int b = base + threadIdx.x;
        const int n = b < B ? seq_geom<MODE>(clamp_len(lens[b], L_max), w).n_tiles : 0;
        int x = n;   // inclusive scan within the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {   // scan of the 32 warp totals
            int v = wsum[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, v, off);
                if (lane >= off) v += y;
            }
            wsum[lane] = v;
        }
        __syncthreads();
        const int excl = carry + (warp ? wsum[warp - 1] : 0) + x - n;
        if (b < B) tile_start[b] = excl;
        __syncthreads();
        if (threadIdx.x == VT_THREADS - 1) carry = excl + n;
        __syncthreads();
    }
    if (threadIdx.x == 0) tile_start[B] = carry;
}

}  // namespace lca
