// append.cuh -- a decode loop's per-step bookkeeping in one launch: the
// current token's cache row of every sequence into row `pos` of its cache,
// and its absorbed query into one slot of the recent-query ring (whose mean
// is the summary query of 关键设计 1).  Plain 16-byte copies, one CTA per
// sequence.
#pragma once
#include "common.cuh"

namespace lca {

constexpr int K_APPEND = 9;
constexpr int APPEND_THREADS = 256;
constexpr int ROW_VEC = LCA_D * 2 / 16;                 // 72 x 16 B per cache row
constexpr int QUERY_VEC = LCA_HEADS * LCA_D * 2 / 16;   // 1152 x 16 B per query

// Ordering: waits for everything earlier in the stream before it reads the
// new rows and queries or overwrites cache and ring (an earlier kernel may
// still read them), and lets its dependent (the decode's first kernel, which
// waits for this grid to complete before it reads them) launch at once.
__global__ void __launch_bounds__(APPEND_THREADS) append_token_kernel(const uint4 *__restrict__ rows,
                                                                      uint4 *__restrict__ cache, int64_t pitch,
                                                                      int64_t pos, const uint4 *__restrict__ q,
                                                                      uint4 *__restrict__ ring, int g, int slot)
{
    griddep_wait();
    griddep_launch_dependents();
    const int b = blockIdx.x;
    for (int i = threadIdx.x; i < ROW_VEC; i += APPEND_THREADS)
        cache[(size_t(b) * size_t(pitch) + size_t(pos)) * ROW_VEC + i] = rows[size_t(b) * ROW_VEC + i];
    if (q) {
        const uint4 *src = q + size_t(b) * QUERY_VEC;
        uint4 *dst = ring + (size_t(b) * g + slot) * QUERY_VEC;
        for (int i = threadIdx.x; i < QUERY_VEC; i += APPEND_THREADS) dst[i] = src[i];
    }
}

}  // namespace lca
