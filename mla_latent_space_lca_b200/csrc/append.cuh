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
constexpr int APPEND_SPLIT = 8;                          // CTAs per sequence
constexpr int ROW_VEC = LCA_D * 2 / 16;                 // 72 x 16 B per cache row
constexpr int QUERY_VEC = LCA_HEADS * LCA_D * 2 / 16;   // 1152 x 16 B per query

// Ordering: waits for everything earlier in the stream before it reads the
// new rows and queries or overwrites cache and ring (an earlier kernel may
// still read them), and lets its dependent (the decode's first kernel, which
// waits for this grid to complete before it reads them) launch at once.
// Each sequence's [row | query] vectors are split over APPEND_SPLIT CTAs so
// that every thread moves at most one 16-byte vector: the sources may be
// pinned host memory, and then the whole copy costs one round trip over the
// host link.
__global__ void __launch_bounds__(APPEND_THREADS) append_token_kernel(const uint4 *__restrict__ rows,
                                                                      uint4 *__restrict__ cache, int64_t pitch,
                                                                      int64_t pos, const uint4 *__restrict__ q,
                                                                      uint4 *__restrict__ ring, int g, int slot,
                                                                      uint4 *__restrict__ q_dst)
{
    griddep_wait();
    griddep_launch_dependents();
    const int b = blockIdx.x;
    const int n = ROW_VEC + (q ? QUERY_VEC : 0);
    const int per = (n + int(gridDim.y) - 1) / int(gridDim.y);
    const int i1 = min(n, (int(blockIdx.y) + 1) * per);
    for (int i = int(blockIdx.y) * per + int(threadIdx.x); i < i1; i += APPEND_THREADS) {
        if (i < ROW_VEC) {
            cache[(size_t(b) * size_t(pitch) + size_t(pos)) * ROW_VEC + i] = rows[size_t(b) * ROW_VEC + i];
        } else {
            const int j = i - ROW_VEC;
            const uint4 v = q[size_t(b) * QUERY_VEC + j];
            ring[(size_t(b) * g + slot) * QUERY_VEC + j] = v;
            if (q_dst) q_dst[size_t(b) * QUERY_VEC + j] = v;
        }
    }
}

}  // namespace lca
