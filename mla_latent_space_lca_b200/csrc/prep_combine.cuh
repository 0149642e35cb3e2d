// prep_combine.cuh -- summary-query fold ahead of the split-L attention
//  (the log-sum-exp combine is fused with W_UV in wuv_gemm.cuh):
//  * (关键设计 1: the summary query is the mean of the last
//    g queries; the importance of token i is the head-mean of its scaled
//    logits, which is linear in the query, so it folds into one 576-vector
//    u = scale/(H*g) * sum_t sum_h q_{t,h} and s_i = u . row_i).
#pragma once
#include "common.cuh"

namespace lca {

// u[b][576] fp32 (skipped when u is NULL) and its bf16 hi/lo split
// uhl[b][2][576] (u = hi + lo to ~2^-17 relative), used by the tensor-core
// importance pass.  Unit b reads the g*16 query rows starting at
// q_recent + (b / nbs) * seq_stride + (b % nbs) * g*16*576: decode has one
// unit per sequence (nbs = 1), blockwise prefill one per block of g queries.
// Grid (units, 9): a block owns 64 columns of one unit; its 256 threads are
// 8 column groups (16-byte loads) x 32 row slices of the g*16 (t, h) query
// rows, with all of a thread's loads in flight at once (one round trip for
// g = 16), reduced by shuffles within a warp and through 2 KB of shared
// memory across the 8 warps.
//
// Ordering: every CTA first waits for its predecessor in the stream (whose
// output may be q_recent, or the cache row of the current token) and only
// then lets its dependent (the attention or condense kernel) launch.  So the
// dependent launches only once everything earlier in the stream has
// completed: it may stream the cache at once, overlapping this kernel, and
// waits for this grid to complete only before it reads u.  The dependent
// cannot launch before every CTA of this grid has triggered, so it never
// starves this grid of an SM.
constexpr int PREP_THREADS = 256;

__global__ void __launch_bounds__(PREP_THREADS) prep_summary_kernel(const uint16_t *__restrict__ q_recent,
                                                                    int g, int nbs, int64_t seq_stride,
                                                                    float coef, float *__restrict__ u,
                                                                    uint16_t *__restrict__ uhl)
{
    __shared__ float part[8][64];
    griddep_wait();
    griddep_launch_dependents();
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cg = threadIdx.x & 7, sl = threadIdx.x >> 3;   // 32 slices
    const int col0 = blockIdx.y * 64 + 8 * cg;
    const int rows = g * LCA_HEADS;
    const uint16_t *base =
        q_recent + size_t(b / nbs) * size_t(seq_stride) + size_t(b % nbs) * rows * LCA_D + col0;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int r0 = sl; r0 < rows; r0 += 32 * 8) {
        uint4 x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int r = r0 + 32 * e;
            x[e] = (r < rows) ? __ldg(reinterpret_cast<const uint4 *>(base + size_t(r) * LCA_D))
                              : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            acc[0] += bf_lo(x[e].x); acc[1] += bf_hi(x[e].x);
            acc[2] += bf_lo(x[e].y); acc[3] += bf_hi(x[e].y);
            acc[4] += bf_lo(x[e].z); acc[5] += bf_hi(x[e].z);
            acc[6] += bf_lo(x[e].w); acc[7] += bf_hi(x[e].w);
        }
    }
    // the warp's 4 slices of each column group (lane bits 3 and 4)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    }
    if (lane < 8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) part[warp][8 * lane + e] = acc[e];
    }
    __syncthreads();
    if (threadIdx.x < 64) {
        const int c = threadIdx.x;
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += part[w][c];
        const int col = blockIdx.y * 64 + c;
        const float uu = t * coef;
        if (u) u[size_t(b) * LCA_D + col] = uu;
        const __nv_bfloat16 hi = __float2bfloat16_rn(uu);
        const __nv_bfloat16 lo = __float2bfloat16_rn(uu - __bfloat162float(hi));
        uhl[(size_t(b) * 2 + 0) * LCA_D + col] = __bfloat16_as_ushort(hi);
        uhl[(size_t(b) * 2 + 1) * LCA_D + col] = __bfloat16_as_ushort(lo);
    }
}

}  // namespace lca
