// prep_combine.cuh -- summary-query fold ahead of the split-L attention
//  (the log-sum-exp combine is fused with W_UV in wuv_gemm.cuh):
//  * (关键设计 1: the summary query is the mean of the last
//    g queries; the importance of token i is the head-mean of its scaled
//    logits, which is linear in the query, so it folds into one 576-vector
//    u = scale/(H*g) * sum_t sum_h q_{t,h} and s_i = u . row_i).
#pragma once
#include "common.cuh"

namespace lca {

// u[b][576] fp32 and its bf16 hi/lo split uhl[b][2][576] (u = hi + lo to
// ~2^-17 relative), used by the tensor-core importance pass.
// Grid (B, 9): a block sums 64 columns over the g*16 (t, h) query rows with
// 4 row-slices per column, then combines the slices through shared memory.
__global__ void __launch_bounds__(256) prep_summary_kernel(const uint16_t *__restrict__ q_recent,
                                                           int g, float coef, float *__restrict__ u,
                                                           uint16_t *__restrict__ uhl)
{
    __shared__ float part[4][64];
    const int b = blockIdx.x;
    const int col = blockIdx.y * 64 + (threadIdx.x & 63);
    const int slice = threadIdx.x >> 6;
    const int rows = g * LCA_HEADS;
    const uint16_t *base = q_recent + size_t(b) * rows * LCA_D + col;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int r = slice;
    for (; r + 12 < rows; r += 16) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
            acc[e] += __uint_as_float(uint32_t(__ldg(base + size_t(r + 4 * e) * LCA_D)) << 16);
    }
    for (; r < rows; r += 4) acc[0] += __uint_as_float(uint32_t(__ldg(base + size_t(r) * LCA_D)) << 16);
    part[slice][threadIdx.x & 63] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    __syncthreads();
    if (slice == 0) {
        const int c = threadIdx.x;
        const float uu = ((part[0][c] + part[1][c]) + (part[2][c] + part[3][c])) * coef;
        u[size_t(b) * LCA_D + col] = uu;
        const __nv_bfloat16 hi = __float2bfloat16_rn(uu);
        const __nv_bfloat16 lo = __float2bfloat16_rn(uu - __bfloat162float(hi));
        uhl[(size_t(b) * 2 + 0) * LCA_D + col] = __bfloat16_as_ushort(hi);
        uhl[(size_t(b) * 2 + 1) * LCA_D + col] = __bfloat16_as_ushort(lo);
    }
}

}  // namespace lca
