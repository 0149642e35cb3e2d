// prep_combine.cuh -- the two small kernels around the split-L attention:
//  * summary-query fold (关键设计 1: the summary query is the mean of the last
//    g queries; the importance of token i is the head-mean of its scaled
//    logits, which is linear in the query, so it folds into one 576-vector
//    u = scale/(H*g) * sum_t sum_h q_{t,h} and s_i = u . row_i);
//  * log-sum-exp combine of the per-CTA partial attention outputs.
#pragma once
#include "common.cuh"

namespace lca {

// u[b][576] fp32 and its bf16 hi/lo split uhl[b][2][576] (u = hi + lo to
// ~2^-17 relative), used by the tensor-core importance pass.
__global__ void __launch_bounds__(192) prep_summary_kernel(const uint16_t *__restrict__ q_recent,
                                                           int g, float coef, float *__restrict__ u,
                                                           uint16_t *__restrict__ uhl)
{
    const int b = blockIdx.x;
    const uint16_t *base = q_recent + size_t(b) * g * LCA_HEADS * LCA_D;
    for (int d = threadIdx.x; d < LCA_D; d += blockDim.x) {
        float acc = 0.f;
        for (int t = 0; t < g; ++t)
#pragma unroll
            for (int h = 0; h < LCA_HEADS; ++h)
                acc += __uint_as_float(uint32_t(base[(size_t(t) * LCA_HEADS + h) * LCA_D + d]) << 16);
        const float uu = acc * coef;
        u[size_t(b) * LCA_D + d] = uu;
        const __nv_bfloat16 hi = __float2bfloat16_rn(uu);
        const __nv_bfloat16 lo = __float2bfloat16_rn(uu - __bfloat162float(hi));
        uhl[(size_t(b) * 2 + 0) * LCA_D + d] = __bfloat16_as_ushort(hi);
        uhl[(size_t(b) * 2 + 1) * LCA_D + d] = __bfloat16_as_ushort(lo);
    }
}

// Partials of sequence b live in slots c + b for the CTAs c that own its
// tiles.  part_o [slot][16][512] holds sum_r 2^(x_r - m) c_r, part_ml
// [slot][16][2] holds (m, sum_r 2^(x_r - m)) with x in log2 units.
__global__ void __launch_bounds__(128) combine_kernel(const float *__restrict__ part_o,
                                                      const float *__restrict__ part_ml,
                                                      int n_tiles, int64_t T, int G,
                                                      float *__restrict__ o_lat,
                                                      uint16_t *__restrict__ o_bf16)
{
    const int b = blockIdx.x, h = blockIdx.y;
    const int c0 = split_owner(int64_t(b) * n_tiles, T, G);
    const int c1 = split_owner(int64_t(b + 1) * n_tiles - 1, T, G);
    float M = -INFINITY;
    for (int c = c0; c <= c1; ++c) M = fmaxf(M, part_ml[(size_t(c + b) * LCA_HEADS + h) * 2]);
    float den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = c0; c <= c1; ++c) {
        const size_t sl = size_t(c + b) * LCA_HEADS + h;
        const float wgt = exp2f(part_ml[sl * 2] - M);
        den += wgt * part_ml[sl * 2 + 1];
        const float4 o = reinterpret_cast<const float4 *>(part_o + sl * LCA_DC)[threadIdx.x];
        acc.x += wgt * o.x;
        acc.y += wgt * o.y;
        acc.z += wgt * o.z;
        acc.w += wgt * o.w;
    }
    const float inv = 1.f / den;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    const size_t row = (size_t(b) * LCA_HEADS + h) * LCA_DC;
    if (o_lat) reinterpret_cast<float4 *>(o_lat + row)[threadIdx.x] = acc;
    uint2 pk;
    pk.x = pack_bf16(acc.x, acc.y);
    pk.y = pack_bf16(acc.z, acc.w);
    reinterpret_cast<uint2 *>(o_bf16 + row)[threadIdx.x] = pk;
}

}  // namespace lca
