// condense.cuh -- streaming LCA condensation (关键设计 1 and 2) that writes
// representatives to memory in cache-row format.
//
// One warp condenses one group of 16 tokens at a time.  The group is one
// contiguous 18 KB span of the cache ([16 rows x 1152 B]), copied into the
// warp's own shared-memory slot by cp.async.bulk with an L2 evict-first hint;
// twelve warps per CTA (three per scheduler) keep ~216 KB per SM in flight
// while the cache streams through once.  Per group, from shared memory:
//   s_i   = u . row_i           (u = folded summary query, fp32 FMA, held in
//                                registers; lanes own 16-byte column slices,
//                                36 of the 16 x 72 per lane, and a halving
//                                shuffle transpose sums the 16 dots so that
//                                lanes 2t, 2t+1 end up with token t)
//   alpha = softmax(s)          (shuffle max / sum over the 16 tokens)
//   I     = first argmax s      (shuffle reduction on (s, index))
//   rep   = [sum_i alpha_i c_i (fp32 accumulate, bf16 store) | k^R_I (bit copy)]
// The ablations of the page's 消融实验 table replace the last step:
// LCA_VARIANT_POOL_POSITION pools k^R with the same alpha too, and
// LCA_VARIANT_SPARSE stores the anchor token's whole row.
#pragma once
#include "common.cuh"

namespace lca {

// Each warp owns S group slots and issues its own copies, so no slot
// is ever shared between warps.  The per-group arithmetic is a chain of
// dependent shared-memory loads, FMAs and shuffles; one warp per scheduler
// cannot hide its latency, so a CTA runs several warps per scheduler.
template <int W, int S>
struct CondenseShape {
    static constexpr int kWarps = W;
    static constexpr int kSlots = S;
    static constexpr int kGroupBytes = 16 * LCA_D * 2;                          // 18432
    static constexpr int kSmem = W * S * kGroupBytes + W * S * 8;
};
constexpr int CD_GROUP_BYTES = 16 * LCA_D * 2;
using CdShape = CondenseShape<12, 1>;    // the shape the library launches

struct CondenseArgs {
    const uint16_t *cache;   // [B][pitch][576], rows 0 .. L-1 of each sequence used
    const float *u;          // [B][576]
    int64_t pitch;           // rows between consecutive sequences
    int64_t m;               // groups condensed per sequence: j0 .. j0+m-1
    int64_t j0;              // first group
    int64_t stride;          // rows per sequence of rep / anchor / alpha
    int64_t total;           // B * m
    uint16_t *rep;           // [B][stride][576], rows j0 .. j0+m-1 written
    int32_t *anchor;         // [B][stride] or NULL
    float *alpha;            // [B][stride][16] or NULL
    int variant;             // LCA_VARIANT_*: the method or one of its ablations
};

// acc + x . u over one 16-byte slice (8 bf16) of a row
__device__ __forceinline__ float dot8(const uint4 x, const float *u, float acc)
{
    acc = fmaf(bf_lo(x.x), u[0], acc);
    acc = fmaf(bf_hi(x.x), u[1], acc);
    acc = fmaf(bf_lo(x.y), u[2], acc);
    acc = fmaf(bf_hi(x.y), u[3], acc);
    acc = fmaf(bf_lo(x.z), u[4], acc);
    acc = fmaf(bf_hi(x.z), u[5], acc);
    acc = fmaf(bf_lo(x.w), u[6], acc);
    acc = fmaf(bf_hi(x.w), u[7], acc);
    return acc;
}

__device__ __forceinline__ void load_u8(const float *p, float *uu)
{
    const float4 x0 = __ldg(reinterpret_cast<const float4 *>(p)), x1 = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    uu[0] = x0.x, uu[1] = x0.y, uu[2] = x0.z, uu[3] = x0.w;
    uu[4] = x1.x, uu[5] = x1.y, uu[6] = x1.z, uu[7] = x1.w;
}

template <int W, int S>
__global__ void __launch_bounds__(W * 32, 1) condense_kernel(const CondenseArgs a)
{
    using Shape = CondenseShape<W, S>;
    extern __shared__ __align__(128) uint8_t cd_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *ring = cd_smem + size_t(warp) * S * CD_GROUP_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(cd_smem + W * S * CD_GROUP_BYTES) + warp * S;
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(smem_u32(&bars[s]), 1);
        fence_mbar_init();
    }
    __syncwarp();
    static_assert(Shape::kSmem <= 227 * 1024, "slots exceed shared memory");

    const int64_t nw = int64_t(gridDim.x) * W;
    const int64_t gw = int64_t(blockIdx.x) * W + warp;
    const uint64_t pol = policy_evict_first();

    auto issue = [&](int64_t gi, int s) {
        const int64_t b = gi / a.m, j = a.j0 + (gi - b * a.m);
        const uint16_t *src = a.cache + (size_t(b) * a.pitch + size_t(j) * 16) * LCA_D;
        const uint32_t bar = smem_u32(&bars[s]);
        mbar_expect_tx(bar, CD_GROUP_BYTES);
        bulk_load(smem_u32(ring + s * CD_GROUP_BYTES), src, CD_GROUP_BYTES, bar, pol);
    };

    // The library launches this kernel right after the summary-query fold,
    // which lets it launch only once everything before that fold in the
    // stream has completed: the cache rows are final, so the first copies go
    // out at once; u (the fold's output) is read only after the wait below.
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const int64_t gi = gw + s * nw;
            if (gi < a.total) issue(gi, s);
        }
    }
    griddep_wait();

    // this lane's 16-byte column slices of u: lane, lane + 32 (for all 16
    // rows) and 64 + lane % 8 (for rows 4 (lane / 8) .. + 3), so that the
    // 16 x 72 slices of a group split evenly, 36 per lane
    float u0[8], u1[8], u2[8];
    int64_t ub = -1;
    const int xrow = 4 * (lane >> 3), xslice = 64 + (lane & 7);

    bool ok = true;
    int it = 0;
    for (int64_t gi = gw; gi < a.total; gi += nw, ++it) {
        const int s = it % S;
        ok = mbar_wait(smem_u32(&bars[s]), (it / S) & 1, nullptr, K_CONDENSE, 1);
        if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
        }
        const int64_t b = gi / a.m, j = a.j0 + (gi - b * a.m);
        const uint8_t *tile = ring + s * CD_GROUP_BYTES;
        if (b != ub) {
            const float *ur = a.u + size_t(b) * LCA_D;
            load_u8(ur + 8 * lane, u0);
            load_u8(ur + 8 * (lane + 32), u1);
            load_u8(ur + 8 * xslice, u2);
            ub = b;
        }

        // importance: partial dots of the 16 rows over this lane's slices
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint8_t *row = tile + i * (LCA_D * 2);
            acc[i] = dot8(*reinterpret_cast<const uint4 *>(row + lane * 16), u0, 0.f);
            acc[i] = dot8(*reinterpret_cast<const uint4 *>(row + (lane + 32) * 16), u1, acc[i]);
        }
        {
            float e[4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
                e[t] = dot8(*reinterpret_cast<const uint4 *>(tile + (xrow + t) * (LCA_D * 2) + xslice * 16), u2, 0.f);
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] += ((i >> 2) == (lane >> 3)) ? e[i & 3] : 0.f;
        }
        // halving transpose-reduce: after it lanes 2t and 2t+1 hold token t
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const bool up = lane & 16;
            const float send = up ? acc[k] : acc[k + 8];
            const float keep = up ? acc[k + 8] : acc[k];
            acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const bool up = lane & 8;
            const float send = up ? acc[k] : acc[k + 4];
            const float keep = up ? acc[k + 4] : acc[k];
            acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const bool up = lane & 4;
            const float send = up ? acc[k] : acc[k + 2];
            const float keep = up ? acc[k + 2] : acc[k];
            acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        }
        {
            const bool up = lane & 2;
            const float send = up ? acc[0] : acc[1];
            const float keep = up ? acc[1] : acc[0];
            acc[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
        }
        const float sc = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 1);
        const int tok = lane >> 1;

        // group max and first-index argmax
        float best = sc;
        int bi = tok;
#pragma unroll
        for (int off = 2; off <= 16; off <<= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ob > best || (ob == best && oi < bi)) {
                best = ob;
                bi = oi;
            }
        }
        const float e = fast_exp2((sc - best) * kLog2e);
        float den = e;
#pragma unroll
        for (int off = 2; off <= 16; off <<= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
        const float al = e / den;

        uint16_t *dst = a.rep + (size_t(b) * a.stride + size_t(j)) * LCA_D;
        const uint8_t *arow = tile + bi * (LCA_D * 2);   // the anchor token's row
        if (a.variant == LCA_VARIANT_SPARSE) {
            // ablation "纯稀疏": the representative is the anchor token's row
#pragma unroll
            for (int r = 0; r < 2; ++r)
                reinterpret_cast<uint4 *>(dst)[lane + 32 * r] = *reinterpret_cast<const uint4 *>(arow + (lane + 32 * r) * 16);
            if (lane < 8)
                reinterpret_cast<uint4 *>(dst + LCA_DC)[lane] = *reinterpret_cast<const uint4 *>(arow + LCA_DC * 2 + lane * 16);
        } else {
            // pooled latent: lane owns 16-byte slices lane and lane+32 of c;
            // with LCA_VARIANT_POOL_POSITION lanes 0-7 also pool slice 64+lane (k^R)
            const bool pool_key = a.variant == LCA_VARIANT_POOL_POSITION;
            float pa[3][8];
#pragma unroll
            for (int r = 0; r < 3; ++r)
#pragma unroll
                for (int k = 0; k < 8; ++k) pa[r][k] = 0.f;
#pragma unroll 4
            for (int i = 0; i < 16; ++i) {
                const float ai = __shfl_sync(0xffffffffu, al, 2 * i);
                const uint8_t *row = tile + i * (LCA_D * 2);
#pragma unroll
                for (int r = 0; r < 3; ++r) {
                    if (r == 2 && !(pool_key && lane < 8)) continue;
                    const uint4 x = *reinterpret_cast<const uint4 *>(row + (lane + 32 * r) * 16);
                    pa[r][0] = fmaf(ai, bf_lo(x.x), pa[r][0]);
                    pa[r][1] = fmaf(ai, bf_hi(x.x), pa[r][1]);
                    pa[r][2] = fmaf(ai, bf_lo(x.y), pa[r][2]);
                    pa[r][3] = fmaf(ai, bf_hi(x.y), pa[r][3]);
                    pa[r][4] = fmaf(ai, bf_lo(x.z), pa[r][4]);
                    pa[r][5] = fmaf(ai, bf_hi(x.z), pa[r][5]);
                    pa[r][6] = fmaf(ai, bf_lo(x.w), pa[r][6]);
                    pa[r][7] = fmaf(ai, bf_hi(x.w), pa[r][7]);
                }
            }
#pragma unroll
            for (int r = 0; r < 3; ++r) {
                if (r == 2 && !(pool_key && lane < 8)) continue;
                uint4 o;
                o.x = pack_bf16(pa[r][0], pa[r][1]);
                o.y = pack_bf16(pa[r][2], pa[r][3]);
                o.z = pack_bf16(pa[r][4], pa[r][5]);
                o.w = pack_bf16(pa[r][6], pa[r][7]);
                reinterpret_cast<uint4 *>(dst)[lane + 32 * r] = o;
            }
            if (!pool_key && lane < 8)   // 关键设计 2: the anchor's key, bit for bit
                reinterpret_cast<uint4 *>(dst + LCA_DC)[lane] = *reinterpret_cast<const uint4 *>(arow + LCA_DC * 2 + lane * 16);
        }
        const size_t gidx = size_t(b) * a.stride + size_t(j);
        if (a.anchor && lane == 0) a.anchor[gidx] = int32_t(j * 16 + bi);
        if (a.alpha && (lane & 1) == 0) a.alpha[gidx * 16 + tok] = al;

        // release the slot and refill it
        __syncwarp();
        if (lane == 0) {
            const int64_t nxt = gi + S * nw;
            if (nxt < a.total) {
                fence_proxy_async();
                issue(nxt, s);
            }
        }
    }
    if (!ok && lane == 0) {
        // a wait expired at item `it`: items 0 .. it - 1 + S of this warp had
        // been issued; let the last one of each slot land before exiting
        const int64_t n = (a.total - gw + nw - 1) / nw;
        const int64_t hi = min64(int64_t(it) - 1 + S, n - 1);
        for (int s = 0; s < S; ++s) {
            if (hi < s) continue;
            const int64_t i = hi - (hi - s) % S;
            mbar_wait(smem_u32(&bars[s]), uint32_t(i / S) & 1u, nullptr, K_CONDENSE, 2);
        }
    }
}

}  // namespace lca
