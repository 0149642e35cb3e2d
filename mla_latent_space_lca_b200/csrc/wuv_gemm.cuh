// wuv_gemm.cuh -- per-head value up-projection out[r,h,:] = o_lat[r,h,:] . W_UV[h]
// as a dense bf16 GEMM on tcgen05 tensor cores (fp32 accumulate in TMEM).
//
// One CTA computes a [128 rows x 128] tile of one head: A = o_lat rows of
// head h (bf16 [R][16][512], TMA box {64, 1, 128}, K-major, 128-byte swizzle),
// B = W_UV[h] ([512][128], TMA boxes {64, 64, 1}, N-contiguous = MN-major),
// K = 512 in 8 chunks of 64 through a 4-stage TMA ring.  Rows past R are
// zero-filled by TMA and never stored.
#pragma once
#include "common.cuh"

namespace lca {

constexpr int GM_STAGES = 4;
constexpr int GM_A = 128 * 128;            // 16 KB: [128 rows x 64 k] bf16
constexpr int GM_B = 2 * 64 * 128;         // 16 KB: 2 x [64 k x 64 n] bf16
constexpr int GM_STAGE = GM_A + GM_B;
constexpr int GM_OFF_BAR = GM_STAGES * GM_STAGE;   // 131072
constexpr int GM_SMEM = GM_OFF_BAR + 256;
constexpr int GM_SMEM_ALLOC = GM_SMEM + 1024;
constexpr uint32_t GM_TM_COLS = 128;

__global__ void __launch_bounds__(128, 1)
    wuv_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    float *__restrict__ out, int64_t R)
{
    extern __shared__ uint8_t gm_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(gm_smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x, h = blockIdx.y;

    auto full = [&](int s) -> uint32_t { return sbase + GM_OFF_BAR + 8 * s; };
    auto empty = [&](int s) -> uint32_t { return sbase + GM_OFF_BAR + 8 * (GM_STAGES + s); };
    const uint32_t accf = sbase + GM_OFF_BAR + 8 * (2 * GM_STAGES);
    const uint32_t drain = accf + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + GM_OFF_BAR + 128);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + GM_OFF_BAR + 132);

    if (threadIdx.x == 0) {
        for (int s = 0; s < GM_STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), GM_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr int KC = LCA_DC / 64;   // 8 k-chunks

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&map_a);
        prefetch_tensormap(&map_b);
        const uint64_t pa = policy_evict_first(), pb = policy_evict_last();
        int last[GM_STAGES] = {-1, -1, -1, -1};
        for (int kc = 0; kc < KC; ++kc) {
            const int s = kc % GM_STAGES;
            if (!mbar_wait(empty(s), ((kc / GM_STAGES) & 1) ^ 1, abort_flag, K_GEMM, 1)) break;
            mbar_expect_tx(full(s), GM_STAGE);
            const uint32_t st = sbase + s * GM_STAGE;
            tma_load_3d(st, &map_a, full(s), 64 * kc, h, mt * 128, pa);
            tma_load_3d(st + GM_A, &map_b, full(s), 0, 64 * kc, h, pb);
            tma_load_3d(st + GM_A + 8192, &map_b, full(s), 64, 64 * kc, h, pb);
            last[s] = kc;
        }
        for (int s = 0; s < GM_STAGES; ++s)
            if (last[s] >= 0) mbar_wait(full(s), (last[s] / GM_STAGES) & 1, nullptr, K_GEMM, 2);
    } else if (warp == 1 && lane == 0) {
        constexpr uint32_t IDESC = idesc_bf16(128, 128, 0, 1);
        bool ok = true;
        for (int kc = 0; kc < KC && ok; ++kc) {
            const int s = kc % GM_STAGES;
            if (!mbar_wait(full(s), (kc / GM_STAGES) & 1, abort_flag, K_GEMM, 3)) { ok = false; break; }
            tc_fence_after();
            const uint32_t st = sbase + s * GM_STAGE;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sdesc_sw128(st + ks * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(st + GM_A + ks * 2048, 8192, 1024);
                mma_ss(tmem, ad, bd, IDESC, (kc | ks) ? 1u : 0u);
            }
            tc_commit(empty(s));
        }
        if (ok) tc_commit(accf);
        tc_commit(drain);
        mbar_wait(drain, 0, nullptr, K_GEMM, 4);
    }
    __syncwarp();

    // epilogue: lane = row within the tile, 128 fp32 columns per row
    bool ok = mbar_wait(accf, 0, abort_flag, K_GEMM, 5);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        tc_fence_after();
        const int64_t row = int64_t(mt) * 128 + 32 * warp + lane;
        const uint32_t ta = tmem + (uint32_t(32 * warp) << 16);
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            float v[32];
            tmem_ld32(ta + 32 * cc, v);
            if (row < R) {
                float4 *dst = reinterpret_cast<float4 *>(out + (size_t(row) * LCA_HEADS + h) * LCA_DV + 32 * cc);
#pragma unroll
                for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, GM_TM_COLS);
}


// ------------------------------------------------------------------------
// Decode tail, fused: log-sum-exp combine of the split-L partials and the
// W_UV up-projection in one kernel, swap-AB so the tensor-core M dimension is
// the 128 output columns:  out^T[128 x nb] = W_UV[h]^T[128 x 512] * o^T[512 x nb].
// Grid (16 heads, ceil(B/64)); 128 threads.  W_UV[h] (128 KB, MN-major A) is
// TMA-loaded at entry while the warps combine the partials of their batch
// rows straight into the K-major B operand in shared memory (bf16).
constexpr int CW_ROWS = 64;                       // batch rows per CTA
constexpr int CW_A = LCA_DC * LCA_DV * 2;         // 131072 B: W_UV[h]
constexpr int CW_BCHUNK = CW_ROWS * 128;          // 8192 B per 64-k chunk
constexpr int CW_OFF_B = CW_A;
constexpr int CW_OFF_BAR = CW_OFF_B + 8 * CW_BCHUNK;      // 196608
constexpr int CW_SMEM = CW_OFF_BAR + 256;
constexpr int CW_SMEM_ALLOC = CW_SMEM + 1024;

__global__ void __launch_bounds__(128, 1)
    combine_wuv_kernel(const __grid_constant__ CUtensorMap map_w, const float *__restrict__ part_o,
                       const float *__restrict__ part_ml, int B, int n_tiles, int64_t T, int G,
                       float *__restrict__ o_lat, float *__restrict__ out)
{
    extern __shared__ uint8_t cw_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(cw_smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x;
    const int b0 = blockIdx.y * CW_ROWS;
    const int nb = min(CW_ROWS, B - b0);
    const int nb16 = (nb + 15) & ~15;
    const uint32_t wfull = sbase + CW_OFF_BAR, accf = wfull + 8, drain = wfull + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + CW_OFF_BAR + 64);

    if (threadIdx.x == 0) {
        mbar_init(wfull, 1);
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) {
        prefetch_tensormap(&map_w);
        const uint64_t pol = policy_evict_last();
        mbar_expect_tx(wfull, CW_A);
        for (int kc = 0; kc < 8; ++kc)
            for (int nh = 0; nh < 2; ++nh)
                tma_load_3d(sbase + kc * 16384 + nh * 8192, &map_w, wfull, 64 * nh, 64 * kc, h, pol);
    }

    // combine: warp w handles rows w, w+4, ...; lane owns k = 16*lane .. 16*lane+15
    for (int r = warp; r < nb16; r += 4) {
        float o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] = 0.f;
        if (r < nb) {
            const int b = b0 + r;
            const int c0 = split_owner(int64_t(b) * n_tiles, T, G);
            const int c1 = split_owner(int64_t(b + 1) * n_tiles - 1, T, G);
            float M = -INFINITY;
            for (int c = c0; c <= c1; ++c) M = fmaxf(M, part_ml[(size_t(c + b) * LCA_HEADS + h) * 2]);
            float den = 0.f;
            for (int c = c0; c <= c1; ++c) {
                const size_t sl = size_t(c + b) * LCA_HEADS + h;
                const float wgt = exp2f(part_ml[sl * 2] - M);
                den += wgt * part_ml[sl * 2 + 1];
                const float4 *po = reinterpret_cast<const float4 *>(part_o + sl * LCA_DC + 16 * lane);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float4 x = po[v];
                    o[4 * v + 0] = fmaf(wgt, x.x, o[4 * v + 0]);
                    o[4 * v + 1] = fmaf(wgt, x.y, o[4 * v + 1]);
                    o[4 * v + 2] = fmaf(wgt, x.z, o[4 * v + 2]);
                    o[4 * v + 3] = fmaf(wgt, x.w, o[4 * v + 3]);
                }
            }
            const float inv = 1.f / den;
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] *= inv;
            if (o_lat) {
                float4 *dst = reinterpret_cast<float4 *>(o_lat + (size_t(b) * LCA_HEADS + h) * LCA_DC + 16 * lane);
#pragma unroll
                for (int v = 0; v < 4; ++v) dst[v] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
            }
        }
        // K-major SW128 row r of chunk lane/4, 16-byte units 2*(lane%4) and +1
        uint8_t *rowp = smem + CW_OFF_B + (lane >> 2) * CW_BCHUNK + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
            const int unit = 2 * (lane & 3) + hlf;
            uint4 pk;
            pk.x = pack_bf16(o[8 * hlf + 0], o[8 * hlf + 1]);
            pk.y = pack_bf16(o[8 * hlf + 2], o[8 * hlf + 3]);
            pk.z = pack_bf16(o[8 * hlf + 4], o[8 * hlf + 5]);
            pk.w = pack_bf16(o[8 * hlf + 6], o[8 * hlf + 7]);
            *reinterpret_cast<uint4 *>(rowp + ((unit ^ (r & 7)) << 4)) = pk;
        }
    }
    fence_proxy_async();
    __syncthreads();

    if (threadIdx.x == 0) {
        bool ok = mbar_wait(wfull, 0, nullptr, K_GEMM, 11);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, nb16, 1, 0);
#pragma unroll 1
            for (int ks = 0; ks < 32; ++ks) {
                const int kc = ks >> 2, kk = ks & 3;
                const uint64_t ad = sdesc_sw128(sbase + kc * 16384 + kk * 2048, 8192, 1024);
                const uint64_t bd = sdesc_sw128(sbase + CW_OFF_B + kc * CW_BCHUNK + kk * 32, 16, 1024);
                mma_ss(tmem, ad, bd, idesc, ks ? 1u : 0u);
            }
            tc_commit(accf);
        }
        tc_commit(drain);
        mbar_wait(drain, 0, nullptr, K_GEMM, 12);
    }
    __syncwarp();
    bool ok = mbar_wait(accf, 0, nullptr, K_GEMM, 13);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        tc_fence_after();
        const int n = 32 * warp + lane;
        const uint32_t ta = tmem + (uint32_t(32 * warp) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < nb16; c0 += 16) {
            float v[16];
            tmem_ld16(ta + c0, v);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                if (c0 + e < nb) out[(size_t(b0 + c0 + e) * LCA_HEADS + h) * LCA_DV + n] = v[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

}  // namespace lca
