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
// the 128 output columns:  out^T[128 x 16] = W_UV[h]^T[128 x 512] * o^T[512 x 16]
// (N = 16: up to 8 batch rows per CTA, the rest zero).  Grid (16 heads,
// ceil(B/8)); 256 threads.  W_UV[h] (128 KB, MN-major A) is TMA-loaded at
// entry.  Meanwhile, per batch row, the 8 warps split that row's partial
// slots (online max/rescale merge inside a warp, then across warps through
// shared memory) and write the normalised o row as bf16 straight into the
// K-major B operand.
constexpr int CW_ROWS = 8;                        // batch rows per CTA
constexpr int CW_N = 16;                          // MMA N (rows padded)
constexpr int CW_THREADS = 256;
constexpr int CW_A = LCA_DC * LCA_DV * 2;         // 131072 B: W_UV[h]
constexpr int CW_BCHUNK = CW_N * 128;             // 2048 B per 64-k chunk
constexpr int CW_OFF_B = CW_A;                    // 8 chunks = 16 KB
constexpr int CW_OFF_SCR = CW_OFF_B + 8 * CW_BCHUNK;          // 147456
constexpr int CW_SCR = 8 * (LCA_DC + 2) * 4;                  // per-warp (o, M, den)
constexpr int CW_OFF_BAR = CW_OFF_SCR + CW_SCR;
constexpr int CW_SMEM = CW_OFF_BAR + 256;
constexpr int CW_SMEM_ALLOC = CW_SMEM + 1024;

__global__ void __launch_bounds__(CW_THREADS, 1)
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
    const uint32_t wfull = sbase + CW_OFF_BAR, accf = wfull + 8, drain = wfull + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + CW_OFF_BAR + 64);
    float *scr = reinterpret_cast<float *>(smem + CW_OFF_SCR);   // [8][512 + 2]

    if (threadIdx.x == 0) {
        mbar_init(wfull, 1);
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 32);
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

    for (int r = 0; r < CW_N; ++r) {
        float o[2] = {0.f, 0.f};   // merged o for k = 2*threadIdx.x, +1
        if (r < nb) {
            const int b = b0 + r;
            const int c0 = split_owner(int64_t(b) * n_tiles, T, G);
            const int ns = split_owner(int64_t(b + 1) * n_tiles - 1, T, G) - c0 + 1;
            float M = -INFINITY, den = 0.f, acc[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = 0.f;
            for (int sidx = warp; sidx < ns; sidx += 8) {
                const size_t sl = size_t(c0 + sidx + b) * LCA_HEADS + h;
                const float m = part_ml[sl * 2], l = part_ml[sl * 2 + 1];
                const float4 *po = reinterpret_cast<const float4 *>(part_o + sl * LCA_DC + 16 * lane);
                const float4 x0 = po[0], x1 = po[1], x2 = po[2], x3 = po[3];
                if (m > M) {
                    const float sc = exp2f(M - m);   // 0 on the first slot
                    den *= sc;
#pragma unroll
                    for (int e = 0; e < 16; ++e) acc[e] *= sc;
                    M = m;
                }
                const float wgt = exp2f(m - M);
                den = fmaf(wgt, l, den);
                const float xs[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                      x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = fmaf(wgt, xs[e], acc[e]);
            }
            float *my = scr + warp * (LCA_DC + 2);
#pragma unroll
            for (int e = 0; e < 16; ++e) my[16 * lane + e] = acc[e];
            if (lane == 0) {
                my[LCA_DC] = M;
                my[LCA_DC + 1] = den;
            }
            __syncthreads();
            float Mt = -INFINITY;
#pragma unroll
            for (int w8 = 0; w8 < 8; ++w8) Mt = fmaxf(Mt, scr[w8 * (LCA_DC + 2) + LCA_DC]);
            float dt = 0.f;
#pragma unroll
            for (int w8 = 0; w8 < 8; ++w8) {
                const float *wp = scr + w8 * (LCA_DC + 2);
                const float Mw = wp[LCA_DC];
                const float f = (Mw == -INFINITY) ? 0.f : exp2f(Mw - Mt);
                dt = fmaf(f, wp[LCA_DC + 1], dt);
                o[0] = fmaf(f, wp[2 * threadIdx.x], o[0]);
                o[1] = fmaf(f, wp[2 * threadIdx.x + 1], o[1]);
            }
            const float inv = 1.f / dt;
            o[0] *= inv;
            o[1] *= inv;
            if (o_lat)
                *reinterpret_cast<float2 *>(o_lat + (size_t(b) * LCA_HEADS + h) * LCA_DC + 2 * threadIdx.x) =
                    make_float2(o[0], o[1]);
        }
        // row r of the K-major SW128 B operand: k = 2*tid -> chunk k/64, byte (k%64)*2
        {
            const int k = 2 * threadIdx.x;
            const int unit = (k & 63) >> 3, within = (k & 7) * 2;
            uint8_t *rowp = smem + CW_OFF_B + (k >> 6) * CW_BCHUNK + (r >> 3) * 1024 + (r & 7) * 128;
            *reinterpret_cast<uint32_t *>(rowp + ((unit ^ (r & 7)) << 4) + within) = pack_bf16(o[0], o[1]);
        }
        __syncthreads();
    }
    fence_proxy_async();
    __syncthreads();

    if (threadIdx.x == 0) {
        if (mbar_wait(wfull, 0, nullptr, K_GEMM, 11)) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, CW_N, 1, 0);
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
    if (warp < 4) {
        bool ok = mbar_wait(accf, 0, nullptr, K_GEMM, 13);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const int n = 32 * warp + lane;
            float v[16];
            tmem_ld16(tmem + (uint32_t(32 * warp) << 16), v);
#pragma unroll
            for (int e = 0; e < CW_ROWS; ++e)
                if (e < nb) out[(size_t(b0 + e) * LCA_HEADS + h) * LCA_DV + n] = v[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 32);
}

}  // namespace lca
