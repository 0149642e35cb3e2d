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
// per-head W_UV up-projection, swap-AB so the tensor-core M dimension is the
// 128 output columns:
//   out^T[128 x 16] = W_UV[h]^T[128 x 512] * o^T[512 x 16]
// (N = 16: up to 8 batch rows per CTA, the rest zero).  Grid (16 heads,
// ceil(B/rpc)), 256 threads, rpc rows per CTA chosen by the host so that the
// grid fills the GPU (fewer rows per CTA = more warps per row's slots).  W_UV[h] (128 KB, MN-major A) is TMA-loaded before
// waiting on the attention kernel.  Combine: with nb rows, each row gets
// 8/nb warps (at least one); a warp merges its share of the row's partial
// slots online (rescaling on a new maximum, lanes own 16 of the 512 columns),
// and the warps of a row are merged through shared memory into the bf16
// K-major B operand.  K = 512 runs as four MMA chains of 8 k-steps, each on
// its own issuing thread and TMEM accumulator; the epilogue sums them.
//
// Two further uses serve a decode split along L across devices:
//  - out == NULL skips W_UV: the kernel only merges the slots, writes the
//    normalised o (o_lat) and, through lse_out, each row's base-2
//    log-sum-exp M + log2(den) -- one shard's partial;
//  - n_shards > 0 reads n_shards such partials instead of the split-L
//    workspace: record s starts at part_o + s * shard_stride and holds o
//    [B][16][512] followed by lse2 [B][16] (part_ml is unused); each acts as
//    a slot with maximum lse2 and denominator 1.
// For a ragged batch tile_start (B+1 offsets into the batch's tile list)
// replaces the uniform b * n_tiles.
constexpr int TD_ROWS = 8;
constexpr int TD_N = 16;
constexpr int TD_A = LCA_DC * LCA_DV * 2;               // 131072
constexpr int TD_BCHUNK = TD_N * 128;                   // 2048 per 64-k chunk
constexpr int TD_OFF_B = TD_A;                          // 8 chunks = 16 KB
constexpr int TD_OFF_SCR = TD_OFF_B + 8 * TD_BCHUNK;    // 147456
constexpr int TD_SCR_STRIDE = LCA_DC + 4;               // floats per warp state
constexpr int TD_OFF_COEF = TD_OFF_SCR + 8 * TD_SCR_STRIDE * 4;   // [TD_ROWS][8] warp weights
constexpr int TD_OFF_BAR = TD_OFF_COEF + TD_ROWS * 8 * 4;
constexpr int TD_SMEM = TD_OFF_BAR + 256;
constexpr int TD_SMEM_ALLOC = TD_SMEM + 1024;

__global__ void __launch_bounds__(256, 1)
    tail_decode_kernel(const __grid_constant__ CUtensorMap map_w, const float *__restrict__ part_o,
                       const float *__restrict__ part_ml, int B, int n_tiles, int64_t T, int G,
                       float *__restrict__ o_lat, float *__restrict__ out, int rpc,
                       float *__restrict__ lse_out, int n_shards, int64_t shard_stride,
                       const int32_t *__restrict__ tile_start)
{
    extern __shared__ uint8_t td_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(td_smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x;
    const int b0 = blockIdx.y * rpc;           // rpc <= TD_ROWS rows (sequences) per CTA
    const int nb = min(rpc, B - b0);
    const int wpr = max(1, TD_ROWS / nb);     // warps per row
    const bool gemm = out != nullptr;
    const size_t lse_off = size_t(B) * LCA_HEADS * LCA_DC;   // lse2 within a shard record
    const uint32_t wbar = sbase + TD_OFF_BAR, accf = wbar + 8, drain0 = wbar + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + TD_OFF_BAR + 128);
    float *scr = reinterpret_cast<float *>(smem + TD_OFF_SCR);

    if (threadIdx.x == 0) {
        mbar_init(wbar, 1);
        mbar_init(accf, 4);
        for (int k = 0; k < 4; ++k) mbar_init(drain0 + 8 * k, 1);
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
    if (gemm && threadIdx.x == 0) {
        prefetch_tensormap(&map_w);
        const uint64_t pol = policy_evict_last();
        mbar_expect_tx(wbar, TD_A);
        for (int kc = 0; kc < 8; ++kc)
            for (int nh = 0; nh < 2; ++nh)
                tma_load_3d(sbase + kc * 16384 + nh * 8192, &map_w, wbar, 64 * nh, 64 * kc, h, pol);
    }
    // The slots of this warp's row: known from the arguments alone for an
    // even split (worked out while the attention kernel finishes); a ragged
    // batch's tile list comes from a kernel earlier in the stream and is
    // read after the wait.
    const int r = warp / wpr, sub = warp % wpr;
    int c0 = 0, ns = n_shards;
    int64_t TT = T;
    if (r < nb && !n_shards && !tile_start) {
        c0 = split_owner(int64_t(b0 + r) * n_tiles, T, G);
        ns = split_owner(int64_t(b0 + r + 1) * n_tiles - 1, T, G) - c0 + 1;
    }
    griddep_wait();   // the split-L partials come from the attention kernel
    // Only now may the next kernel (the next step's summary-query fold)
    // start: the attention kernel that read its output buffer has finished.
    griddep_launch_dependents();

    // ---- per-warp merge of its share of one row's slots: the (m, l) pairs of
    // up to 32 slots at a time are read by the lanes, reduced to their max M
    // and sum, and then the slot vectors are accumulated with independent
    // loads (no serial rescaling chain).
    {
        float M = -INFINITY, den = 0.f, acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
        if (r < nb) {
            const int b = b0 + r;
            if (tile_start && !n_shards) {
                TT = tile_start[B];
                c0 = split_owner(int64_t(tile_start[b]), TT, G);
                ns = split_owner(int64_t(tile_start[b + 1]) - 1, TT, G) - c0 + 1;
            }
            const int mine = (ns - sub + wpr - 1) / wpr;   // slots sub, sub+wpr, ...
            auto slot_vec = [&](int k) {   // this lane's 16 floats of the warp's k-th slot
                const int s = sub + wpr * k;
                const float *rec = n_shards ? part_o + size_t(s) * shard_stride + (size_t(b) * LCA_HEADS + h) * LCA_DC
                                            : part_o + (size_t(c0 + s + b) * LCA_HEADS + h) * LCA_DC;
                return reinterpret_cast<const float4 *>(rec + 16 * lane);
            };
            // the first NPRE slot vectors are requested together with the
            // (m, l) pairs: one memory round trip before the first FMAs
            constexpr int NPRE = 4;
            const int npre = min(NPRE, mine);
            float4 pre[NPRE][4];
#pragma unroll
            for (int k = 0; k < NPRE; ++k)
                if (k < npre) {
                    const float4 *po = slot_vec(k);
#pragma unroll
                    for (int v = 0; v < 4; ++v) pre[k][v] = po[v];
                }
            for (int base = 0; base < mine; base += 32) {
                const int cnt = min(32, mine - base);
                float m = -INFINITY, l = 0.f;
                if (lane < cnt) {
                    const int s = sub + wpr * (base + lane);
                    if (n_shards) {
                        m = part_o[size_t(s) * shard_stride + lse_off + size_t(b) * LCA_HEADS + h];
                        l = 1.f;
                    } else if (!tile_start || split_begin(c0 + s + 1, TT, G) > split_begin(c0 + s, TT, G)) {
                        // (a ragged batch can have fewer tiles than CTAs: a CTA
                        // owning none wrote no slot, and its slot is skipped;
                        // an even split gives every CTA a tile)
                        const size_t sl = size_t(c0 + s + b) * LCA_HEADS + h;
                        const float2 ml = *reinterpret_cast<const float2 *>(part_ml + sl * 2);
                        m = ml.x;
                        l = ml.y;
                    }
                }
                float Mc = m;
#pragma unroll
                for (int off = 16; off; off >>= 1) Mc = fmaxf(Mc, __shfl_xor_sync(0xffffffffu, Mc, off));
                if (Mc == -INFINITY) continue;   // every slot of the chunk skipped (warp-uniform)
                const float Mn = fmaxf(M, Mc);
                const float sc = fast_exp2(M - Mn);   // rescale the earlier chunks (0 at first)
                den *= sc;
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] *= sc;
                M = Mn;
                const float wl = (lane < cnt) ? fast_exp2(m - M) : 0.f;
                float dl = wl * l;
#pragma unroll
                for (int off = 16; off; off >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, off);
                den += dl;
                auto accumulate = [&](float wk, const float4 &x0, const float4 &x1, const float4 &x2,
                                      const float4 &x3) {
                    acc[0] = fmaf(wk, x0.x, acc[0]); acc[1] = fmaf(wk, x0.y, acc[1]);
                    acc[2] = fmaf(wk, x0.z, acc[2]); acc[3] = fmaf(wk, x0.w, acc[3]);
                    acc[4] = fmaf(wk, x1.x, acc[4]); acc[5] = fmaf(wk, x1.y, acc[5]);
                    acc[6] = fmaf(wk, x1.z, acc[6]); acc[7] = fmaf(wk, x1.w, acc[7]);
                    acc[8] = fmaf(wk, x2.x, acc[8]); acc[9] = fmaf(wk, x2.y, acc[9]);
                    acc[10] = fmaf(wk, x2.z, acc[10]); acc[11] = fmaf(wk, x2.w, acc[11]);
                    acc[12] = fmaf(wk, x3.x, acc[12]); acc[13] = fmaf(wk, x3.y, acc[13]);
                    acc[14] = fmaf(wk, x3.z, acc[14]); acc[15] = fmaf(wk, x3.w, acc[15]);
                };
                int k0 = 0;
                if (base == 0) {
#pragma unroll
                    for (int k = 0; k < NPRE; ++k) {
                        if (k >= npre) break;
                        const float wk = __shfl_sync(0xffffffffu, wl, k);
                        if (wk != 0.f) accumulate(wk, pre[k][0], pre[k][1], pre[k][2], pre[k][3]);
                    }
                    k0 = npre;
                }
#pragma unroll 4
                for (int k = k0; k < cnt; ++k) {
                    const float wk = __shfl_sync(0xffffffffu, wl, k);
                    if (wk == 0.f) continue;   // warp-uniform: skipped slots contribute nothing
                    const float4 *po = slot_vec(base + k);
                    accumulate(wk, po[0], po[1], po[2], po[3]);
                }
            }
        }
        float *my = scr + warp * TD_SCR_STRIDE;
#pragma unroll
        for (int v = 0; v < 4; ++v)
            *reinterpret_cast<float4 *>(my + 16 * lane + 4 * v) =
                make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
        if (lane == 0) {
            my[LCA_DC] = M;
            my[LCA_DC + 1] = den;
        }
    }
    __syncthreads();
    // ---- per row: the warps' common max, the denominator and each warp's
    // weight (warp r handles row r, lane i the state of warp i of the row)
    float *coef = reinterpret_cast<float *>(smem + TD_OFF_COEF);
    if (warp < nb) {
        const int rr = warp;
        const float *wp = scr + (rr * wpr + (lane & 7)) * TD_SCR_STRIDE;
        const float mi = (lane < wpr) ? wp[LCA_DC] : -INFINITY;
        const float di = (lane < wpr) ? wp[LCA_DC + 1] : 0.f;
        float Mt = mi;
#pragma unroll
        for (int off = 4; off; off >>= 1) Mt = fmaxf(Mt, __shfl_xor_sync(0xffffffffu, Mt, off));
        const float f = (mi == -INFINITY) ? 0.f : fast_exp2(mi - Mt);
        float dt = f * di;
#pragma unroll
        for (int off = 4; off; off >>= 1) dt += __shfl_xor_sync(0xffffffffu, dt, off);
        if (lane < wpr) coef[rr * 8 + lane] = f * (1.f / dt);
        if (lse_out && lane == 0) lse_out[size_t(b0 + rr) * LCA_HEADS + h] = Mt + log2f(dt);
    }
    __syncthreads();
    // ---- merge the warps of each row; o -> o_lat (fp32) and the B operand (bf16)
    // (rows nb .. TD_N-1 of the B operand are left as they are: they only
    // feed output columns that are never stored)
    for (int r = 0; r < nb; ++r) {
        const int k = 2 * threadIdx.x;   // 256 threads x 2 columns
        float o0 = 0.f, o1 = 0.f;
        {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i < wpr) {
                    const float c = coef[r * 8 + i];
                    const float2 x = *reinterpret_cast<const float2 *>(scr + (r * wpr + i) * TD_SCR_STRIDE + k);
                    o0 = fmaf(c, x.x, o0);
                    o1 = fmaf(c, x.y, o1);
                }
            }
            if (o_lat)
                *reinterpret_cast<float2 *>(o_lat + (size_t(b0 + r) * LCA_HEADS + h) * LCA_DC + k) =
                    make_float2(o0, o1);
        }
        const int unit = (k & 63) >> 3, within = (k & 7) * 2;
        uint8_t *rowp = smem + TD_OFF_B + (k >> 6) * TD_BCHUNK + (r >> 3) * 1024 + (r & 7) * 128;
        *reinterpret_cast<uint32_t *>(rowp + ((unit ^ (r & 7)) << 4) + within) = pack_bf16(o0, o1);
    }
    fence_proxy_async();
    __syncthreads();

    if (gemm && warp >= 4 && lane == 0) {
        const int j = warp - 4;   // k-chunks 2j, 2j+1
        if (mbar_wait(wbar, 0, nullptr, K_GEMM, 31)) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, TD_N, 1, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int kc = 2 * j + (kk >> 2), ks = kk & 3;
                const uint64_t ad = sdesc_sw128(sbase + kc * 16384 + ks * 2048, 8192, 1024);
                const uint64_t bd = sdesc_sw128(sbase + TD_OFF_B + kc * TD_BCHUNK + ks * 32, 16, 1024);
                mma_ss(tmem + 16 * j, ad, bd, idesc, kk ? 1u : 0u);
            }
            tc_commit(accf);
        }
        tc_commit(drain0 + 8 * j);
        mbar_wait(drain0 + 8 * j, 0, nullptr, K_GEMM, 32);
    }
    if (gemm && warp < 4) {
        bool ok = mbar_wait(accf, 0, nullptr, K_GEMM, 33);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const int n = 32 * warp + lane;
            const uint32_t ta = tmem + (uint32_t(32 * warp) << 16);
            float v[16], p[16];
            tmem_ld16(ta, v);
#pragma unroll 1
            for (int j = 1; j < 4; ++j) {
                tmem_ld16(ta + 16 * j, p);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] += p[e];
            }
#pragma unroll
            for (int e = 0; e < TD_ROWS; ++e)
                if (e < nb) out[(size_t(b0 + e) * LCA_HEADS + h) * LCA_DV + n] = v[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

}  // namespace lca
