// prefill.cuh -- blockwise LCA prefill on tcgen05 tensor cores.
//
// Queries come in blocks of g = 16 positions; block k (t0 = 16k) condenses
// the history rows 0 .. 16 m_k - 1, m_k = max(0, floor((t0 - w) / 16)), with
// the mean of its own 16 queries as summary query (LCT 关键设计 1, 2), and each
// of its queries t attends [m_k representatives || cache rows 16 m_k .. t]
// causally (整体框架, 关键设计 3).  With g = 16, m_k = max(0, k - cw) where
// cw = ceil(w / 16).  A chunk's representatives are stored group-major,
// rep[j][block], so a condense task writes contiguous runs and the attention
// reads a block's tile of 64 groups as one strided TMA box.
//
// Every block has its own representatives, and one representative tile is
// attended by only 16 queries x 16 heads, so fusing the pooling into the
// attention pass would re-read each raw history row once per block.  Instead
// a chunk of blocks is condensed into a workspace first:
//
//   condense_prefill_kernel: one CTA per (128 blocks, 2 groups = 32 rows),
//     two CTAs per SM.  S [128 blocks x 32 rows] = U_hi * R^T + U_lo * R^T
//     (two MMA chains, M = 128, N = 32, K = 576; u = u_hi + u_lo is the
//     folded summary query in two bf16 halves), a per-lane group softmax /
//     first-index argmax (TMEM lane = block), then the pooling itself on the
//     tensor cores: rep_j [128 blocks x 512] = alpha_j [128 x 16] * C_j [16 x 512]
//     (K = 16, four N = 128 MMAs per group through one TMEM buffer), the
//     anchor's RoPE key copied bit for bit.  Every (group < 2 n_gt, block)
//     entry of the chunk is written, so the rows the attention masks out are
//     finite.  Outputs leave through a per-warp shared-memory transpose, so
//     each store instruction writes whole 256-byte row segments.  Bound: the
//     representative writes (1152 B per block and group).
//
//   attn_prefill_kernel: one CTA per (block, 4 consecutive queries) = 64
//     query rows (query-major, 16 heads each), Q in shared memory.  Per tile
//     of 64 rows (representatives, then window rows):
//       S_c [64 x 64] = Q[:, 144c : +144] * tile[:, 144c : +144]^T, c = 0..3
//         (four K-quarter chains on four issuing warps, SS MMA, M = 64 ->
//         TMEM lanes 0-15 per quadrant; S = sum of the four)
//       O^T[128c .. +127, 64] += tile_lat[:, 128c ..]^T * P^T, c = 0..3
//         (four PV chains, M = 128, N = 64)
//     Online softmax per query row with a reference max moved only when it
//     grows by more than 2^8; causal and ragged-tile masks; the epilogue
//     writes o = O / l as bf16 (the W_UV GEMM's A operand) and optionally fp32.
//     O^T (256 columns) plus the four S partials (256) fill TMEM exactly,
//     which is what caps a CTA at 64 query rows.
#pragma once
#include "common.cuh"

namespace lca {

// 4-D tiled TMA load without an eviction hint, and its L2 prefetch form (a
// box into L2 only: no shared memory, no completion).
__device__ __forceinline__ void tma_load_4d_plain(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y,
                                                  int z, int w)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void pf_prefetch_4d(const CUtensorMap *map, int x, int y, int z, int w)
{
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}

// Representatives of block k.
__host__ __device__ __forceinline__ int64_t pf_groups(int64_t k, int cw) { return k > cw ? k - cw : 0; }

// ====================================================================== condense
// One task = 128 blocks x CP_G groups (16 CP_G history rows); two CTAs share
// an SM, so one CTA's loads, importance MMAs and softmax overlap the other's
// HBM-bound output drains.
constexpr int CP_THREADS = 224;                 // 7 warps
constexpr int CP_G = 2;                         // groups per task
constexpr int CP_ROWS = 16 * CP_G;              // history rows per task
constexpr int CP_BOX = CP_ROWS * 128;           // [CP_ROWS rows x 64 cols] bf16
constexpr int CP_R = 9 * CP_BOX;                // the task's rows, 36 KB
constexpr int CP_UBOX = 16384;                  // [128 blocks x 64 cols] bf16
constexpr int CP_USTAGES = 2;
constexpr int CP_OFF_U = CP_R;                  // U ring; once S is done: alpha + staging
constexpr int CP_OFF_BAR = CP_OFF_U + CP_USTAGES * 2 * CP_UBOX;
constexpr int CP_OFF_MISC = CP_OFF_BAR + 8 * 16;
constexpr int CP_SMEM = CP_OFF_MISC + 64;
constexpr int CP_SMEM_ALLOC = CP_SMEM + 1024;
// after the importance MMAs, the U ring holds: alpha [128 x 64] bf16 (16 KB,
// the first 16 CP_G columns used), then per drain warp 32 rows x 256 B of
// latent and 32 rows x 128 B of RoPE key staging
constexpr int CP_OFF_ALPHA = CP_OFF_U;
constexpr int CP_OFF_STG_LAT = CP_OFF_ALPHA + 16384;
constexpr int CP_OFF_STG_ROPE = CP_OFF_STG_LAT + 4 * 8192;
static_assert(CP_OFF_STG_ROPE + 4 * 4096 <= CP_OFF_U + CP_USTAGES * 2 * CP_UBOX, "staging exceeds the U ring");
static_assert(2 * (CP_SMEM_ALLOC + 1024) <= 228 * 1024, "two CTAs must fit an SM");
constexpr uint32_t CP_TM_S = 0;                 // S_hi, S_lo: CP_ROWS columns each
constexpr uint32_t CP_TM_P = 128;               // one pooling buffer of 128 columns
constexpr uint32_t CP_TM_COLS = 256;

struct CondPreArgs {
    int64_t kc0;       // first block of the chunk (block k = queries 16k .. 16k+15)
    int nbc;           // blocks in the chunk
    int cw;            // ceil(w / 16)
    int b;             // sequence
    int n_gt;          // group tiles (of CP_G groups) per block tile (grid = block tiles x n_gt)
    int ublk0;         // row of block kc0 in the summary-query array
    uint16_t *rep;     // the chunk's representatives, group-major [CP_G n_gt][nbc][576]
    int64_t k0;        // first block of the call (anchor rows)
    int64_t m_ld;      // anchor row length
    int32_t *anchor;   // this sequence's anchor rows [(k - k0)][m_ld], or NULL
    int variant;       // LCA_VARIANT_*: the method or one of its ablations
};

__global__ void __launch_bounds__(CP_THREADS, 2)
    condense_prefill_kernel(const __grid_constant__ CUtensorMap map_rows, const __grid_constant__ CUtensorMap map_u,
                            const CondPreArgs a)
{
    const int bt = blockIdx.x / a.n_gt, gt = blockIdx.x - bt * a.n_gt;
    const int64_t kb0 = a.kc0 + int64_t(bt) * 128;
    const int nblk = min(128, a.nbc - 128 * bt);

    extern __shared__ uint8_t cp_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(cp_smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    auto BAR = [&](int i) -> uint32_t { return sbase + CP_OFF_BAR + 8 * i; };
    const uint32_t rfull = BAR(0), sfull = BAR(5), aready = BAR(6), pfull = BAR(7), pempty = BAR(8),
                   drain5 = BAR(9), drain6 = BAR(10);
    auto ufull = [&](int s) { return BAR(1 + s); };
    auto uempty = [&](int s) { return BAR(3 + s); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + CP_OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + CP_OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(rfull, 1);
        for (int s = 0; s < CP_USTAGES; ++s) {
            mbar_init(ufull(s), 1);
            mbar_init(uempty(s), 2);     // both importance chains
        }
        mbar_init(sfull, 2);
        mbar_init(aready, 4);
        mbar_init(pfull, 1);
        mbar_init(pempty, 4);            // four drain warps
        mbar_init(drain5, 1);
        mbar_init(drain6, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + CP_OFF_MISC, CP_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t rbase = sbase, ubase = sbase + CP_OFF_U, abase = sbase + CP_OFF_ALPHA;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&map_rows);
            prefetch_tensormap(&map_u);
            const uint64_t pol_r = policy_evict_first(), pol_u = policy_evict_last();
            mbar_expect_tx(rfull, CP_R);
#pragma unroll 1
            for (int ch = 0; ch < 9; ++ch)
                tma_load_3d(rbase + ch * CP_BOX, &map_rows, rfull, 64 * ch, CP_ROWS * gt, a.b, pol_r);
            const int ublk = a.ublk0 + 128 * bt;
            int last[CP_USTAGES] = {-1, -1};
#pragma unroll 1
            for (int kb = 0; kb < 9; ++kb) {
                const int s = kb % CP_USTAGES;
                if (!mbar_wait(uempty(s), ((kb / CP_USTAGES) & 1) ^ 1, abort_flag, K_PREFILL_CONDENSE, 1)) break;
                mbar_expect_tx(ufull(s), 2 * CP_UBOX);
                const uint32_t dst = ubase + s * 2 * CP_UBOX;
                tma_load_3d(dst, &map_u, ufull(s), 64 * kb, 0, ublk, pol_u);
                tma_load_3d(dst + CP_UBOX, &map_u, ufull(s), 64 * kb, 1, ublk, pol_u);
                last[s] = kb;
            }
            mbar_wait(rfull, 0, nullptr, K_PREFILL_CONDENSE, 2);
            for (int s = 0; s < CP_USTAGES; ++s)
                if (last[s] >= 0) mbar_wait(ufull(s), (last[s] / CP_USTAGES) & 1, nullptr, K_PREFILL_CONDENSE, 2);
        }
    } else if (warp == 5 || warp == 6) {
        // ------------------------------------------------------------ MMA issuers
        // warp 5: S_hi chain, then the pooling MMAs; warp 6: S_lo chain
        if (lane == 0) {
            const int hl = warp - 5;
            constexpr uint32_t IDESC_S = idesc_bf16(128, CP_ROWS, 0, 0);
            bool ok = mbar_wait(rfull, 0, abort_flag, K_PREFILL_CONDENSE, 3);
#pragma unroll 1
            for (int kb = 0; kb < 9 && ok; ++kb) {
                const int s = kb % CP_USTAGES;
                if (!(ok = mbar_wait(ufull(s), (kb / CP_USTAGES) & 1, abort_flag, K_PREFILL_CONDENSE, 4))) break;
                tc_fence_after();
                const uint32_t ua = ubase + s * 2 * CP_UBOX + hl * CP_UBOX;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + CP_TM_S + CP_ROWS * hl, sdesc_sw128(ua + 32 * ks, 16, 1024),
                           sdesc_sw128(rbase + kb * CP_BOX + 32 * ks, 16, 1024), IDESC_S, (kb | ks) ? 1u : 0u);
                tc_commit(uempty(s));
            }
            if (ok) tc_commit(sfull);
            if (hl == 0 && ok) {
                // rep_j[128 x 128c..] = alpha_j (A, K-major, K = 16 at column 16 jj of
                // the alpha tile) * rows 16 jj.. of the tile (B, MN-major, N = 128
                // spanning boxes 2c and 2c+1); one TMEM buffer, drained in turn
                // (pooled-key ablation: a fifth N = 64 MMA pools the RoPE box)
                constexpr uint32_t IDESC_P = idesc_bf16(128, 128, 0, 1);
                constexpr uint32_t IDESC_PK = idesc_bf16(128, 64, 0, 1);
                const int np = a.variant == LCA_VARIANT_POOL_POSITION ? 5 : 4;
                ok = mbar_wait(aready, 0, abort_flag, K_PREFILL_CONDENSE, 5);
                if (ok) tc_fence_after();
#pragma unroll 1
                for (int idx = 0; idx < np * CP_G && ok; ++idx) {
                    const int jj = idx / np, cc = idx - jj * np;
                    if (!(ok = mbar_wait(pempty, (idx & 1) ^ 1, abort_flag, K_PREFILL_CONDENSE, 6))) break;
                    tc_fence_after();
                    if (cc < 4)
                        mma_ss(tmem + CP_TM_P, sdesc_sw128(abase + 32 * jj, 16, 1024),
                               sdesc_sw128(rbase + 2 * cc * CP_BOX + 2048 * jj, CP_BOX, 1024), IDESC_P, 0u);
                    else
                        mma_ss(tmem + CP_TM_P, sdesc_sw128(abase + 32 * jj, 16, 1024),
                               sdesc_sw128(rbase + 8 * CP_BOX + 2048 * jj, CP_BOX, 1024), IDESC_PK, 0u);
                    tc_commit(pfull);
                }
            }
            const uint32_t dr = hl ? drain6 : drain5;
            tc_commit(dr);
            mbar_wait(dr, 0, nullptr, K_PREFILL_CONDENSE, 7);
        }
    } else {
        // ------------------------------------------------------------ softmax / drain
        const int row = 32 * warp + lane;          // block lane of the tile
        const int64_t k = kb0 + row;
        const bool vblk = row < nblk;
        const int64_t mk = vblk ? pf_groups(k, a.cw) : 0;
        const uint32_t lane_base = uint32_t(32 * warp) << 16;
        int anc[CP_G];
#pragma unroll
        for (int jj = 0; jj < CP_G; ++jj) anc[jj] = 0;
        bool ok = __all_sync(0xffffffffu, mbar_wait(sfull, 0, abort_flag, K_PREFILL_CONDENSE, 8));
        if (ok) {
            tc_fence_after();
            float s[CP_ROWS];
            {
                float v[32];
                tmem_ld32(tmem + lane_base + CP_TM_S, v);
#pragma unroll
                for (int e = 0; e < CP_ROWS; ++e) s[e] = v[e];
                tmem_ld32(tmem + lane_base + CP_TM_S + CP_ROWS, v);
#pragma unroll
                for (int e = 0; e < CP_ROWS; ++e) s[e] += v[e];
            }
            // alpha row of this block, K-major with 128-byte swizzle (the U ring
            // is idle: the importance MMAs have consumed every U stage)
            uint8_t *arow = smem + CP_OFF_ALPHA + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
            for (int jj = 0; jj < CP_G; ++jj) {
                float gm = s[16 * jj];
                int gi = 0;
#pragma unroll
                for (int e = 1; e < 16; ++e)
                    if (s[16 * jj + e] > gm) { gm = s[16 * jj + e]; gi = e; }
                float ex[16], den = 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    ex[e] = fast_exp2((s[16 * jj + e] - gm) * kLog2e);
                    den += ex[e];
                }
                const float inv = 1.f / den;
                // sparse ablation: weight 1 on the anchor (the pooling MMA then
                // reproduces the anchor's latent exactly), 0 elsewhere
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    ex[e] = a.variant == LCA_VARIANT_SPARSE ? (e == gi ? 1.f : 0.f) : ex[e] * inv;
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    uint4 pk;
                    pk.x = pack_bf16(ex[8 * c2 + 0], ex[8 * c2 + 1]);
                    pk.y = pack_bf16(ex[8 * c2 + 2], ex[8 * c2 + 3]);
                    pk.z = pack_bf16(ex[8 * c2 + 4], ex[8 * c2 + 5]);
                    pk.w = pack_bf16(ex[8 * c2 + 6], ex[8 * c2 + 7]);
                    const int c = 2 * jj + c2;
                    *reinterpret_cast<uint4 *>(arow + ((c ^ (row & 7)) << 4)) = pk;
                }
                anc[jj] = gi;
            }
            fence_proxy_async();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(aready);

        // Output rows go through a per-warp staging area so that every store
        // instruction writes whole row segments: lat 32 rows x 256 B (one
        // d-chunk), rope 32 rows x 128 B.
        uint8_t *stg_lat = smem + CP_OFF_STG_LAT + warp * 8192;
        uint8_t *stg_rope = smem + CP_OFF_STG_ROPE + warp * 4096;
        const int64_t kk_warp = int64_t(128) * bt + 32 * warp;   // chunk block of the warp's first lane
        const int hl = lane >> 4, c16 = lane & 15;                // store phase: row 2x + hl, chunk c16
        // representative (group j, chunk block kk) lives in row j nbc + kk
        auto rep_row = [&](int64_t j, int64_t kk) -> size_t { return size_t(j * a.nbc + kk); };

        // anchor keys (bit copies from the tile) and anchor positions; the
        // pooled-key ablation writes its pooled keys with the latents below
        const bool pool_key = a.variant == LCA_VARIANT_POOL_POSITION;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(rfull, 0, abort_flag, K_PREFILL_CONDENSE, 9));
#pragma unroll 1
        for (int jj = 0; jj < CP_G && ok; ++jj) {
            const int64_t j = int64_t(CP_G) * gt + jj;
            if (pool_key) {
                if (a.anchor && vblk && j < mk)
                    a.anchor[size_t(k - a.k0) * size_t(a.m_ld) + size_t(j)] = int32_t(16 * j + anc[jj]);
                continue;
            }
            {
                const int rr = 16 * jj + anc[jj];
                const uint8_t *src = smem + 8 * CP_BOX + rr * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(stg_rope + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                        *reinterpret_cast<const uint4 *>(src + ((c ^ (rr & 7)) << 4));
                if (a.anchor && vblk && j < mk)
                    a.anchor[size_t(k - a.k0) * size_t(a.m_ld) + size_t(j)] = int32_t(16 * j + anc[jj]);
            }
            __syncwarp();
            // 4 rows of 128 B per instruction: lane -> row 4x + lane/8, chunk lane%8
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int rr = 4 * x + (lane >> 3), c = lane & 7;
                if (kk_warp + rr < a.nbc) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(stg_rope + rr * 128 + ((c ^ (rr & 7)) << 4));
                    *reinterpret_cast<uint4 *>(a.rep + rep_row(j, kk_warp + rr) * LCA_D + LCA_DC + 8 * c) = v;
                }
            }
            __syncwarp();
        }

        // drain the pooled latents: group jj, d-chunk cc, one TMEM buffer
        // (cc = 4: the pooled RoPE key of the pooled-key ablation)
        const int np = pool_key ? 5 : 4;
#pragma unroll 1
        for (int idx = 0; idx < np * CP_G && ok; ++idx) {
            const int jj = idx / np, cc = idx - jj * np;
            ok = __all_sync(0xffffffffu, mbar_wait(pfull, idx & 1, abort_flag, K_PREFILL_CONDENSE, 10));
            if (!ok) break;
            tc_fence_after();
            if (cc == 4) {
#pragma unroll 1
                for (int q2 = 0; q2 < 2; ++q2) {   // columns 32 q2 .. 32 q2 + 31
                    float v[32];
                    tmem_ld32(tmem + lane_base + CP_TM_P + 32 * q2, v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 4 * q2 + e;   // 16-byte chunk of the 128-byte row
                        *reinterpret_cast<uint4 *>(stg_rope + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                            make_uint4(pack_bf16(v[8 * e], v[8 * e + 1]), pack_bf16(v[8 * e + 2], v[8 * e + 3]),
                                       pack_bf16(v[8 * e + 4], v[8 * e + 5]), pack_bf16(v[8 * e + 6], v[8 * e + 7]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(pempty);
                const int64_t j = int64_t(CP_G) * gt + jj;
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const int rr = 4 * x + (lane >> 3), c = lane & 7;
                    if (kk_warp + rr < a.nbc) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(stg_rope + rr * 128 + ((c ^ (rr & 7)) << 4));
                        *reinterpret_cast<uint4 *>(a.rep + rep_row(j, kk_warp + rr) * LCA_D + LCA_DC + 8 * c) = v;
                    }
                }
                __syncwarp();
                continue;
            }
#pragma unroll 1
            for (int q4 = 0; q4 < 4; ++q4) {   // columns 32 q4 .. 32 q4 + 31
                float v[32];
                tmem_ld32(tmem + lane_base + CP_TM_P + 32 * q4, v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int cix = 4 * q4 + e;   // 16-byte chunk of the 256-byte row segment
                    *reinterpret_cast<uint4 *>(stg_lat + lane * 256 + ((cix ^ c16) << 4)) =
                        make_uint4(pack_bf16(v[8 * e], v[8 * e + 1]), pack_bf16(v[8 * e + 2], v[8 * e + 3]),
                                   pack_bf16(v[8 * e + 4], v[8 * e + 5]), pack_bf16(v[8 * e + 6], v[8 * e + 7]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pempty);
            const int64_t j = int64_t(CP_G) * gt + jj;
            // 2 rows of 256 B per instruction
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const int rr = 2 * x + hl;
                if (kk_warp + rr < a.nbc) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(stg_lat + rr * 256 + ((c16 ^ (rr & 15)) << 4));
                    *reinterpret_cast<uint4 *>(a.rep + rep_row(j, kk_warp + rr) * LCA_D + 128 * cc + 8 * c16) = v;
                }
            }
            __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, CP_TM_COLS);
}
// ====================================================================== attention
constexpr int AP_THREADS = 416;                 // 13 warps
constexpr int AP_CHUNK = 8192;                  // [64 rows x 64 cols] bf16
constexpr int AP_STAGE = 9 * AP_CHUNK;          // 73728: Q, then two row stages
constexpr int AP_OFF_BAR = 3 * AP_STAGE;
constexpr int AP_OFF_MISC = AP_OFF_BAR + 8 * 20;
constexpr int AP_OFF_FSC = AP_OFF_MISC + 16;    // [2][64] rescale factors
constexpr int AP_OFF_LINV = AP_OFF_FSC + 512;   // [64] 1 / l
constexpr int AP_SMEM = AP_OFF_LINV + 256;
constexpr int AP_SMEM_ALLOC = AP_SMEM + 1024;
constexpr uint32_t AP_TM_S = 0;                 // S partials of the 4 K-quarter chains: 4 x 64 columns
constexpr uint32_t AP_TM_O = 256;               // O^T: 4 d-chunks x 64 columns
constexpr uint32_t AP_TM_COLS = 512;

struct AttnPreArgs {
    int64_t L;
    int b;             // sequence
    int64_t kc0;       // first block of the chunk
    int nbc;           // blocks in the chunk
    int cw;            // ceil(w / 16)
    float sl2;         // scale * log2(e)
    uint16_t *o_bf16;  // chunk rows [(k - kc0) * 16 + tt][16][512]
    float *o_lat;      // the same rows in fp32, or NULL
};

__global__ void __launch_bounds__(AP_THREADS, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap map_cache, const __grid_constant__ CUtensorMap map_q,
                        const __grid_constant__ CUtensorMap map_rep, const AttnPreArgs a)
{
    // heaviest blocks (most representatives) first
    const int blk = a.nbc - 1 - int(blockIdx.x >> 2);
    const int qq = blockIdx.x & 3;
    const int64_t k = a.kc0 + blk;
    const int64_t t_first = 16 * k + 4 * qq;
    const int64_t mk = pf_groups(k, a.cw);
    const int64_t win0 = 16 * mk;
    const int n_rep = int((mk + 63) / 64);
    const int n_tiles = n_rep + int((t_first + 4 - win0 + 63) / 64);

    extern __shared__ uint8_t ap_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(ap_smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    auto BAR = [&](int i) -> uint32_t { return sbase + AP_OFF_BAR + 8 * i; };
    const uint32_t qfull = BAR(0), sfull = BAR(5), sempty = BAR(6), pfull = BAR(7), pempty = BAR(8),
                   ofull = BAR(9);
    auto full = [&](int s) { return BAR(1 + s); };
    auto empty = [&](int s) { return BAR(3 + s); };
    auto fex = [&](int s) { return BAR(10 + s); };
    auto drain = [&](int w) { return BAR(12 + (w - 5)); };   // issuing warps 5..12
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + AP_OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + AP_OFF_MISC + 4);
    float *fsc = reinterpret_cast<float *>(smem + AP_OFF_FSC);
    float *linv = reinterpret_cast<float *>(smem + AP_OFF_LINV);

    if (threadIdx.x == 0) {
        mbar_init(qfull, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 4);      // four PV chains
            mbar_init(fex(s), 4);
        }
        mbar_init(sfull, 4);             // four S chains
        mbar_init(sempty, 4);            // four softmax warps
        mbar_init(pfull, 4);
        mbar_init(pempty, 4);
        mbar_init(ofull, 4);
        for (int i = 12; i < 20; ++i) mbar_init(BAR(i), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + AP_OFF_MISC, AP_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t qbase = sbase;
    // tile i lives in stage i & 1; once S(i) has completed, its RoPE box (box
    // 8) is dead and holds P(i) [64 query rows x 64 tile rows] for PV(i)
    auto stage_addr = [&](int i) -> uint32_t { return sbase + AP_STAGE * (1 + (i & 1)); };

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&map_q);
            prefetch_tensormap(&map_cache);
            if (n_rep > 0) prefetch_tensormap(&map_rep);
            mbar_expect_tx(qfull, AP_STAGE);
            // each of these copies brings 64 whole rows (nine 64-column blocks)
            tma_load_4d_plain(qbase, &map_q, qfull, 0, int(16 * t_first), 0, a.b);
            int last[2] = {-1, -1};
#pragma unroll 1
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i & 1;
                if (!mbar_wait(empty(s), ((i >> 1) & 1) ^ 1, abort_flag, K_PREFILL, 1)) break;
                mbar_expect_tx(full(s), AP_STAGE);
                const uint32_t dst = stage_addr(i);
                if (i < n_rep) {
                    tma_load_4d_plain(dst, &map_rep, full(s), 0, int(k - a.kc0), 64 * i, 0);
                    // the block's first CTA warms L2 with the next representative
                    // tile for itself and the block's other three CTAs
                    if (qq == 0 && i + 1 < n_rep) {
                        pf_prefetch_4d(&map_rep, 0, int(k - a.kc0), 64 * (i + 1), 0);
                    }
                } else {
                    const int row = int(win0 + 64 * (i - n_rep));
                    tma_load_4d_plain(dst, &map_cache, full(s), 0, row, 0, a.b);
                }
                last[s] = i;
            }
            mbar_wait(qfull, 0, nullptr, K_PREFILL, 2);
            for (int s = 0; s < 2; ++s)
                if (last[s] >= 0) mbar_wait(full(s), (last[s] >> 1) & 1, nullptr, K_PREFILL, 2);
        }
    } else if (warp >= 5 && warp <= 8) {
        // ------------------------------------------------------------ S chains (K quarters)
        // chain c = warp - 5 accumulates k-steps 9c .. 9c+8 into its own 64
        // columns; a single S buffer, released by the softmax warps as soon as
        // they have loaded it
        if (lane == 0) {
            const int c = warp - 5;
            constexpr uint32_t IDESC_S = idesc_bf16(64, 64, 0, 0);
            bool ok = mbar_wait(qfull, 0, abort_flag, K_PREFILL, 3);
#pragma unroll 1
            for (int i = 0; i < n_tiles && ok; ++i) {
                if (!(ok = mbar_wait(full(i & 1), (i >> 1) & 1, abort_flag, K_PREFILL, 4))) break;
                if (!(ok = mbar_wait(sempty, (i & 1) ^ 1, abort_flag, K_PREFILL, 5))) break;
                tc_fence_after();
                const uint32_t stage = stage_addr(i);
                const uint32_t dS = tmem + AP_TM_S + 64 * c;
#pragma unroll
                for (int ks = 0; ks < 9; ++ks) {
                    const int kg = 9 * c + ks;
                    const uint32_t o = (kg >> 2) * AP_CHUNK + (kg & 3) * 32;
                    mma_ss(dS, sdesc_sw128(qbase + o, 16, 1024), sdesc_sw128(stage + o, 16, 1024), IDESC_S,
                           ks > 0 ? 1u : 0u);
                }
                tc_commit(sfull);
            }
            tc_commit(drain(warp));
            mbar_wait(drain(warp), 0, nullptr, K_PREFILL, 6);
        }
    } else if (warp >= 9) {
        // ------------------------------------------------------------ PV chains (d-chunks)
        if (lane == 0) {
            const int cc = warp - 9;
            constexpr uint32_t IDESC_PV = idesc_bf16(128, 64, 1, 0);
            bool ok = true;
#pragma unroll 1
            for (int j = 0; j < n_tiles && ok; ++j) {
                if (!(ok = mbar_wait(pfull, j & 1, abort_flag, K_PREFILL, 7))) break;
                tc_fence_after();
                const uint32_t stage = stage_addr(j);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + AP_TM_O + 64 * cc, sdesc_sw128(stage + 2 * cc * AP_CHUNK + ks * 2048, AP_CHUNK, 1024),
                           sdesc_sw128(stage + 8 * AP_CHUNK + ks * 32, 16, 1024), IDESC_PV, (j | ks) ? 1u : 0u);
                tc_commit(empty(j & 1));
                tc_commit(pempty);
                if (j == n_tiles - 1) tc_commit(ofull);
            }
            tc_commit(drain(warp));
            mbar_wait(drain(warp), 0, nullptr, K_PREFILL, 8);
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        // warp `quad` owns query t = t_first + quad (TMEM lanes 32 quad .. +15 =
        // query rows 16 quad + h); thread T holds heads g = T/4 and g + 8, 16 of
        // the 64 tile rows each (8x + 2 sub + {0,1}).
        const int quad = warp;
        const int64_t t = t_first + quad;
        const int g = lane >> 2, sub = lane & 3;
        const uint32_t lane_base = uint32_t(32 * quad) << 16;
        const int r0 = 16 * quad + g, r1 = r0 + 8;   // query rows of this thread
        float m0 = -1e30f, m1 = -1e30f, l0 = 0.f, l1 = 0.f;
        bool ok = true;
#pragma unroll 1
        for (int i = 0; i < n_tiles; ++i) {
            const int sb = i & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(sfull, i & 1, abort_flag, K_PREFILL, 9));
            if (!ok) break;
            tc_fence_after();
            float va[16], vb[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) va[x] = vb[x] = 0.f;
#pragma unroll
            for (int c = 0; c < 2; ++c) {   // partials 2c and 2c+1 in one load
                uint32_t r[64];
                tmem_ld_16x256b_x16(tmem + AP_TM_S + 128 * c + lane_base, r);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    va[2 * (j & 7)] += __uint_as_float(r[4 * j]);
                    va[2 * (j & 7) + 1] += __uint_as_float(r[4 * j + 1]);
                    vb[2 * (j & 7)] += __uint_as_float(r[4 * j + 2]);
                    vb[2 * (j & 7) + 1] += __uint_as_float(r[4 * j + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sempty);

            // valid columns of this tile for query t
            int64_t nv;
            if (i < n_rep) {
                nv = min64(64, mk - 64 * int64_t(i));
            } else {
                const int64_t row0 = win0 + 64 * int64_t(i - n_rep);
                nv = t - row0 + 1;
                nv = nv < 0 ? 0 : (nv > 64 ? 64 : nv);
            }
            float ta = -INFINITY, tb = -INFINITY;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const int col = 8 * (x >> 1) + 2 * sub + (x & 1);
                va[x] = (col < nv) ? va[x] * a.sl2 : -INFINITY;
                vb[x] = (col < nv) ? vb[x] * a.sl2 : -INFINITY;
                ta = fmaxf(ta, va[x]);
                tb = fmaxf(tb, vb[x]);
            }
            ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 1));
            ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 2));
            tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 1));
            tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 2));
            float fa = 1.f, fb = 1.f;
            if (i == 0) {
                m0 = fmaxf(ta, -1e30f);
                m1 = fmaxf(tb, -1e30f);
            } else {
                if (ta > m0 + 8.f) { fa = fast_exp2(m0 - ta); m0 = ta; l0 *= fa; }
                if (tb > m1 + 8.f) { fb = fast_exp2(m1 - tb); m1 = tb; l1 *= fb; }
            }
            float sa = 0.f, sbm = 0.f;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                va[x] = fast_exp2(va[x] - m0);   // exp2(-inf) = 0 for masked columns
                vb[x] = fast_exp2(vb[x] - m1);
                sa += va[x];
                sbm += vb[x];
            }
            sa += __shfl_xor_sync(0xffffffffu, sa, 1);
            sa += __shfl_xor_sync(0xffffffffu, sa, 2);
            sbm += __shfl_xor_sync(0xffffffffu, sbm, 1);
            sbm += __shfl_xor_sync(0xffffffffu, sbm, 2);
            l0 += sa;
            l1 += sbm;
            if (sub == 0) {
                fsc[sb * 64 + r0] = fa;
                fsc[sb * 64 + r1] = fb;
            }

            // P rows (K-major, 128-byte swizzle) into box 8 of this tile's stage
            {
                uint8_t *pb = smem + AP_STAGE * (1 + sb) + 8 * AP_CHUNK;
                uint8_t *p0 = pb + (r0 >> 3) * 1024 + (r0 & 7) * 128;
                uint8_t *p1 = pb + (r1 >> 3) * 1024 + (r1 & 7) * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    *reinterpret_cast<uint32_t *>(p0 + ((j ^ (r0 & 7)) << 4) + 4 * sub) = pack_bf16(va[2 * j], va[2 * j + 1]);
                    *reinterpret_cast<uint32_t *>(p1 + ((j ^ (r1 & 7)) << 4) + 4 * sub) = pack_bf16(vb[2 * j], vb[2 * j + 1]);
                }
            }
            fence_proxy_async();

            // exchange the rescale factors of all 64 rows, rescale O^T columns
            __syncwarp();
            if (lane == 0) mbar_arrive(fex(sb));
            ok = __all_sync(0xffffffffu, mbar_wait(fex(sb), (i >> 1) & 1, abort_flag, K_PREFILL, 11));
            if (!ok) break;
            const bool any = __any_sync(0xffffffffu, fsc[sb * 64 + lane] != 1.f || fsc[sb * 64 + 32 + lane] != 1.f);
            if (any) {
                // O must hold PV(i-1) before it is rescaled
                ok = __all_sync(0xffffffffu, mbar_wait(pempty, (i & 1) ^ 1, abort_flag, K_PREFILL, 10));
                if (!ok) break;
                tc_fence_after();
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    const uint32_t ta_ = tmem + lane_base + AP_TM_O + 64 * cc;
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        float o[32];
                        tmem_ld32(ta_ + 32 * hh, o);
                        uint32_t rr[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(o[e] * fsc[sb * 64 + 32 * hh + e]);
                        tmem_st32(ta_ + 32 * hh, rr);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull);
        }
        if (ok && sub == 0) {
            linv[r0] = 1.f / l0;
            linv[r1] = 1.f / l1;
        }
        named_bar_sync(1, 128);   // all four softmax warps, on every path
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(ofull, 0, abort_flag, K_PREFILL, 12));
        if (ok) {
            tc_fence_after();
            const size_t row0 = size_t(16) * size_t(k - a.kc0) + 4 * qq;   // chunk row of query t_first
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                const int d = 128 * cc + 32 * quad + lane;
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    float o[32];
                    tmem_ld32(tmem + lane_base + AP_TM_O + 64 * cc + 32 * hh, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int r = 32 * hh + e;            // query row: query r/16, head r%16
                        const float v = o[e] * linv[r];
                        const size_t idx = ((row0 + (r >> 4)) * LCA_HEADS + (r & 15)) * LCA_DC + d;
                        a.o_bf16[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                        if (a.o_lat) a.o_lat[idx] = v;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, AP_TM_COLS);
}

}  // namespace lca
