// attn_decode.cuh -- split-L flash-decode attention on tcgen05 tensor cores,
// read straight from the MLA latent cache, with the LCA condensation fused in.
//
// Row sources ("tiles" of 64 rows, 1152 B each, brought in by one 4-D TMA
// copy as 9 blocks of [64 rows x 64 columns] with 128-byte swizzle, 72 KB
// per stage, 3 stages):
//   MODE_MLA : cache rows 0..L-1 (MLA decode, every token attends).
//   MODE_REPS: stored representatives rep[b][0..m) then window rows m*g..L-1.
//   MODE_LCA : raw history rows 0..m*16-1 (4 groups of 16 per tile), condensed
//              on the fly, then window rows m*16..L-1.
//
// Tensor-core formulation (per tile).  A tcgen05.mma chain issued by one
// thread runs at ~one instruction per ~120 cycles whatever its shape, while
// chains issued by different threads overlap, so the work is split into
// independent chains, each with its own issuing thread and accumulator:
//   S_j [64 x 64] = A(TMEM) * rows[:, 288j : 288j+288]^T,  j = 0, 1
//     (two K-halves of the 576-wide row, 18 k-steps each, TS MMA, M = 64)
//   O^T[128c..128c+127, 16] += rows_lat[:, 128c..]^T * P^T,  c = 0..3
//     (four PV chains of 4 k-steps; A is the same smem tile read MN-major,
//     so each tile is read from HBM exactly once)
// The A operand (TMEM, 144 columns = 288 bf16) holds per-lane query rows,
// all in lanes 0-15 of each warp quadrant q, which is exactly the lane set of
// an M=64 MMA.  Row r = g + 8*half (g = 0..7) holds a 288-element half-row:
//   MLA/REPS: g<4: q_h[288*half : +288]      (h = 4q + g)          -> F = q . row
//   LCA:      g<4: half 0: q_h[0:288], half 1: [q_h[288:512] | 0]    -> X = q_lat . c
//             g=4: u_hi halves,  g=5: u_lo halves (folded summary query
//                  u = u_hi + u_lo in bf16)                         -> s = u . row (关键设计 1)
//             g=6: half 1 = [0 | q_rope] of heads 4q (r=6), 4q+2 (r=14),
//             g=7: the same for heads 4q+1 (r=7), 4q+3 (r=15)        -> Y = q_rope . k^R
//   everything else zero.  S_0 and S_1 are read back with the 16x256b shape:
//   thread T (g = T/4) gets rows g and 8+g of both, for 16 of the 64 tokens
//   (8i + 2(T%4) + {0,1}), so
//     lo = S_0[g] + S_1[8+g]           (F, X, u_hi . row or u_lo . row)
//     ya = S_1[g], yb = S_1[8+g]       (g = 6, 7: Y of two heads each)
//   land in one thread, and every row's tokens are spread over 4 threads.
// For an LCA history tile, with alpha the group softmax of s and I_j the
// group argmax, the logit of representative j for head h is
//   z_hj = scale * (sum_{i in G_j} alpha_i X_hi + Y_h,I_j)
// = scale * (q_lat,h . c_j^rep + q_rope,h . k^R_{I_j}), exactly the
// representative's logit (关键设计 1 and 2) without materialising c_j^rep, and
// its value contribution p_hj c_j^rep = sum_i (p_hj alpha_i) c_i is the PV
// MMA with per-token weights p_hj * alpha_i.
//
// Warp roles (352 threads): warps 0-3 softmax / epilogue (one TMEM lane
// quadrant each), warps 4 and 7 issue the two S chains, warp 5 is the TMA
// producer, warps 6, 8, 9, 10 issue the PV chains of d-chunks 0..3.  Online softmax
// keeps a per-head reference max and rescales O only when the max grows by
// more than 2^8 (the final normalisation uses the same reference, so the
// result is exact either way).  Each CTA writes one (O, m, l) partial per
// sequence piece it owns; tail_decode_kernel merges them.
#pragma once
#include "common.cuh"

namespace lca {

constexpr int AT_TILE = 64;
constexpr int AT_STAGES = 3;
constexpr int AT_CHUNK = AT_TILE * 128;          // 8192 B: [64 rows x 64 cols] bf16
constexpr int AT_STAGE = 9 * AT_CHUNK;           // 73728 B
constexpr int AT_PBUF = LCA_HEADS * 128;         // 2048 B: P^T [16 heads x 64 rows] bf16
constexpr uint32_t AT_TM_Q = 0;                  // 144 columns (288 bf16 per lane)
constexpr uint32_t AT_TM_S = 160;                // S[buf][half]: 4 x 64 columns
constexpr uint32_t AT_TM_O = 416;                // 4 x 16 columns
constexpr uint32_t AT_TM_COLS = 512;
constexpr int AT_THREADS = 352;

constexpr int AT_OFF_P = AT_STAGES * AT_STAGE;          // 221184
constexpr int AT_OFF_BAR = AT_OFF_P + 2 * AT_PBUF;      // 225280
constexpr int AT_NBAR = 26;
constexpr int AT_OFF_MISC = AT_OFF_BAR + 8 * 32;        // 225536
// per softmax warp: e [4 sub][16], anchors [4], 1/den [4], then the tile's
// importance halves u_hi . row [64] and u_lo . row [64]
constexpr int AT_OFF_ALB = AT_OFF_MISC + 256;
// The first segment's query rows (and, fused, the folded summary query) are
// staged in stage 2 by two bulk copies before its first tile load.
constexpr int AT_OFF_QSTAGE = 2 * AT_STAGE;
constexpr int AT_QBYTES = LCA_HEADS * LCA_D * 2;         // 18432: q of one sequence
constexpr int AT_UBYTES = 2 * LCA_D * 2;                 // 2304: u_hi, u_lo of one sequence
constexpr int AT_ALB = 200;                              // floats per softmax warp
constexpr int AT_ALB_SC = 72;                            // offset of the importance halves
constexpr int AT_SMEM = AT_OFF_ALB + 4 * AT_ALB * 4;     // 226944
constexpr int AT_SMEM_ALLOC = AT_SMEM + 1024;           // + alignment slack

enum { MODE_MLA = 0, MODE_REPS = 1, MODE_LCA = 2 };

struct AttnArgs {
    const uint16_t *q;     // [B][16][576]
    const uint16_t *uhl;   // [B][2][576] (LCA)
    int64_t L;             // rows per sequence (varlen: the largest length)
    int64_t m;             // representatives / groups per sequence (0 for MLA); varlen: the
                           // anchor row stride (groups of the largest length)
    int64_t win0;          // first window row (m*g), 0 for MLA
    int n_hist;            // tiles before the window per sequence
    int n_tiles;           // tiles per sequence
    int64_t T;             // B * n_tiles
    int G;                 // CTAs
    float sl2;             // scale * log2(e)
    float *part_o;         // [G+B][16][512]
    float *part_ml;        // [G+B][16][2]
    int32_t *anchor;       // [B][m] or NULL (LCA)
    // ragged batches only: sequence b holds lens[b] rows (clamped to
    // [1, L]) and tiles tile_start[b] .. tile_start[b+1]-1 of the batch's
    // tile list; T = tile_start[B]
    const int32_t *lens;
    const int32_t *tile_start;
    int B;
    int w;
    // 1: launched right after prep_summary_kernel, which lets this grid
    // launch only once everything before it in the stream has completed, so
    // the cache may be read without waiting for the summary query
    int after_prep;
};

// Geometry of one sequence of L rows: its groups m, first window row and
// tiles before the window (history tiles of 4 groups, or stored
// representative tiles of 64 rows), and its tile count.
struct SeqGeom {
    int64_t L, m, win0;
    int n_hist, n_tiles;
};

template <int MODE>
__host__ __device__ __forceinline__ SeqGeom seq_geom(int64_t L, int w)
{
    SeqGeom g;
    g.L = L;
    g.m = (MODE == MODE_MLA || L <= w) ? 0 : (L - w) / 16;
    g.win0 = 16 * g.m;
    g.n_hist = MODE == MODE_MLA ? 0 : MODE == MODE_REPS ? int((g.m + AT_TILE - 1) / AT_TILE) : int((g.m + 3) / 4);
    g.n_tiles = g.n_hist + int((L - g.win0 + AT_TILE - 1) / AT_TILE);
    return g;
}

// The tiles [t0, t1) of sequence b, with its geometry.
struct SeqTiles {
    int64_t b, t0, t1;
    SeqGeom g;
};

__device__ __forceinline__ int64_t clamp_len(int32_t len, int64_t L)
{
    return len < 1 ? 1 : (int64_t(len) > L ? L : int64_t(len));
}

// The sequence that tile t belongs to.  Each role walks its tiles in
// increasing order, so a ragged batch advances from the previous answer
// (cur.b < 0 the first time: a binary search over tile_start).
template <int MODE, bool VARLEN>
__device__ __forceinline__ SeqTiles seq_of(const AttnArgs &a, int64_t t, const SeqTiles &cur)
{
    SeqTiles s;
    if constexpr (!VARLEN) {
        // the same sequence, or the next one (a 64-bit division otherwise)
        if (cur.b >= 0 && t >= cur.t0 && t < cur.t1) return cur;
        if (cur.b >= 0 && t == cur.t1) {
            s = cur;
            s.b = cur.b + 1;
            s.t0 = cur.t1;
            s.t1 = cur.t1 + a.n_tiles;
            return s;
        }
        s.b = t / a.n_tiles;
        s.t0 = s.b * a.n_tiles;
        s.t1 = s.t0 + a.n_tiles;
        s.g.L = a.L;
        s.g.m = a.m;
        s.g.win0 = a.win0;
        s.g.n_hist = a.n_hist;
        s.g.n_tiles = a.n_tiles;
        return s;
    } else {
        if (cur.b >= 0 && t >= cur.t0 && t < cur.t1) return cur;
        int64_t b;
        if (cur.b < 0) {
            int lo = 0, hi = a.B - 1;   // the last b with tile_start[b] <= t
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (a.tile_start[mid] <= t) lo = mid;
                else hi = mid - 1;
            }
            b = lo;
        } else {
            b = cur.b;
            while (b + 1 < a.B && a.tile_start[b + 1] <= t) ++b;
        }
        s.b = b;
        s.t0 = a.tile_start[b];
        s.t1 = a.tile_start[b + 1];
        s.g = seq_geom<MODE>(clamp_len(a.lens[b], a.L), a.w);
        return s;
    }
}

struct TileInfo {
    int from_rep;   // 1: rows come from the representative tensor
    int hist;       // 1: LCA history tile (groups), 0: plain rows
    int64_t row;    // first row
    int valid;      // valid rows (plain) or valid groups (hist)
};

template <int MODE>
__device__ __forceinline__ TileInfo tile_info(const SeqGeom &a, int k)
{
    TileInfo ti;
    ti.from_rep = 0;
    ti.hist = 0;
    if (MODE != MODE_MLA && k < a.n_hist) {
        if (MODE == MODE_REPS) {
            ti.from_rep = 1;
            ti.row = int64_t(k) * AT_TILE;
            ti.valid = int(min64(AT_TILE, a.m - ti.row));
        } else {
            ti.hist = 1;
            ti.row = int64_t(k) * AT_TILE;
            ti.valid = int(min64(4, a.m - int64_t(k) * 4));
        }
        return ti;
    }
    const int kw = (MODE == MODE_MLA) ? k : k - a.n_hist;
    ti.row = a.win0 + int64_t(kw) * AT_TILE;
    ti.valid = int(min64(AT_TILE, a.L - ti.row));
    return ti;
}

// Write this lane's 288-wide query half-row (or zeros) into TMEM columns
// AT_TM_Q.. of its lane.  See the row map in the file header.  qb: the
// sequence's 16 query rows, ub: its u_hi, u_lo rows (LCA), in global or
// shared memory.
template <int MODE>
__device__ __forceinline__ void load_q_rows(const uint16_t *qb, const uint16_t *ub, int quad, int lane,
                                            uint32_t tmem)
{
    const int g = lane & 7, half = (lane >> 3) & 1;
    const uint16_t *src = nullptr;   // a 576-wide vector
    int off = 288 * half;            // first element of the half-row
    int z0 = 0, z1 = 0;              // elements [z0, z1) are zeroed (32-aligned)
    if (lane < 16) {
        if (g < 4) {
            src = qb + size_t(4 * quad + g) * LCA_D;
            if (MODE == MODE_LCA) { z0 = LCA_DC; z1 = LCA_D; }   // X: latent only
        } else if (MODE == MODE_LCA && (g == 4 || g == 5)) {
            src = ub + size_t(g - 4) * LCA_D;
        } else if (MODE == MODE_LCA) {
            // g = 6, 7: Y rows of heads 4q + (g-6) + 2*half, always the
            // second half [0 | q_rope] so that S_1 carries q_rope . k^R
            src = qb + size_t(4 * quad + (g - 6) + 2 * half) * LCA_D;
            off = 288;
            z0 = 288;
            z1 = LCA_DC;
        }
    }
    const uint32_t base = tmem + (uint32_t(32 * quad) << 16) + AT_TM_Q;
    // three 32-element chunks per round trip: their loads are all issued
    // before the first TMEM store (which orders memory), so the 9 chunks take
    // 3 global-memory latencies instead of 9
#pragma unroll 1
    for (int c0 = 0; c0 < 9; c0 += 3) {
        uint4 x[3][4];
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            const int e0 = off + 32 * (c0 + u);
            if (src && !(e0 >= z0 && e0 < z1)) {
                const uint4 *p = reinterpret_cast<const uint4 *>(src + e0);
#pragma unroll
                for (int v = 0; v < 4; ++v) x[u][v] = p[v];
            } else {
#pragma unroll
                for (int v = 0; v < 4; ++v) x[u][v] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            uint32_t r[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                r[4 * v + 0] = x[u][v].x;
                r[4 * v + 1] = x[u][v].y;
                r[4 * v + 2] = x[u][v].z;
                r[4 * v + 3] = x[u][v].w;
            }
            tmem_st16(base + 16 * (c0 + u), r);
        }
    }
}

template <int MODE, bool VARLEN = false>
__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap map_cache,
                       const __grid_constant__ CUtensorMap map_rep, const AttnArgs a)
{
    extern __shared__ uint8_t at_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(at_smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // barrier ids
    auto BAR = [&](int i) -> uint32_t { return sbase + AT_OFF_BAR + 8 * i; };
    auto full = [&](int s) { return BAR(s); };
    auto empty = [&](int s) { return BAR(3 + s); };
    auto sfull = [&](int s) { return BAR(6 + s); };
    auto sempty = [&](int s) { return BAR(8 + s); };
    auto pfull = [&](int s) { return BAR(10 + s); };
    auto pempty = [&](int s) { return BAR(12 + s); };
    auto fex = [&](int s) { return BAR(17 + s); };
    const uint32_t drain2 = BAR(19), drain3 = BAR(20), drain4 = BAR(21), drain5 = BAR(22), drain6 = BAR(23);
    const uint32_t ofull = BAR(14), segready = BAR(15), drain = BAR(16);
    const uint32_t qfull = BAR(24), qempty = BAR(25);   // the staged first query rows
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + AT_OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + AT_OFF_MISC + 4);
    float *fsc = reinterpret_cast<float *>(smem + AT_OFF_MISC + 128);   // [2][16]
    float *alb = reinterpret_cast<float *>(smem + AT_OFF_ALB) + AT_ALB * (warp & 3);   // this softmax warp's

    if (threadIdx.x == 0) {
        for (int s = 0; s < 3; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 4);      // four PV chains
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(sfull(s), 2);      // both S chains
            mbar_init(sempty(s), 4);
            mbar_init(pfull(s), 4);
            mbar_init(pempty(s), 4);     // four PV chains
        }
        mbar_init(ofull, 4);
        mbar_init(segready, 4);
        mbar_init(drain, 1);
        mbar_init(drain2, 1);
        mbar_init(drain3, 1);
        mbar_init(drain4, 1);
        mbar_init(drain5, 1);
        mbar_init(drain6, 1);
        mbar_init(fex(0), 4);
        mbar_init(fex(1), 4);
        mbar_init(qfull, MODE == MODE_LCA ? 2 : 1);   // producer (q); softmax warp 0 (u)
        mbar_init(qempty, 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + AT_OFF_MISC, AT_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_launch_dependents();

    // a ragged batch's tile list comes from the kernel before: wait for it
    // (and so for everything earlier in the stream) before reading it
    if constexpr (VARLEN) griddep_wait();
    const int64_t T = VARLEN ? int64_t(a.tile_start[a.B]) : a.T;
    const int c = blockIdx.x;
    const int64_t t_begin = split_begin(c, T, a.G);
    const int64_t t_end = split_begin(c + 1, T, a.G);

    if (warp == 5) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&map_cache);
            if (MODE == MODE_REPS && a.m > 0) prefetch_tensormap(&map_rep);
            // rows may come from a kernel earlier in the stream: read them only
            // once the preceding grid (and so everything before it) is
            // complete -- already the case when that grid is the summary-query
            // fold, which triggers this launch after its own wait
            if (!a.after_prep) griddep_wait();
            const uint64_t pol = policy_evict_first();
            // the first segment's query rows, in one copy ahead of the tiles;
            // stage 2 takes its first tile once they have moved to TMEM
            const bool staged = t_begin < t_end;
            if (staged) {
                SeqTiles s0{};
                s0.b = -1;
                s0 = seq_of<MODE, VARLEN>(a, t_begin, s0);
                mbar_expect_tx(qfull, AT_QBYTES);
                bulk_load(sbase + AT_OFF_QSTAGE, a.q + size_t(s0.b) * LCA_HEADS * LCA_D, AT_QBYTES, qfull,
                          policy_evict_last());
            }
            int last[3] = {-1, -1, -1};
            int i = 0;
            SeqTiles sq{};
            sq.b = -1;
            for (int64_t t = t_begin; t < t_end; ++t, ++i) {
                const int s = i % 3;
                if (i == 2 && !mbar_wait(qempty, 0, abort_flag, K_ATTN, 14)) break;
                if (!mbar_wait(empty(s), ((i / 3) & 1) ^ 1, abort_flag, K_ATTN, 1)) break;
                sq = seq_of<MODE, VARLEN>(a, t, sq);
                const int64_t b = sq.b;
                const TileInfo ti = tile_info<MODE>(sq.g, int(t - sq.t0));
                mbar_expect_tx(full(s), AT_STAGE);
                const CUtensorMap *mp = ti.from_rep ? &map_rep : &map_cache;
                // the whole tile, all nine 64-column blocks, in one copy
                tma_load_4d(sbase + s * AT_STAGE, mp, full(s), 0, int(ti.row), 0, int(b), pol);
                last[s] = i;
            }
            for (int s = 0; s < 3; ++s)
                if (last[s] >= 0) mbar_wait(full(s), (last[s] / 3) & 1, nullptr, K_ATTN, 2);
            if (staged) mbar_wait(qfull, 0, nullptr, K_ATTN, 15);   // no copy left in flight
        }
    } else if (warp == 4 || warp == 7) {
        // ------------------------------------------------------------ S issuers
        // warp 4: K-half 0 (row columns 0..287), warp 7: K-half 1 (288..575)
        if (lane == 0) {
            const int half = (warp == 7) ? 1 : 0;
            constexpr uint32_t IDESC_S = idesc_bf16(64, AT_TILE, 0, 0);
            int i = 0, seg = 0;
            SeqTiles sq{};
            sq.b = -1;
            for (int64_t t = t_begin; t < t_end; ++t, ++i) {
                sq = seq_of<MODE, VARLEN>(a, t, sq);
                const bool first = (i == 0) || (t == sq.t0);
                if (first && !mbar_wait(segready, seg++ & 1, abort_flag, K_ATTN, 3)) break;
                if (!mbar_wait(full(i % 3), (i / 3) & 1, abort_flag, K_ATTN, 4)) break;
                if (!mbar_wait(sempty(i & 1), ((i >> 1) & 1) ^ 1, abort_flag, K_ATTN, 5)) break;
                tc_fence_after();
                const uint32_t stage = sbase + (i % 3) * AT_STAGE;
                const uint32_t dS = tmem + AT_TM_S + 64 * (2 * (i & 1) + half);
#pragma unroll 6
                for (int ks = 0; ks < 18; ++ks) {
                    const int kg = 18 * half + ks;
                    const uint64_t bd = sdesc_sw128(stage + (kg >> 2) * AT_CHUNK + (kg & 3) * 32, 16, 1024);
                    mma_ts(dS, tmem + AT_TM_Q + 8 * ks, bd, IDESC_S, ks > 0 ? 1u : 0u);
                }
                tc_commit(sfull(i & 1));
            }
            const uint32_t dr = half ? drain3 : drain;
            tc_commit(dr);
            mbar_wait(dr, 0, nullptr, K_ATTN, 6);
        }
    } else if (warp == 6 || warp >= 8) {
        // ------------------------------------------------------------ PV chains
        // One thread per d-chunk (warps 6, 8, 9, 10 -> chunks 0..3), so each
        // chain is 4 MMAs long and the commits track only PV MMAs: a stage is
        // released as soon as the four chunks of its PV complete.
        if (lane == 0) {
            const int cc = (warp == 6) ? 0 : warp - 7;
            constexpr uint32_t IDESC_PV = idesc_bf16(128, LCA_HEADS, 1, 0);
            int j = 0, first_j = 0;
            SeqTiles sq{};
            sq.b = -1;
            for (int64_t t = t_begin; t < t_end; ++t, ++j) {
                sq = seq_of<MODE, VARLEN>(a, t, sq);
                if (j == 0 || t == sq.t0) first_j = j;
                const bool last = (t + 1 == t_end) || (t + 1 == sq.t1);
                if (!mbar_wait(pfull(j & 1), (j >> 1) & 1, abort_flag, K_ATTN, 7)) break;
                tc_fence_after();
                const uint32_t stage = sbase + (j % 3) * AT_STAGE;
                const uint32_t pbuf = sbase + AT_OFF_P + (j & 1) * AT_PBUF;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = sdesc_sw128(stage + 2 * cc * AT_CHUNK + ks * 2048, AT_CHUNK, 1024);
                    const uint64_t bd = sdesc_sw128(pbuf + ks * 32, 16, 1024);
                    mma_ss(tmem + AT_TM_O + 16 * cc, ad, bd, IDESC_PV, (j == first_j && ks == 0) ? 0u : 1u);
                }
                tc_commit(empty(j % 3));
                tc_commit(pempty(j & 1));
                if (last) tc_commit(ofull);
            }
            const uint32_t dr = cc == 0 ? drain2 : cc == 1 ? drain4 : cc == 2 ? drain5 : drain6;
            tc_commit(dr);
            mbar_wait(dr, 0, nullptr, K_ATTN, 13);
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int quad = warp;
        const float NEG_INF = -INFINITY;
        const uint32_t lane_base = uint32_t(32 * quad) << 16;
        int i = 0, seg = 0;
        int64_t t = t_begin;
        bool ok = true;
        float m_use = NEG_INF, l_run = 0.f;   // threads with lane/4 < 4: head 4*quad + lane/4
        griddep_wait();   // the folded summary query comes from the previous kernel
        SeqTiles sq{};
        sq.b = -1;
        if (MODE == MODE_LCA && warp == 0 && lane == 0 && t_begin < t_end) {
            sq = seq_of<MODE, VARLEN>(a, t_begin, sq);
            mbar_expect_tx(qfull, AT_UBYTES);
            bulk_load(sbase + AT_OFF_QSTAGE + AT_QBYTES, a.uhl + size_t(sq.b) * 2 * LCA_D, AT_UBYTES, qfull,
                      policy_evict_last());
        }
        while (ok && t < t_end) {
            sq = seq_of<MODE, VARLEN>(a, t, sq);
            const int64_t b = sq.b;
            const int64_t seg_end = min64(t_end, sq.t1);
            if (seg == 0) {
                // staged by the producer (q) and by warp 0 (u) in stage 2
                ok = mbar_wait(qfull, 0, abort_flag, K_ATTN, 16);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                const uint16_t *qs = reinterpret_cast<const uint16_t *>(smem + AT_OFF_QSTAGE);
                load_q_rows<MODE>(qs, qs + LCA_HEADS * LCA_D, quad, lane, tmem);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(qempty);
            } else {
                load_q_rows<MODE>(a.q + size_t(b) * LCA_HEADS * LCA_D, a.uhl + size_t(b) * 2 * LCA_D, quad, lane,
                                  tmem);
                tc_fence_before();
                __syncwarp();
            }
            if (lane == 0) mbar_arrive(segready);
            m_use = NEG_INF;
            l_run = 0.f;
            const int first = i;
            for (; t < seg_end; ++t, ++i) {
                const int k = int(t - sq.t0);
                const int sb = i & 1;
                const TileInfo ti = tile_info<MODE>(sq.g, k);
                ok = mbar_wait(sfull(sb), (i >> 1) & 1, abort_flag, K_ATTN, 8);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                // thread T: rows g = T/4 (lo) and g+8 (hi), tokens
                // tok(x) = 8*(x>>1) + 2*sub + (x&1), x = 0..15; group of x = x>>2
                const int g = lane >> 2, sub = lane & 3;
                float lo[16], ya[16], yb[16];
                {
                    const uint32_t s0 = tmem + AT_TM_S + 64 * (2 * sb) + lane_base;
                    float r[32];
                    tmem_ld_16x256b_x8(s0, r);                 // rows g, 8+g of S_0
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        lo[2 * j] = r[4 * j];
                        lo[2 * j + 1] = r[4 * j + 1];
                    }
                    tmem_ld_16x256b_x8(s0 + 64, r);            // rows g, 8+g of S_1
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        lo[2 * j] += r[4 * j + 2];
                        lo[2 * j + 1] += r[4 * j + 3];
                        ya[2 * j] = r[4 * j];
                        ya[2 * j + 1] = r[4 * j + 1];
                        yb[2 * j] = r[4 * j + 2];
                        yb[2 * j + 1] = r[4 * j + 3];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sempty(sb));
                if constexpr (VARLEN) {
                    // Rows past this sequence's end (or past its kept
                    // representatives) lie inside the tensor map, which spans
                    // the longest sequence, and may hold anything.
                    // Their P weights are 0, but 0 * NaN is NaN in the PV MMA,
                    // so zero them in the stage's 8 latent boxes; S has read
                    // the stage, and the proxy fence before pfull orders these
                    // stores before PV.
                    const int ok_rows = ti.from_rep ? ti.valid : int(min64(AT_TILE, sq.g.L - ti.row));
                    if (ok_rows < AT_TILE) {
                        const int nr = AT_TILE - ok_rows;
                        uint8_t *stg = smem + (i % 3) * AT_STAGE;
                        for (int x = 32 * quad + lane; x < 8 * nr * 8; x += 128) {
                            const int box = x / (8 * nr), r = ok_rows + (x / 8) % nr, ch = x % 8;
                            *reinterpret_cast<uint4 *>(stg + box * AT_CHUNK + r * 128 + ch * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }

                float w[16];        // P^T weights of this thread's head and tokens (g < 4)
                float f = 1.f;      // reference-max rescale factor of this head
                if (MODE == MODE_LCA && ti.hist) {
                    // ---- fused condensation of 4 groups.  Rows g = 4 and g = 5
                    // hold u_hi . row and u_lo . row; they go through this warp's
                    // shared-memory slot so that every lane takes 2 of the 64
                    // tokens (group j = lanes 8j .. 8j+7): group max, first-index
                    // argmax and denominator in 3 shuffle rounds, 2 exponentials
                    // per lane.  al (exp(s - group max), unnormalised) comes back
                    // in the layout each thread reads: [sub][x] for its tokens.
                    float al[16];       // exp(s - group max); alpha = al * rinv
                    float rinv[4];      // 1 / sum of the group's al
                    int anc[4];         // the group's argmax (offset within the group)
                    float *sch = alb + AT_ALB_SC;
                    if (g == 4 || g == 5) {
                        float *dst = sch + 64 * (g - 4);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            *reinterpret_cast<float2 *>(dst + 8 * j + 2 * sub) = make_float2(lo[2 * j], lo[2 * j + 1]);
                    }
                    __syncwarp();
                    {
                        const float2 h2 = *reinterpret_cast<const float2 *>(sch + 2 * lane);
                        const float2 l2 = *reinterpret_cast<const float2 *>(sch + 64 + 2 * lane);
                        const float s0 = h2.x + l2.x, s1 = h2.y + l2.y;   // tokens 2 lane, 2 lane + 1
                        float gm = s0;
                        int gi = 2 * lane;
                        if (s1 > gm) { gm = s1; gi = 2 * lane + 1; }
#pragma unroll
                        for (int off = 1; off <= 4; off <<= 1) {
                            const float og = __shfl_xor_sync(0xffffffffu, gm, off);
                            const int oi = __shfl_xor_sync(0xffffffffu, gi, off);
                            if (og > gm || (og == gm && oi < gi)) { gm = og; gi = oi; }
                        }
                        const float e0 = fast_exp2((s0 - gm) * kLog2e), e1 = fast_exp2((s1 - gm) * kLog2e);
                        float den = e0 + e1;
#pragma unroll
                        for (int off = 1; off <= 4; off <<= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
                        *reinterpret_cast<float2 *>(alb + 16 * (lane & 3) + 2 * (lane >> 2)) = make_float2(e0, e1);
                        if ((lane & 7) == 0) {
                            const int j = lane >> 3;
                            reinterpret_cast<int *>(alb + 64)[j] = gi - 16 * j;
                            alb[68 + j] = __fdividef(1.f, den);   // den >= 1 (the maximum's term)
                        }
                    }
                    __syncwarp();
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float4 t4 = *reinterpret_cast<const float4 *>(alb + 16 * sub + 4 * v);
                        al[4 * v] = t4.x;
                        al[4 * v + 1] = t4.y;
                        al[4 * v + 2] = t4.z;
                        al[4 * v + 3] = t4.w;
                    }
                    {
                        const int4 a4 = *reinterpret_cast<const int4 *>(alb + 64);
                        anc[0] = a4.x;
                        anc[1] = a4.y;
                        anc[2] = a4.z;
                        anc[3] = a4.w;
                        const float4 r4 = *reinterpret_cast<const float4 *>(alb + 68);
                        rinv[0] = r4.x;
                        rinv[1] = r4.y;
                        rinv[2] = r4.z;
                        rinv[3] = r4.w;
                    }
                    if (a.anchor && quad == 0 && lane == 0) {
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4)
                            if (k4 < ti.valid)
                                a.anchor[size_t(b) * a.m + size_t(k) * 4 + k4] = int32_t((k * 4 + k4) * 16 + anc[k4]);
                    }
                    // per group: zx = sum alpha X (threads g < 4, summed over the 4
                    // threads of the row) and the anchor's Y of two heads (threads
                    // g = 6, 7: only the thread holding the anchor token keeps it)
                    float zx[4], y0[4], y1[4];
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        float acc = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int x = 4 * k4 + e;
                            const int te = 8 * (e >> 1) + 2 * sub + (e & 1);
                            acc = fmaf(al[x], lo[x], acc);
                            if (te == anc[k4]) { a0 = ya[x]; a1 = yb[x]; }
                        }
                        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                        zx[k4] = acc * rinv[k4];
                        y0[k4] = a0;
                        y1[k4] = a1;
                    }
                    // head 4q+g's Y lives in thread g' = 6 + (g&1) (ya for g < 2,
                    // yb for g >= 2), in the sub-lane whose tokens hold the anchor
                    float z[4];
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int ysrc = 24 + 4 * (g & 1) + ((anc[k4] & 7) >> 1);
                        const float v0 = __shfl_sync(0xffffffffu, y0[k4], ysrc);
                        const float v1 = __shfl_sync(0xffffffffu, y1[k4], ysrc);
                        const float yv = (g & 2) ? v1 : v0;
                        z[k4] = (k4 < ti.valid) ? (zx[k4] + yv) * a.sl2 : NEG_INF;
                    }
                    const float tmax = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
                    if (i == first) {
                        m_use = tmax;
                    } else if (tmax > m_use + 8.f) {
                        f = fast_exp2(m_use - tmax);
                        m_use = tmax;
                        l_run *= f;
                    }
                    float psum = 0.f;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const float p = (k4 < ti.valid) ? fast_exp2(z[k4] - m_use) : 0.f;
                        psum += p;
                        const float pr = p * rinv[k4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) w[4 * k4 + e] = pr * al[4 * k4 + e];
                    }
                    l_run += psum;
                } else {
                    // ---- plain rows (MLA, stored reps, window; LCA adds Y)
                    if (MODE == MODE_LCA) {
                        // window rows: F = X + Y, Y of head 4q+g from thread 6 + (g&1)
                        const int ysrc = 24 + 4 * (g & 1) + sub;
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            const float v0 = __shfl_sync(0xffffffffu, ya[x], ysrc);
                            const float v1 = __shfl_sync(0xffffffffu, yb[x], ysrc);
                            lo[x] += (g & 2) ? v1 : v0;
                        }
                    }
                    float tmax = NEG_INF;
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const int tok = 8 * (x >> 1) + 2 * sub + (x & 1);
                        w[x] = (tok < ti.valid) ? lo[x] * a.sl2 : NEG_INF;
                        tmax = fmaxf(tmax, w[x]);
                    }
                    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
                    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
                    if (i == first) {
                        m_use = tmax;
                    } else if (tmax > m_use + 8.f) {
                        f = fast_exp2(m_use - tmax);
                        m_use = tmax;
                        l_run *= f;
                    }
                    float psum = 0.f;
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        w[x] = fast_exp2(w[x] - m_use);   // exp2(-inf) = 0 for masked rows
                        psum += w[x];
                    }
                    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
                    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
                    l_run += psum;
                }
                if (g < 4 && sub == 0) fsc[(i & 1) * 16 + 4 * quad + g] = f;

                // ---- P^T row of this thread's head: token pairs (8j+2sub, +1)
                ok = mbar_wait(pempty(sb), ((i >> 1) & 1) ^ 1, abort_flag, K_ATTN, 9);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                if (g < 4) {
                    const int h = 4 * quad + g;
                    uint8_t *prow = smem + AT_OFF_P + sb * AT_PBUF + (h >> 3) * 1024 + (h & 7) * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint32_t *>(prow + ((j ^ (h & 7)) << 4) + 4 * sub) =
                            pack_bf16(w[2 * j], w[2 * j + 1]);
                }
                fence_proxy_async();

                // ---- rescale O^T columns whose reference max moved (the
                // factors of all 16 heads are exchanged through fsc)
                __syncwarp();
                if (lane == 0) mbar_arrive(fex(i & 1));
                ok = mbar_wait(fex(i & 1), (i >> 1) & 1, abort_flag, K_ATTN, 12);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                bool any = false;
                float fs[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    fs[h] = fsc[(i & 1) * 16 + h];
                    any |= (fs[h] != 1.f);
                }
                if (any) {
                    // PV(i-1) must have landed before O is touched
                    ok = mbar_wait(pempty((i - 1) & 1), ((i - 1) >> 1) & 1, abort_flag, K_ATTN, 11);
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < 4; ++cc) {
                        float o[16];
                        const uint32_t ta = tmem + lane_base + AT_TM_O + 16 * cc;
                        tmem_ld16(ta, o);
                        uint32_t r[16];
#pragma unroll
                        for (int h = 0; h < 16; ++h) r[h] = __float_as_uint(o[h] * fs[h]);
                        tmem_st16(ta, r);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(pfull(sb));
            }
            if (!ok) break;

            // ---- segment done: write the partial (O, m, l) of sequence b
            ok = mbar_wait(ofull, seg & 1, abort_flag, K_ATTN, 10);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const size_t slot = size_t(c) + size_t(b);
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float o[16];
                tmem_ld16(tmem + lane_base + AT_TM_O + 16 * cc, o);
                const int d = 128 * cc + 32 * quad + lane;
#pragma unroll
                for (int h = 0; h < 16; ++h) a.part_o[(slot * LCA_HEADS + h) * LCA_DC + d] = o[h];
            }
            if ((lane & 3) == 0 && lane < 16) {
                const size_t hh = slot * LCA_HEADS + 4 * quad + (lane >> 2);
                a.part_ml[hh * 2 + 0] = m_use;
                a.part_ml[hh * 2 + 1] = l_run;
            }
            tc_fence_before();
            ++seg;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, AT_TM_COLS);
}

}  // namespace lca
