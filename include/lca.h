/*
 * lca.h -- C ABI of liblca_b200.so: multi-head latent attention (MLA) decode
 * read straight from the compressed latent KV cache, and latent-condensed
 * attention (LCA) on top of it, as hand-written sm_100a (B200) kernels.
 *
 * Method: "Latent-Condensed Transformer for Efficient Long Context Modeling"
 * (papernotes.org notes on the ACL 2026 paper).  整体框架 (overall
 * framework): history outside a local window of w recent tokens is cut into
 * m = floor((L - w) / g) groups; each group is condensed into one
 * representative; attention runs over [m representatives || window].
 * 关键设计 1: the representative latent is c_j^rep = sum_i alpha_i c_i^KV with
 * alpha = softmax of the tokens' importance under the summary query (mean of
 * the last g queries).  关键设计 2: the representative RoPE key is the key of
 * the group's most important token, k_j^{R_rep} = k^R_{I_j}.  关键设计 3: the
 * window is kept uncompressed.
 *
 * Fixed model dimensions: H = 16 heads, latent d_c = 512, RoPE key d_r = 64,
 * cache row D = 576 bf16 (1152 bytes: [c^KV | k^R]), value width d_v = 128.
 * Queries come in the weight-absorbed form q = [q_lat (512) | q_rope (64)]
 * per head, so logits are taken against the latent directly:
 *   z = scale * (q_lat . c + q_rope . k^R),  o_lat = sum p c,
 *   out_h = W_UV[h]^T o_lat,h  (W_UV laid out [16][512][128]).
 * The importance of token i is s_i = (1/H) sum_h scale * (qbar_h . row_i);
 * a representative carries no logit bias; the anchor is the first index of
 * the group maximum; tokens left over by the floor join the window.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the
 *    library allocates no device memory.  Two exceptions read or write host
 *    memory in place over the host link (no copy engine involved): `out` of
 *    every decode and prefill entry point and of lca_combine_shards, and the
 *    inputs of lca_append_token, may be pinned host memory mapped at the
 *    same address (cudaHostAlloc / cudaMallocHost / cudaHostRegister); such
 *    a pointer is checked with cudaPointerGetAttributes, and pageable or
 *    unknown memory is refused with LCA_ERR_INVALID_ARG.  bf16 tensors are
 *    passed as `const void*` holding IEEE bfloat16 values, row-major and
 *    contiguous.
 *  - Every bf16 / fp32 tensor pointer must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *    asynchronous on it and never synchronise the host.  The kernels of a
 *    call are chained with programmatic dependent launch, but none reads an
 *    input before all earlier work in the stream has completed: writes
 *    issued on the stream before the call (copies, or the caller's kernels,
 *    programmatic-launch ones included) are seen by it.
 *  - Return 0 (LCA_OK) or a negative lca_status.  Invalid arguments are
 *    rejected before anything is launched.  A launch failure returns
 *    LCA_ERR_CUDA with nothing further enqueued.
 *  - `ws` is caller-owned device scratch of at least
 *    lca_workspace_bytes(op, ...) bytes, 256-byte aligned.  Its contents on
 *    entry do not matter; two calls in flight at once need separate ws.
 *  - Every in-kernel wait is bounded; a kernel whose wait expires records
 *    LCA_ERR_DEVICE_TIMEOUT in a device status word (read it with
 *    lca_device_status) and returns early, leaving outputs undefined.
 *  - The current token is already in the cache: the query of a decode step
 *    sits at position L-1 of a cache of length L.
 */
#ifndef LCA_B200_H
#define LCA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LCA_HEADS 16
#define LCA_DC 512
#define LCA_DR 64
#define LCA_D 576
#define LCA_DV 128

/* Status codes. */
#define LCA_OK 0
#define LCA_ERR_INVALID_ARG (-1)   /* NULL pointer, bad size or range */
#define LCA_ERR_MISALIGNED (-2)    /* a pointer is not 16-byte aligned (ws: 256) */
#define LCA_ERR_WORKSPACE (-3)     /* ws NULL or smaller than lca_workspace_bytes */
#define LCA_ERR_UNSUPPORTED (-4)   /* parameter outside what the kernels implement */
#define LCA_ERR_CUDA (-5)          /* a CUDA runtime/driver call or launch failed */
#define LCA_ERR_NO_DEVICE (-6)     /* the current device is not sm_100 */
#define LCA_ERR_DEVICE_TIMEOUT (-7) /* a kernel's bounded wait expired */
#define LCA_ERR_SCRATCH_LIMIT (-8) /* problem larger than lca_decode_noalloc's built-in scratch */

/* Condensation parameters.  g: group size (16; g = 1 makes every token its
 * own representative, which is exactly MLA).  w: local window (>= 0).
 * scale: logit scale (1/sqrt(192) for the 128+64 per-head MLA width).
 * variant: LCA_VARIANT_LCA (0) is the method; the other two are the
 * ablations of the page's 消融实验 table, accepted by lca_condense,
 * lca_condense_append and lca_prefill_block (the decode entry points that
 * condense on the fly return LCA_ERR_UNSUPPORTED for them: decode an
 * ablation with lca_condense + lca_decode_attn, since the attention over
 * stored representatives is the same for all three):
 *   LCA_VARIANT_POOL_POSITION: the RoPE key is pooled with the same weights
 *     as the latent, k_rep = sum_i alpha_i k^R_i ("纯池化（含位置）");
 *   LCA_VARIANT_SPARSE: the representative is the most important token's row,
 *     [c_I | k^R_I] ("纯稀疏"). */
#define LCA_VARIANT_LCA 0
#define LCA_VARIANT_POOL_POSITION 1
#define LCA_VARIANT_SPARSE 2
/* cache_pitch: rows from the first row of one sequence's cache to the
 * next one's.  0 means the packed layout [B][L][576] (pitch L).  A decoder
 * that keeps a preallocated cache [B][L_max][576] and lets L grow passes
 * L_max here, and rows L .. L_max-1 of each sequence are never read.
 * Otherwise it must satisfy cache_pitch >= L and B * cache_pitch < 2^40.
 * It applies to every entry point taking lca_params (the cache_shard of
 * lca_decode_shard, rows L_shard); mla_decode_attn takes the packed layout,
 * and lca_decode with g = 1 is MLA decode with a pitch. */
typedef struct {
    int g;
    int w;
    float scale;
    int variant;
    int64_t cache_pitch;
} lca_params;

/* Operation ids for lca_workspace_bytes. */
#define LCA_OP_MLA_DECODE 0
#define LCA_OP_CONDENSE 1
#define LCA_OP_DECODE_ATTN 2
#define LCA_OP_DECODE 3
#define LCA_OP_PREFILL 4

/* m = max(0, floor((L - w) / g)); 0 for invalid parameters. */
int64_t lca_num_groups(int64_t L, lca_params p);

/* Device scratch an entry point needs for this problem size, in bytes
 * (0 for invalid parameters).  q_len is used by LCA_OP_PREFILL only. */
size_t lca_workspace_bytes(int op, int B, int64_t L, int64_t q_len, lca_params p);

/* MLA decode (the uncondensed reference point, "MLA keeps all L tokens in
 * attention", 研究背景与动机): each of B sequences' current query attends
 * all L cached rows; split-L across the GPU, log-sum-exp combine, then the
 * per-head W_UV up-projection.
 *   cache [B][L][576] bf16, q [B][16][576] bf16, w_uv [16][512][128] bf16
 *   out   [B][16][128] fp32            (required)
 *   o_lat [B][16][512] fp32 or NULL    (attention output before W_UV)
 * 1 <= B, 1 <= L < 2^31. */
int mla_decode_attn(const void *cache, const void *q, const void *w_uv, int B, int64_t L,
                    float scale, float *out, float *o_lat, void *ws, size_t ws_bytes,
                    void *stream);

/* LCA condensation (关键设计 1 and 2) of the m history groups of each
 * sequence with the summary query qbar = mean of q_recent:
 *   cache    [B][L][576] bf16
 *   q_recent [B][g][16][576] bf16: the last g queries (current one
 *            included).  Only their mean is used, so the order of the g
 *            slots does not matter: a decode loop may keep q_recent on the
 *            device as a ring and overwrite the oldest slot each step.
 *   rep      [B][m][576] bf16  out: [c_rep (512) | k^R of the anchor (64)],
 *            the latent rounded to bf16 like a cache row, the key copied
 *            bit for bit
 *   anchor   [B][m] int32 out or NULL: absolute position of each anchor
 *   alpha    [B][m][g] fp32 out or NULL: pooling weights
 * Requires g == 16.  m == 0 is valid (nothing is written). */
int lca_condense(const void *cache, const void *q_recent, int B, int64_t L, lca_params p,
                 void *rep, int32_t *anchor, float *alpha, void *ws, size_t ws_bytes,
                 void *stream);

/* LCA decode attention over stored representatives (整体框架): the current
 * query attends [rep rows 0..m-1 || cache rows m*g .. L-1], then W_UV.
 *   rep [B][m][576] bf16 (as written by lca_condense); may be NULL if m == 0.
 * Other arguments as mla_decode_attn.  Requires g == 16. */
int lca_decode_attn(const void *cache, const void *rep, const void *q, const void *w_uv, int B,
                    int64_t L, lca_params p, float *out, float *o_lat, void *ws, size_t ws_bytes,
                    void *stream);

/* Stored-representative ("condensed cache") decode: the reading of the
 * page's 90% KV-cache compression (一句话总结, 关键发现) in which a group is
 * condensed once, when it leaves the window, and kept.  Group j leaves the
 * window at the step whose cache length is w + g (j + 1); the caller keeps a
 * representative cache rep[B][rep_cap][576] (rep_cap >= the largest m it
 * will reach) and, at each step where m = lca_num_groups(L, p) has grown,
 * appends the new groups with lca_condense_append, then attends with
 * lca_decode_stored, which reads only the m kept rows and the window.
 *
 * lca_condense_append: condense groups j0 .. m-1 of every sequence with the
 * summary query of q_recent (as lca_condense) into rows j0 .. m-1 of rep
 * (row stride rep_cap rows per sequence); anchor [B][rep_cap] int32 and
 * alpha [B][rep_cap][g] fp32 are optional, same rows.  0 <= j0 <= m;
 * j0 == m writes nothing.  Requires g == 16.  ws: LCA_OP_CONDENSE bytes. */
int lca_condense_append(const void *cache, const void *q_recent, int B, int64_t L, lca_params p,
                        int64_t j0, void *rep, int64_t rep_cap, int32_t *anchor, float *alpha,
                        void *ws, size_t ws_bytes, void *stream);

/* lca_decode_stored: the current query attends [rep rows 0 .. m-1 || cache
 * rows m*g .. L-1] of each sequence, then W_UV (as lca_decode_attn, with the
 * representative rows read at a stride of rep_cap rows per sequence).
 * rep_cap >= m; rep may be NULL if m == 0.  Requires g == 16.
 * ws: LCA_OP_DECODE_ATTN bytes. */
int lca_decode_stored(const void *cache, const void *rep, int64_t rep_cap, const void *q,
                      const void *w_uv, int B, int64_t L, lca_params p, float *out, float *o_lat,
                      void *ws, size_t ws_bytes, void *stream);

/* One whole LCA decode step, fused: summary query, per-group importance,
 * softmax pooling, anchor pick and attention over [representatives ||
 * window] in one pass over the cache (representatives never leave the
 * chip), log-sum-exp combine, W_UV.  Same results as lca_condense followed
 * by lca_decode_attn, except that representatives are not rounded to bf16.
 *   anchor [B][m] int32 out or NULL.
 * g == 1 runs mla_decode_attn (every token is its own representative).
 * Otherwise requires g == 16. */
int lca_decode(const void *cache, const void *q_recent, const void *q, const void *w_uv, int B,
               int64_t L, lca_params p, float *out, float *o_lat, int32_t *anchor, void *ws,
               size_t ws_bytes, void *stream);

/* lca_decode for a ragged batch: sequence b holds lens[b] cached rows
 * (1 <= lens[b] <= L; values outside are clamped), at rows 0 .. lens[b]-1
 * of its cache, [B][pitch][576] with pitch = cache_pitch or L.  Each
 * sequence is decoded exactly as lca_decode would decode it alone: its own
 * m_b = lca_num_groups(lens[b], p) groups and window; its query sits at
 * position lens[b]-1.  (Not part of the page's method: a serving batch holds
 * sequences of different lengths.)
 *   lens   [B] int32, a DEVICE array (4-byte aligned), read by the kernels
 *   anchor [B][m] int32 or NULL with m = lca_num_groups(L, p): row b holds
 *          sequence b's m_b anchors (the rest of the row is not written)
 * g == 1 is MLA decode of each sequence's lens[b] rows.  Otherwise requires
 * g == 16 and variant LCA.  B * (L / 64 + 2) < 2^31 (LCA_ERR_UNSUPPORTED
 * otherwise).  ws: LCA_OP_DECODE bytes for (B, L). */
int lca_decode_varlen(const void *cache, const int32_t *lens, const void *q_recent, const void *q,
                      const void *w_uv, int B, int64_t L, lca_params p, float *out, float *o_lat,
                      int32_t *anchor, void *ws, size_t ws_bytes, void *stream);

/* lca_decode_stored for a ragged batch: sequence b holds lens[b] cached rows
 * (clamped to [1, L]) and its first m_b = lca_num_groups(lens[b], p)
 * representatives in rep [B][rep_cap][576] (rep_cap >= lca_num_groups(L,
 * p)); its query attends [rep rows 0 .. m_b-1 || cache rows 16 m_b ..
 * lens[b]-1], then W_UV.  lens is a DEVICE int32 array [B].  A decode loop
 * appends a sequence's groups with lca_condense_append on that sequence's
 * views when its length crosses a group boundary.  Requires g == 16 and
 * B * (L / 64 + 2) < 2^31.  ws: LCA_OP_DECODE_ATTN bytes for (B, L). */
int lca_decode_stored_varlen(const void *cache, const void *rep, int64_t rep_cap, const int32_t *lens,
                             const void *q, const void *w_uv, int B, int64_t L, lca_params p, float *out,
                             float *o_lat, void *ws, size_t ws_bytes, void *stream);

/* Blockwise LCA prefill of query positions [q_start, q_start + q_len) (both
 * multiples of g).  The page reports prefill speed but does not spell out the
 * procedure; this is its plainest reading.  Block k covers t0 = k*g ..
 * t0+g-1; its summary query is the mean of its own g queries; history rows
 * 0 .. m_k*g-1 with m_k = max(0, floor((t0 - w)/g)) are condensed with it
 * (关键设计 1, 2); each query t of the block attends [m_k representatives ||
 * cache rows m_k*g .. t] causally (整体框架, 关键设计 3).
 *   cache  [B][L][576] bf16, q [B][L][16][576] bf16 (the absorbed queries of
 *          every position; rows outside the range are not read),
 *   w_uv   [16][512][128] bf16
 *   out    [B][q_len][16][128] fp32            (required)
 *   o_lat  [B][q_len][16][512] fp32 or NULL    (attention output before W_UV)
 *   anchor [B][q_len/g][m_last] int32 or NULL, m_last = m of the range's last
 *          block: absolute anchor positions of block k's groups j < m_k in
 *          row (k - q_start/g); the rest of each row is not written.
 * Representatives are rounded to bf16 like cache rows.  p.variant selects
 * the method or one of its two ablations (see lca_params).  Requires g == 16,
 * L <= 2^27 and B * q_len / 16 < 2^31 (LCA_ERR_UNSUPPORTED otherwise).  ws: lca_workspace_bytes(LCA_OP_PREFILL, B, L, q_len, p) bytes
 * (enough for any q_start; the blocks are processed in chunks of 256 so the
 * workspace stays near 256 * m_last * 1152 bytes). */
int lca_prefill_block(const void *cache, const void *q, const void *w_uv, int B, int64_t L,
                      int64_t q_start, int64_t q_len, lca_params p, float *out, float *o_lat,
                      int32_t *anchor, void *ws, size_t ws_bytes, void *stream);

/* lca_decode without any device allocation, for callers that cannot call
 * cudaMalloc or hand the library a workspace: plugins and operators that
 * only receive their pre-allocated input and output buffers, runtimes whose
 * device memory plan is fixed before they start, and allocators that forbid
 * new device memory while they run.  (The page has no counterpart: this is
 * an interface convenience, not part of the method.)
 *
 * Same arguments and results as lca_decode, minus ws / ws_bytes: the scratch
 * (summary query, split-L partials) lives in a file-scope device array of
 * this library, about 8.4 MiB, which every GPU that loads the library keeps
 * until the process exits.  Limits: 1 <= B <= LCA_NOALLOC_MAX_BATCH,
 * otherwise LCA_ERR_SCRATCH_LIMIT and nothing is launched; g must be 16
 * (or 1, which is MLA decode as for lca_decode).
 *
 * The first call on a device does its set-up, with that device current: it
 * looks up the array's device address (cudaGetSymbolAddress) and runs the
 * library's one-time per-device set-up (kernel attributes, the tensor-map
 * encoder).  Make that first call before any stream capture.  All calls on
 * a device share the one array: every byte a call reads is written earlier
 * in the same call (nothing needs to start at zero), but two calls whose
 * work overlaps on the GPU (different streams, or host threads racing)
 * corrupt each other's results.  With kernel timing switched on
 * (lca_profile_enable) the library creates CUDA event objects; leave it off
 * where that is not allowed. */
#define LCA_NOALLOC_MAX_BATCH 8
int lca_decode_noalloc(const void *cache, const void *q_recent, const void *q, const void *w_uv,
                       int B, int64_t L, lca_params p, float *out, float *o_lat, int32_t *anchor,
                       void *stream);

/* Decode split along the sequence across devices.  Every query's attention
 * over [representatives || window] (整体框架) is a softmax over a set of rows,
 * so it can be cut into shards of rows.  Each shard yields a partial: o
 * normalised over its own rows plus the log-sum-exp of its logits.
 * lca_combine_shards merges the partials by their log-sum-exp and applies
 * W_UV.  (The page runs on one device; this interface is not part of the
 * method, and the result equals lca_decode up to fp32 rounding.)
 *
 * A shard record is LCA_SHARD_RECORD_PER_HEAD * 16 * B floats, contiguous:
 *   o    [B][16][512] fp32: the attention output over the shard's rows alone
 *   lse2 [B][16]      fp32: log2( sum over the shard's rows of exp(z) ),
 *        z the scaled logit of 整体框架
 * so a plain all-gather of the records feeds lca_combine_shards.
 *
 * lca_decode_shard: cache_shard [B][L_shard][576] bf16 (contiguous) holds
 * rows row0 .. row0+L_shard-1 of every sequence of a cache of length L.
 * Shards cut at group boundaries.  row0 % g == 0, and row0 <= m*g with
 * m = lca_num_groups(L, p).  Either the shard ends at L, which makes it the
 * last shard and gives it the whole window, or it ends at a multiple of g no
 * later than m*g.  Each of its groups is condensed with the summary query
 * of q_recent [B][g][16][576] (NULL allowed only if the shard has no
 * groups), exactly as in lca_decode.  q [B][16][576] is the current query.
 *   part   one shard record (required, 16-byte aligned)
 *   anchor [B][m_shard] int32 or NULL, m_shard = groups in the shard: the
 *          anchor's row within the shard (add row0 for its position).
 * Requires g == 16 and variant LCA.  ws: LCA_OP_DECODE bytes for B.
 *
 * lca_combine_shards: parts [n_shards] shard records (any order),
 * w_uv [16][512][128] bf16 -> out [B][16][128] fp32 and, if not NULL,
 * o_lat [B][16][512] fp32.  No workspace. */
#define LCA_SHARD_RECORD_PER_HEAD 513
int lca_decode_shard(const void *cache_shard, const void *q_recent, const void *q, int B, int64_t L,
                     int64_t row0, int64_t L_shard, lca_params p, float *part, int32_t *anchor,
                     void *ws, size_t ws_bytes, void *stream);
int lca_combine_shards(const float *parts, int n_shards, int B, const void *w_uv, float *out,
                       float *o_lat, void *stream);

/* A decode loop's per-step bookkeeping in one launch (no counterpart on the
 * page, whose method starts from a cache that already holds the current
 * token): the current token's cache row of every sequence goes into row
 * `pos` of its cache, and its absorbed query into slot `slot` of the
 * recent-query ring that lca_decode and lca_condense take as q_recent (only
 * the ring's mean is used, so the oldest slot is the one to overwrite).
 *   rows  [B][576] bf16            the new rows
 *   cache [B][pitch][576] bf16     written at row pos, 0 <= pos < pitch
 *   q     [B][16][576] bf16        the new queries, or NULL (rows only)
 *   ring  [B][g][16][576] bf16     written at slot, 0 <= slot < g; NULL with q
 *   q_dst [B][16][576] bf16        NULL, or a second copy of q (the q that
 *                                  lca_decode takes), written alongside
 * 16-byte aligned; B * pitch < 2^40.  rows and q may be pinned host memory
 * (cudaHostAlloc / cudaMallocHost / cudaHostRegister, mapped at the same
 * address): the kernel then reads them over the host link, in place of a
 * host-to-device copy; the host must not change them until the call has
 * completed.  Every pointer is checked first (cudaPointerGetAttributes):
 * pageable host memory or an unknown address gives LCA_ERR_INVALID_ARG and
 * launches nothing.  The kernel waits for all earlier work in the stream
 * before it reads or writes, so an earlier kernel still reading the cache is
 * never overtaken; the next call in the stream (lca_decode, ...) sees the
 * writes. */
int lca_append_token(const void *rows, void *cache, int B, int64_t pitch, int64_t pos, const void *q,
                     void *ring, int g, int slot, void *q_dst, void *stream);

/* Self-test of the failure path (no counterpart on the page): launches one
 * kernel whose bounded wait can never be satisfied.  After ~2 s it records
 * LCA_ERR_DEVICE_TIMEOUT in the device status word (kernel id 8 in bits
 * 8..15 of lca_device_status's detail, wait site 1 in bits 16..23) and
 * returns; the context stays usable.  Asynchronous on `stream`. */
int lca_selftest_wait_timeout(void *stream);

/* Text for a status code (static storage). */
const char *lca_strerror(int status);

/* Reads (and if clear != 0 resets) the device status word of the current
 * device: LCA_OK or LCA_ERR_DEVICE_TIMEOUT with the kernel id in bits 8..15
 * of *detail.  Synchronises the device. */
int lca_device_status(int clear, int *detail);

/* Kernel timing.  lca_profile_enable(1) makes every later call record a
 * CUDA event pair around each kernel it launches (on the call's stream);
 * lca_profile_collect() waits for them, fills up to `max` entries
 * {name, launches, total_ms} and resets the record.  Returns the number of
 * entries or a negative status. */
typedef struct {
    char name[32];
    int launches;
    double total_ms;
} lca_kernel_time;
int lca_profile_enable(int on);
int lca_profile_collect(lca_kernel_time *out, int max);

/* Number of kernels this library has launched since it was loaded. */
int64_t lca_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* LCA_B200_H */
