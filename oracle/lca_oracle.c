/*
 * lca_oracle.c -- CPU oracle for MLA decode and latent-condensed attention
 * (LCA).  TEST INFRASTRUCTURE ONLY: the CUDA library never links, calls or
 * includes this file, and this file shares no code with it.  Only the tests,
 * the benchmark's CPU-baseline leg and the package smoke check use it.
 *
 * Source of every definition below: the page "Latent-Condensed Transformer
 * for Efficient Long Context Modeling" (papernotes.org notes on the ACL 2026
 * paper), sections 整体框架 (overall framework), 关键设计 1 (query-aware
 * weighted pooling, eq. c_j^rep = sum_i alpha_i^(j) c_i^KV), 关键设计 2
 * (positional anchor, eq. k_j^{R_rep} = k^R_{I_j}) and 关键设计 3 (local
 * window).  Constants the page leaves open (importance score, head count,
 * widths, softmax scale, prefill blocking) take their plainest reading:
 * importance s_i = (1/H) sum_h scale*(qbar_h . row_i) with the same scale
 * as the attention logits, the first index wins an exact argmax tie,
 * groups start at position 0 and leftover tokens join the window, and a
 * condensed representative carries no extra logit bias.
 *
 * Arithmetic: plain loops in fp64, in the order of the definitions.  bf16
 * inputs are widened exactly (bit shift).  OpenMP only splits independent
 * sequences, groups, heads or prefill blocks across threads; it never
 * changes the order of any sum.
 *
 * Layouts (row-major, contiguous):
 *   cache    [B][L][dc+dr]   bf16 bits: row = [c^KV (dc) | k^R (dr)]
 *   q        [B][H][dc+dr]   bf16 bits, absorbed query (q_lat | q_rope)
 *   q_recent [B][g][H][dc+dr] bf16 bits, the last g queries (last = current)
 *   w_uv     [H][dc][dv]     bf16 bits
 *   qpre     [B][L][H][dc+dr] bf16 bits (prefill queries)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf(uint16_t x)
{
    uint32_t u = (uint32_t)x << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int ora_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* 整体框架: history outside the window of w recent tokens is cut into
 * m = floor((L - w) / g) groups; m = 0 when L <= w. */
long ora_num_groups(long L, int g, int w)
{
    if (g <= 0 || L <= (long)w) return 0;
    return (L - (long)w) / g;
}

/* 关键设计 1: the summary query is the mean of the most recent g queries. */
static void summary_query(const uint16_t *qr, int g, int H, int D, double *qbar)
{
    for (int h = 0; h < H; h++)
        for (int k = 0; k < D; k++) {
            double s = 0.0;
            for (int t = 0; t < g; t++) s += bf(qr[((size_t)t * H + h) * D + k]);
            qbar[(size_t)h * D + k] = s / g;
        }
}

/* Importance of one cached row under a (per-head) query set qv[H][D]:
 * s = (1/H) sum_h scale * (q_lat,h . c + q_rope,h . k^R). */
static double importance(const double *qv, const uint16_t *row, int H, int dc, int dr,
                         double scale)
{
    int D = dc + dr;
    double acc = 0.0;
    for (int h = 0; h < H; h++) {
        double lat = 0.0, rope = 0.0;
        for (int k = 0; k < dc; k++) lat += qv[(size_t)h * D + k] * bf(row[k]);
        for (int k = 0; k < dr; k++) rope += qv[(size_t)h * D + dc + k] * bf(row[dc + k]);
        acc += scale * (lat + rope);
    }
    return acc / H;
}

/* Condensation variants: the method (关键设计 1 + 2) and the two ablations of
 * the page's 消融实验 table. */
enum { ORA_LCA = 0, ORA_POOL_POSITION = 1, ORA_SPARSE = 2 };

/* 关键设计 1 + 2 for one group of g rows starting at `rows`:
 * alpha = softmax(s) over the group, rep_c = sum_i alpha_i c_i,
 * I = argmax_i s_i (first index on an exact tie), rep_k = k^R_I.
 * forced >= 0 replaces the argmax by that offset ("forced-anchor" mode: the
 * result for another valid choice of I where the maximum is a near-tie);
 * nothing else changes.
 * Ablations (消融实验): ORA_POOL_POSITION pools the RoPE key with the same
 * weights, rep_k = sum_i alpha_i k^R_i ("纯池化（含位置）"); ORA_SPARSE keeps
 * only the most important token, rep_c = c_I, rep_k = k^R_I ("纯稀疏").
 * Returns I (offset inside the group). */
static int condense_group_v(const double *qv, const uint16_t *rows, int g, int H, int dc, int dr,
                            double scale, int variant, int forced, double *rep_c, double *rep_k,
                            double *alpha_out, double *score_out)
{
    int D = dc + dr;
    double *s = (double *)malloc(sizeof(double) * g);
    double *a = (double *)malloc(sizeof(double) * g);
    for (int i = 0; i < g; i++) s[i] = importance(qv, rows + (size_t)i * D, H, dc, dr, scale);
    int I = 0;
    double mx = s[0];
    for (int i = 1; i < g; i++)
        if (s[i] > mx) { mx = s[i]; I = i; }
    if (forced >= 0) I = forced;
    double den = 0.0;
    for (int i = 0; i < g; i++) { a[i] = exp(s[i] - mx); den += a[i]; }
    for (int i = 0; i < g; i++) a[i] /= den;
    for (int k = 0; k < dc; k++) {
        double acc = 0.0;
        if (variant == ORA_SPARSE) {
            acc = bf(rows[(size_t)I * D + k]);
        } else {
            for (int i = 0; i < g; i++) acc += a[i] * bf(rows[(size_t)i * D + k]);
        }
        rep_c[k] = acc;
    }
    for (int k = 0; k < dr; k++) {
        if (variant == ORA_POOL_POSITION) {
            double acc = 0.0;
            for (int i = 0; i < g; i++) acc += a[i] * bf(rows[(size_t)i * D + dc + k]);
            rep_k[k] = acc;
        } else {
            rep_k[k] = bf(rows[(size_t)I * D + dc + k]);
        }
    }
    if (alpha_out) for (int i = 0; i < g; i++) alpha_out[i] = a[i];
    if (score_out) for (int i = 0; i < g; i++) score_out[i] = s[i];
    free(s);
    free(a);
    return I;
}

/* Forced anchor of group j, or -1 for the argmax: anchor_in [B][m] holds
 * absolute positions (NULL = no forcing).  Returns -2 for a position
 * outside the group, which the callers report as an error. */
static int forced_offset(const int32_t *anchor_in, size_t o, long j, int g)
{
    if (!anchor_in) return -1;
    long off = (long)anchor_in[o] - j * g;
    return (off >= 0 && off < g) ? (int)off : -2;
}

/* Condense every group of every sequence (decode: summary query from
 * q_recent).  Outputs (any may be NULL except none are required):
 * rep_c [B][m][dc], rep_k [B][m][dr], anchor [B][m] (absolute position
 * inside the sequence), alpha [B][m][g], score [B][m][g].  `variant`
 * selects the method or one of its ablations (condense_group_v).
 * anchor_in [B][m] (absolute positions, or NULL) forces each group's anchor
 * (forced-anchor mode); returns -2 if one lies outside its group. */
int ora_lca_condense_fv(const uint16_t *cache, const uint16_t *q_recent, int B, long L, int H,
                        int dc, int dr, int g, int w, double scale, int variant,
                        const int32_t *anchor_in, double *rep_c, double *rep_k, int32_t *anchor,
                        double *alpha, double *score)
{
    int D = dc + dr;
    long m = ora_num_groups(L, g, w);
    if (m == 0) return 0;
    if (anchor_in)
        for (int b = 0; b < B; b++)
            for (long j = 0; j < m; j++)
                if (forced_offset(anchor_in, (size_t)b * m + j, j, g) < 0) return -2;
    double *qbar = (double *)malloc(sizeof(double) * (size_t)B * H * D);
    for (int b = 0; b < B; b++)
        summary_query(q_recent + (size_t)b * g * H * D, g, H, D, qbar + (size_t)b * H * D);
#pragma omp parallel
    {
        double *rc = (double *)malloc(sizeof(double) * dc);
        double *rk = (double *)malloc(sizeof(double) * dr);
        double *al = (double *)malloc(sizeof(double) * g);
        double *sc = (double *)malloc(sizeof(double) * g);
#pragma omp for collapse(2) schedule(static)
        for (int b = 0; b < B; b++)
            for (long j = 0; j < m; j++) {
                const uint16_t *rows = cache + ((size_t)b * L + (size_t)j * g) * D;
                size_t o = (size_t)b * m + j;
                int I = condense_group_v(qbar + (size_t)b * H * D, rows, g, H, dc, dr, scale,
                                         variant, forced_offset(anchor_in, o, j, g), rc, rk, al,
                                         sc);
                if (rep_c) memcpy(rep_c + o * dc, rc, sizeof(double) * dc);
                if (rep_k) memcpy(rep_k + o * dr, rk, sizeof(double) * dr);
                if (anchor) anchor[o] = (int32_t)(j * g + I);
                if (alpha) memcpy(alpha + o * g, al, sizeof(double) * g);
                if (score) memcpy(score + o * g, sc, sizeof(double) * g);
            }
        free(rc);
        free(rk);
        free(al);
        free(sc);
    }
    free(qbar);
    return 0;
}

int ora_lca_condense_v(const uint16_t *cache, const uint16_t *q_recent, int B, long L, int H,
                       int dc, int dr, int g, int w, double scale, int variant, double *rep_c,
                       double *rep_k, int32_t *anchor, double *alpha, double *score)
{
    return ora_lca_condense_fv(cache, q_recent, B, L, H, dc, dr, g, w, scale, variant, NULL,
                               rep_c, rep_k, anchor, alpha, score);
}

int ora_lca_condense(const uint16_t *cache, const uint16_t *q_recent, int B, long L, int H,
                     int dc, int dr, int g, int w, double scale, double *rep_c, double *rep_k,
                     int32_t *anchor, double *alpha, double *score)
{
    return ora_lca_condense_v(cache, q_recent, B, L, H, dc, dr, g, w, scale, ORA_LCA, rep_c,
                              rep_k, anchor, alpha, score);
}

/* 整体框架: standard attention of one query token (H heads, absorbed
 * form) over n_rep fp64 representative rows followed by n_win cache rows:
 * z_hr = scale * (q_lat,h . c_r + q_rope,h . k_r), p = softmax_r(z),
 * o_lat,h = sum_r p_r c_r.  Representatives carry no extra bias. */
static void attend_head_lse(const uint16_t *qh, int dc, int dr, double scale, long n_rep,
                            const double *rep_c, const double *rep_k, const uint16_t *rep_bf,
                            const uint16_t *win, long n_win, double *o, double *lse)
{
    int D = dc + dr;
    long n = n_rep + n_win;
    double *z = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
    for (long r = 0; r < n; r++) {
        double lat = 0.0, rope = 0.0;
        if (r < n_rep) {
            if (rep_bf) {
                const uint16_t *row = rep_bf + (size_t)r * D;
                for (int k = 0; k < dc; k++) lat += bf(qh[k]) * bf(row[k]);
                for (int k = 0; k < dr; k++) rope += bf(qh[dc + k]) * bf(row[dc + k]);
            } else {
                for (int k = 0; k < dc; k++) lat += bf(qh[k]) * rep_c[(size_t)r * dc + k];
                for (int k = 0; k < dr; k++) rope += bf(qh[dc + k]) * rep_k[(size_t)r * dr + k];
            }
        } else {
            const uint16_t *row = win + (size_t)(r - n_rep) * D;
            for (int k = 0; k < dc; k++) lat += bf(qh[k]) * bf(row[k]);
            for (int k = 0; k < dr; k++) rope += bf(qh[dc + k]) * bf(row[dc + k]);
        }
        z[r] = scale * (lat + rope);
    }
    double mx = -INFINITY;
    for (long r = 0; r < n; r++)
        if (z[r] > mx) mx = z[r];
    double den = 0.0;
    for (long r = 0; r < n; r++) { z[r] = exp(z[r] - mx); den += z[r]; }
    for (int k = 0; k < dc; k++) {
        double acc = 0.0;
        for (long r = 0; r < n; r++) {
            double c;
            if (r < n_rep)
                c = rep_bf ? bf(rep_bf[(size_t)r * D + k]) : rep_c[(size_t)r * dc + k];
            else
                c = bf(win[(size_t)(r - n_rep) * D + k]);
            acc += z[r] * c;
        }
        o[k] = acc / den;
    }
    /* log sum_r exp(z_r), for merging attention over disjoint row sets */
    if (lse) *lse = mx + log(den);
    free(z);
}

static void attend_head(const uint16_t *qh, int dc, int dr, double scale, long n_rep,
                        const double *rep_c, const double *rep_k, const uint16_t *rep_bf,
                        const uint16_t *win, long n_win, double *o)
{
    attend_head_lse(qh, dc, dr, scale, n_rep, rep_c, rep_k, rep_bf, win, n_win, o, NULL);
}

/* Per-head value up-projection out_h = W_UV[h]^T o_lat,h (W_UV [H][dc][dv]). */
static void up_project(const double *o_lat, const uint16_t *w_uv, int H, int dc, int dv,
                       double *out)
{
    for (int h = 0; h < H; h++)
        for (int v = 0; v < dv; v++) {
            double acc = 0.0;
            for (int k = 0; k < dc; k++)
                acc += o_lat[(size_t)h * dc + k] * bf(w_uv[((size_t)h * dc + k) * dv + v]);
            out[(size_t)h * dv + v] = acc;
        }
}

/* MLA decode: the query at position L-1 attends all L cached rows. */
int ora_mla_decode(const uint16_t *cache, const uint16_t *q, const uint16_t *w_uv, int B, long L,
                   int H, int dc, int dr, int dv, double scale, double *o_lat, double *out)
{
    int D = dc + dr;
    double *ol = (double *)malloc(sizeof(double) * (size_t)B * H * dc);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            attend_head(q + ((size_t)b * H + h) * D, dc, dr, scale, 0, NULL, NULL, NULL,
                        cache + (size_t)b * L * D, L, ol + ((size_t)b * H + h) * dc);
    for (int b = 0; b < B; b++) {
        if (out) up_project(ol + (size_t)b * H * dc, w_uv, H, dc, dv, out + (size_t)b * H * dv);
    }
    if (o_lat) memcpy(o_lat, ol, sizeof(double) * (size_t)B * H * dc);
    free(ol);
    return 0;
}

/* LCA decode: condense the m groups with the summary query of q_recent,
 * then the current query q attends [m representatives || window rows
 * m*g .. L-1].  anchor_out [B][m] may be NULL.  anchor_in [B][m] (absolute
 * positions) or NULL: forced anchors (ora_lca_condense_fv). */
int ora_lca_decode_f(const uint16_t *cache, const uint16_t *q_recent, const uint16_t *q,
                     const uint16_t *w_uv, int B, long L, int H, int dc, int dr, int dv, int g,
                     int w, double scale, const int32_t *anchor_in, double *o_lat, double *out,
                     int32_t *anchor_out)
{
    int D = dc + dr;
    long m = ora_num_groups(L, g, w);
    double *rc = (double *)malloc(sizeof(double) * (size_t)B * (m > 0 ? m : 1) * dc);
    double *rk = (double *)malloc(sizeof(double) * (size_t)B * (m > 0 ? m : 1) * dr);
    int rcode = ora_lca_condense_fv(cache, q_recent, B, L, H, dc, dr, g, w, scale, ORA_LCA,
                                    anchor_in, rc, rk, anchor_out, NULL, NULL);
    if (rcode) { free(rc); free(rk); return rcode; }
    double *ol = (double *)malloc(sizeof(double) * (size_t)B * H * dc);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            attend_head(q + ((size_t)b * H + h) * D, dc, dr, scale, m, rc + (size_t)b * m * dc,
                        rk + (size_t)b * m * dr, NULL, cache + ((size_t)b * L + (size_t)m * g) * D,
                        L - m * g, ol + ((size_t)b * H + h) * dc);
    for (int b = 0; b < B; b++)
        if (out) up_project(ol + (size_t)b * H * dc, w_uv, H, dc, dv, out + (size_t)b * H * dv);
    if (o_lat) memcpy(o_lat, ol, sizeof(double) * (size_t)B * H * dc);
    free(ol);
    free(rc);
    free(rk);
    return 0;
}

int ora_lca_decode(const uint16_t *cache, const uint16_t *q_recent, const uint16_t *q,
                   const uint16_t *w_uv, int B, long L, int H, int dc, int dr, int dv, int g,
                   int w, double scale, double *o_lat, double *out, int32_t *anchor_out)
{
    return ora_lca_decode_f(cache, q_recent, q, w_uv, B, L, H, dc, dr, dv, g, w, scale, NULL,
                            o_lat, out, anchor_out);
}

/* One shard of the LCA decode attention: the rows row0 .. row1-1 of each
 * sequence (row0 a multiple of g).  The groups among them (those below
 * m*g) are condensed exactly as in ora_lca_decode, and the current query
 * attends [those representatives || the shard's window rows] alone:
 * o_part [B][H][dc] is normalised over the shard's rows and
 * lse [B][H] = log sum exp(z) over them.  anchor_out [B][m_shard] (or NULL)
 * receives absolute positions.  anchor_in [B][m] (absolute positions of
 * every group of the sequence) or NULL: forced anchors. */
int ora_lca_decode_shard_f(const uint16_t *cache, const uint16_t *q_recent, const uint16_t *q,
                           int B, long L, int H, int dc, int dr, int g, int w, double scale,
                           long row0, long row1, const int32_t *anchor_in, double *o_part,
                           double *lse, int32_t *anchor_out)
{
    int D = dc + dr;
    long m = ora_num_groups(L, g, w);
    long hist_end = m * g;
    long j0 = row0 / g, j1 = (row1 < hist_end ? row1 : hist_end) / g;
    long n_rep = j1 > j0 ? j1 - j0 : 0;
    long wstart = row0 > hist_end ? row0 : hist_end;
    long n_win = row1 > wstart ? row1 - wstart : 0;
    if (row0 % g != 0 || row1 <= row0 || row1 > L) return -1;
    double *rc = (double *)malloc(sizeof(double) * (size_t)B * (m > 0 ? m : 1) * dc);
    double *rk = (double *)malloc(sizeof(double) * (size_t)B * (m > 0 ? m : 1) * dr);
    int32_t *an = (int32_t *)malloc(sizeof(int32_t) * (size_t)B * (m > 0 ? m : 1));
    int rcode = ora_lca_condense_fv(cache, q_recent, B, L, H, dc, dr, g, w, scale, ORA_LCA,
                                    anchor_in, rc, rk, an, NULL, NULL);
    if (rcode) { free(an); free(rc); free(rk); return rcode; }
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            attend_head_lse(q + ((size_t)b * H + h) * D, dc, dr, scale, n_rep,
                            rc + ((size_t)b * m + j0) * dc, rk + ((size_t)b * m + j0) * dr, NULL,
                            cache + ((size_t)b * L + wstart) * D, n_win,
                            o_part + ((size_t)b * H + h) * dc, lse + (size_t)b * H + h);
    if (anchor_out)
        for (int b = 0; b < B; b++)
            for (long j = 0; j < n_rep; j++)
                anchor_out[(size_t)b * n_rep + j] = an[(size_t)b * m + j0 + j];
    free(an);
    free(rc);
    free(rk);
    return 0;
}

int ora_lca_decode_shard(const uint16_t *cache, const uint16_t *q_recent, const uint16_t *q, int B,
                         long L, int H, int dc, int dr, int g, int w, double scale, long row0,
                         long row1, double *o_part, double *lse, int32_t *anchor_out)
{
    return ora_lca_decode_shard_f(cache, q_recent, q, B, L, H, dc, dr, g, w, scale, row0, row1,
                                  NULL, o_part, lse, anchor_out);
}

/* LCA decode attention over representatives supplied as bf16 rows
 * rep[B][m][dc+dr] (a cache-format copy of condensed groups), followed by
 * the window rows m*g .. L-1 of the cache. */
int ora_lca_attend_reps(const uint16_t *cache, const uint16_t *rep, const uint16_t *q,
                        const uint16_t *w_uv, int B, long L, int H, int dc, int dr, int dv, int g,
                        int w, double scale, double *o_lat, double *out)
{
    int D = dc + dr;
    long m = ora_num_groups(L, g, w);
    double *ol = (double *)malloc(sizeof(double) * (size_t)B * H * dc);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            attend_head(q + ((size_t)b * H + h) * D, dc, dr, scale, m, NULL, NULL,
                        rep + (size_t)b * m * D, cache + ((size_t)b * L + (size_t)m * g) * D,
                        L - m * g, ol + ((size_t)b * H + h) * dc);
    for (int b = 0; b < B; b++)
        if (out) up_project(ol + (size_t)b * H * dc, w_uv, H, dc, dv, out + (size_t)b * H * dv);
    if (o_lat) memcpy(o_lat, ol, sizeof(double) * (size_t)B * H * dc);
    free(ol);
    return 0;
}

/* Blockwise LCA prefill.  Query positions are cut into blocks of g
 * (block k covers t0 = k*g .. t0+g-1).  For each block: the summary query
 * is the mean of its own g queries; history 0 .. m_k*g-1 with
 * m_k = floor((t0 - w)/g) (0 when t0 <= w) is condensed with it; every
 * query t of the block attends [m_k representatives || rows m_k*g .. t]
 * (causal, itself included).  Blocks processed: all blocks of
 * [q_start, q_start+q_len) (both multiples of g) when blocks == NULL,
 * else the n_blocks absolute block indices listed in `blocks` (each inside
 * that range).  Outputs are indexed by t - q_start:
 * o_lat [B][q_len][H][dc], out [B][q_len][H][dv]; rows of blocks that are
 * not processed are left untouched.  anchor_out, if not NULL, receives
 * [B][q_len/g][m_max] absolute anchor positions (m_max = max m_k over the
 * range, unused slots untouched).  `variant` selects the representative as
 * in condense_group_v: the method or one of the two ablations.  anchor_in
 * (NULL, or laid out like anchor_out) forces the anchors of the processed
 * blocks (forced-anchor mode); returns -2 if one lies outside its group. */
int ora_lca_prefill_fv(const uint16_t *cache, const uint16_t *qpre, const uint16_t *w_uv, int B,
                       long L, long q_start, long q_len, int H, int dc, int dr, int dv, int g,
                       int w, double scale, int variant, const int64_t *blocks, long n_blocks,
                       const int32_t *anchor_in, double *o_lat, double *out, int32_t *anchor_out)
{
    int D = dc + dr;
    if (q_start % g || q_len % g || q_start < 0 || q_start + q_len > L) return -1;
    long nb_range = q_len / g;
    long nb = blocks ? n_blocks : nb_range;
    long m_max = ora_num_groups(q_start + q_len - g, g, w);
    size_t m_row = (size_t)(m_max > 0 ? m_max : 1);
    if (anchor_in)
        for (int b = 0; b < B; b++)
            for (long bi = 0; bi < nb; bi++) {
                long k = blocks ? blocks[bi] : q_start / g + bi;
                if (k * g < q_start || k * g + g > q_start + q_len) continue;
                long m = ora_num_groups(k * g, g, w);
                size_t base = ((size_t)b * nb_range + (size_t)(k - q_start / g)) * m_row;
                for (long j = 0; j < m; j++)
                    if (forced_offset(anchor_in, base + (size_t)j, j, g) < 0) return -2;
            }
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (long bi = 0; bi < nb; bi++) {
            long k = blocks ? blocks[bi] : q_start / g + bi;
            long t0 = k * g;
            if (t0 < q_start || t0 + g > q_start + q_len) continue;
            long m = ora_num_groups(t0, g, w);
            const uint16_t *seq = cache + (size_t)b * L * D;
            const uint16_t *qb = qpre + ((size_t)b * L + t0) * H * D; /* [g][H][D] */
            double *qbar = (double *)malloc(sizeof(double) * H * D);
            summary_query(qb, g, H, D, qbar);
            double *rc = (double *)malloc(sizeof(double) * (m > 0 ? m : 1) * dc);
            double *rk = (double *)malloc(sizeof(double) * (m > 0 ? m : 1) * dr);
            size_t abase = ((size_t)b * nb_range + (size_t)(k - q_start / g)) * m_row;
            for (long j = 0; j < m; j++) {
                int I = condense_group_v(qbar, seq + (size_t)j * g * D, g, H, dc, dr, scale, variant,
                                         forced_offset(anchor_in, abase + (size_t)j, j, g),
                                         rc + (size_t)j * dc, rk + (size_t)j * dr, NULL, NULL);
                if (anchor_out) anchor_out[abase + (size_t)j] = (int32_t)(j * g + I);
            }
            double *ol = (double *)malloc(sizeof(double) * H * dc);
            for (int tt = 0; tt < g; tt++) {
                long t = t0 + tt;
                for (int h = 0; h < H; h++)
                    attend_head(qpre + (((size_t)b * L + t) * H + h) * D, dc, dr, scale, m, rc, rk,
                                NULL, seq + (size_t)m * g * D, t + 1 - m * g,
                                ol + (size_t)h * dc);
                size_t row = (size_t)b * q_len + (size_t)(t - q_start);
                if (o_lat) memcpy(o_lat + row * H * dc, ol, sizeof(double) * H * dc);
                if (out) up_project(ol, w_uv, H, dc, dv, out + row * H * dv);
            }
            free(ol);
            free(rc);
            free(rk);
            free(qbar);
        }
    return 0;
}

int ora_lca_prefill_v(const uint16_t *cache, const uint16_t *qpre, const uint16_t *w_uv, int B,
                      long L, long q_start, long q_len, int H, int dc, int dr, int dv, int g, int w,
                      double scale, int variant, const int64_t *blocks, long n_blocks, double *o_lat,
                      double *out, int32_t *anchor_out)
{
    return ora_lca_prefill_fv(cache, qpre, w_uv, B, L, q_start, q_len, H, dc, dr, dv, g, w, scale,
                              variant, blocks, n_blocks, NULL, o_lat, out, anchor_out);
}

/* The method's prefill (variant ORA_LCA). */
int ora_lca_prefill(const uint16_t *cache, const uint16_t *qpre, const uint16_t *w_uv, int B,
                    long L, long q_start, long q_len, int H, int dc, int dr, int dv, int g, int w,
                    double scale, const int64_t *blocks, long n_blocks, double *o_lat,
                    double *out, int32_t *anchor_out)
{
    return ora_lca_prefill_v(cache, qpre, w_uv, B, L, q_start, q_len, H, dc, dr, dv, g, w, scale,
                             ORA_LCA, blocks, n_blocks, o_lat, out, anchor_out);
}

/* Stored-representative decode: the reading of the page's "90% KV-cache
 * compression" (一句话总结, 关键发现) in which a group is condensed once and
 * kept.  Group j leaves the window at the decode step whose cache length is
 * L_j = w + g (j + 1) (the first L with floor((L - w)/g) > j); it is condensed
 * then, with the summary query of that step: the mean of the g queries at
 * positions L_j - g .. L_j - 1 (关键设计 1, 2).  The decode step at length L
 * attends [the m(L) kept representatives || rows m g .. L-1] with the query
 * at position L - 1 (整体框架).
 *   q_all [B][L][H][D] holds the query of every position.
 *   anchor_out [B][m] (absolute positions) may be NULL.
 *   anchor_in [B][m] (absolute positions) or NULL: forced anchors. */
int ora_lca_decode_stored_f(const uint16_t *cache, const uint16_t *q_all, const uint16_t *w_uv,
                            int B, long L, int H, int dc, int dr, int dv, int g, int w,
                            double scale, const int32_t *anchor_in, double *o_lat, double *out,
                            int32_t *anchor_out)
{
    int D = dc + dr;
    long m = ora_num_groups(L, g, w);
    if (anchor_in)
        for (int b = 0; b < B; b++)
            for (long j = 0; j < m; j++)
                if (forced_offset(anchor_in, (size_t)b * m + j, j, g) < 0) return -2;
    size_t mm = (size_t)(m > 0 ? m : 1);
    double *rc = (double *)malloc(sizeof(double) * (size_t)B * mm * dc);
    double *rk = (double *)malloc(sizeof(double) * (size_t)B * mm * dr);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (long j = 0; j < m; j++) {
            long Lj = (long)w + (long)g * (j + 1);
            double *qbar = (double *)malloc(sizeof(double) * H * D);
            summary_query(q_all + ((size_t)b * L + (size_t)(Lj - g)) * H * D, g, H, D, qbar);
            int I = condense_group_v(qbar, cache + ((size_t)b * L + (size_t)j * g) * D, g, H, dc,
                                     dr, scale, ORA_LCA,
                                     forced_offset(anchor_in, (size_t)b * m + j, j, g),
                                     rc + ((size_t)b * mm + j) * dc,
                                     rk + ((size_t)b * mm + j) * dr, NULL, NULL);
            if (anchor_out) anchor_out[(size_t)b * m + j] = (int32_t)(j * g + I);
            free(qbar);
        }
    double *ol = (double *)malloc(sizeof(double) * (size_t)B * H * dc);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            attend_head(q_all + (((size_t)b * L + (size_t)(L - 1)) * H + h) * D, dc, dr, scale,
                        m, rc + (size_t)b * mm * dc, rk + (size_t)b * mm * dr, NULL,
                        cache + ((size_t)b * L + (size_t)m * g) * D, L - m * g,
                        ol + ((size_t)b * H + h) * dc);
    for (int b = 0; b < B; b++)
        if (out) up_project(ol + (size_t)b * H * dc, w_uv, H, dc, dv, out + (size_t)b * H * dv);
    if (o_lat) memcpy(o_lat, ol, sizeof(double) * (size_t)B * H * dc);
    free(ol);
    free(rc);
    free(rk);
    return 0;
}

int ora_lca_decode_stored(const uint16_t *cache, const uint16_t *q_all, const uint16_t *w_uv,
                          int B, long L, int H, int dc, int dr, int dv, int g, int w,
                          double scale, double *o_lat, double *out, int32_t *anchor_out)
{
    return ora_lca_decode_stored_f(cache, q_all, w_uv, B, L, H, dc, dr, dv, g, w, scale, NULL,
                                   o_lat, out, anchor_out);
}
