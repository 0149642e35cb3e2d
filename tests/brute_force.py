"""Brute-force restatement of latent-condensed attention for tiny inputs.

Test infrastructure, independent of both the C oracle and the CUDA path: it
imports neither, uses no numpy linear algebra, and reads its inputs as plain
Python lists of bf16 bit patterns.  Source: "Latent-Condensed Transformer for
Efficient Long Context Modeling" (papernotes.org notes on the ACL 2026
paper), 整体框架 (history cut into groups of g outside a window of w recent
tokens, attention over [representatives || window]), 关键设计 1 (pooling with
the softmax of the importance under the mean of the last g queries),
关键设计 2 (the anchor's RoPE key), 关键设计 3 (the window stays uncompressed)
and 消融实验 (the two ablations).

It differs from the oracle in how it reaches every intermediate result:

* groups and window are found by walking the positions (a group is taken
  while at least w tokens remain after it), not by the floor formula;
* bf16 values are decoded from their bits by hand into exact Fractions;
* importance scores are exact rationals (the positive factor scale/H is
  left out, which changes neither the argmax nor the softmax once it is put
  back), so anchors and ties are decided exactly;
* the softmaxes, pools and attention run in fp64 with math.fsum (correctly
  rounded sums), so they agree with the oracle's plain fp64 loops to ~1e-12.
"""
from __future__ import annotations

import math
from fractions import Fraction

LCA, POOL_POSITION, SPARSE = 0, 1, 2


def bf16_fraction(bits: int) -> Fraction:
    """Exact value of a finite bf16 bit pattern (1 sign, 8 exponent, 7
    mantissa bits)."""
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    man = bits & 0x7F
    assert e != 0xFF, "inf / nan are not valid inputs"
    if e == 0:
        v = Fraction(man, 128) * Fraction(2) ** -126
    else:
        v = Fraction(128 + man, 128) * Fraction(2) ** (e - 127)
    return sign * v


def walk_groups(L: int, g: int, w: int):
    """Group boundaries by walking: from position 0, take the next g
    positions as a group while at least w positions are left after it.
    -> (list of (start, end) groups, window start)."""
    groups = []
    start = 0
    while start + g + w <= L:
        groups.append((start, start + g))
        start += g
    return groups, start


def _dot_exact(a, b):
    return sum((x * y for x, y in zip(a, b)), Fraction(0))


def _softmax(vals):
    mx = max(vals)
    e = [math.exp(v - mx) for v in vals]
    den = math.fsum(e)
    return [x / den for x in e], mx + math.log(den)


class Problem:
    """Bit patterns -> exact values, for one sequence.

    rows [L][D] bf16 bits (D = dc + dr, row = [c | k^R]); queries are
    [H][D] bf16 bits; w_uv [H][dc][dv] bf16 bits."""

    def __init__(self, rows, dc, dr, w_uv, scale):
        self.dc, self.dr = dc, dr
        self.D = dc + dr
        self.rows = [[bf16_fraction(int(x)) for x in r] for r in rows]
        self.rowsf = [[float(x) for x in r] for r in self.rows]
        self.w_uv = [[[float(bf16_fraction(int(x))) for x in col] for col in head] for head in w_uv]
        self.scale = scale

    def summary_query(self, queries):
        """Mean of the given queries ([t][H][D] bits), exact."""
        g = len(queries)
        H = len(queries[0])
        return [[sum((bf16_fraction(int(queries[t][h][k])) for t in range(g)), Fraction(0)) / g
                 for k in range(self.D)] for h in range(H)]

    def condense(self, qbar, start, end, variant=LCA, forced=None):
        """One group [start, end): exact importance (times H/scale), first
        argmax, fp64 softmax weights, pooled latent and representative key.
        -> dict(anchor (absolute), alpha, rep_c, rep_k, score_exact)."""
        H = len(qbar)
        # s_i * H / scale = sum_h qbar_h . row_i  (exact)
        exact = [sum((_dot_exact(qbar[h], self.rows[i]) for h in range(H)), Fraction(0))
                 for i in range(start, end)]
        best = 0
        for i in range(1, len(exact)):
            if exact[i] > exact[best]:
                best = i
        if forced is not None:
            best = forced - start
        top = max(exact)
        coef = self.scale / H
        alpha, _ = _softmax([float(s - top) * coef for s in exact])
        grp = self.rowsf[start:end]
        if variant == SPARSE:
            rep_c = list(grp[best][:self.dc])
        else:
            rep_c = [math.fsum(alpha[i] * grp[i][k] for i in range(len(grp))) for k in range(self.dc)]
        if variant == POOL_POSITION:
            rep_k = [math.fsum(alpha[i] * grp[i][self.dc + k] for i in range(len(grp)))
                     for k in range(self.dr)]
        else:
            rep_k = list(grp[best][self.dc:])
        return dict(anchor=start + best, alpha=alpha, rep_c=rep_c, rep_k=rep_k, score_exact=exact)

    def attend(self, qh_bits, reps, win_rows):
        """Standard attention of one head's query over [reps || window rows].
        -> (o_lat [dc], natural log-sum-exp of the logits)."""
        qh = [float(bf16_fraction(int(x))) for x in qh_bits]
        keys = [r["rep_c"] + r["rep_k"] for r in reps] + [self.rowsf[i] for i in win_rows]
        z = [self.scale * math.fsum(qh[k] * key[k] for k in range(self.D)) for key in keys]
        p, lse = _softmax(z)
        o = [math.fsum(p[r] * keys[r][k] for r in range(len(keys))) for k in range(self.dc)]
        return o, lse

    def up_project(self, o_lat):
        """out_h = W_UV[h]^T o_lat,h."""
        H = len(o_lat)
        dv = len(self.w_uv[0][0])
        return [[math.fsum(o_lat[h][k] * self.w_uv[h][k][v] for k in range(self.dc)) for v in range(dv)]
                for h in range(H)]


def decode(rows, q_recent, q, w_uv, dc, dr, g, w, scale, variant=LCA, forced=None):
    """One decode step of one sequence (cache of length L = len(rows), query
    at position L-1).  q_recent [g][H][D] bits, q [H][D] bits.
    -> dict(groups, window_start, anchors, alpha, rep_c, rep_k, o_lat, out, exact_scores)."""
    P = Problem(rows, dc, dr, w_uv, scale)
    L = len(rows)
    groups, win0 = walk_groups(L, g, w)
    qbar = P.summary_query(q_recent) if groups else None
    reps = [P.condense(qbar, s, e, variant, None if forced is None else forced[j])
            for j, (s, e) in enumerate(groups)]
    o_lat = [P.attend(q[h], reps, range(win0, L))[0] for h in range(len(q))]
    return dict(groups=groups, window_start=win0, anchors=[r["anchor"] for r in reps],
                alpha=[r["alpha"] for r in reps], rep_c=[r["rep_c"] for r in reps],
                rep_k=[r["rep_k"] for r in reps], exact_scores=[r["score_exact"] for r in reps],
                o_lat=o_lat, out=P.up_project(o_lat))


def mla_decode(rows, q, w_uv, dc, dr, scale):
    """Exact MLA: the query attends every cached row."""
    P = Problem(rows, dc, dr, w_uv, scale)
    o_lat = [P.attend(q[h], [], range(len(rows)))[0] for h in range(len(q))]
    return dict(o_lat=o_lat, out=P.up_project(o_lat))


def prefill(rows, queries, w_uv, dc, dr, g, w, scale, variant=LCA):
    """Blockwise prefill of one whole sequence: block b covers queries
    [b g, b g + g); its summary query is the mean of those g queries; the
    history before (b g - w) is grouped by walking and condensed with it;
    query t attends [representatives || rows from the end of the last group
    through t].  queries [L][H][D] bits.
    -> dict(o_lat [L][H][dc], out [L][H][dv], anchors [n_blocks][m_b])."""
    P = Problem(rows, dc, dr, w_uv, scale)
    L = len(rows)
    o_all, out_all, anchors = [], [], []
    for t0 in range(0, L - g + 1, g):
        groups, win0 = walk_groups(t0, g, w)
        # the walk over a prefix of length t0 stops where t0 - w positions
        # cannot hold another group; the block's window starts there
        qbar = P.summary_query(queries[t0:t0 + g]) if groups else None
        reps = [P.condense(qbar, s, e, variant) for s, e in groups]
        anchors.append([r["anchor"] for r in reps])
        for t in range(t0, t0 + g):
            o = [P.attend(queries[t][h], reps, range(win0, t + 1))[0] for h in range(len(queries[t]))]
            o_all.append(o)
            out_all.append(P.up_project(o))
    return dict(o_lat=o_all, out=out_all, anchors=anchors)


def decode_stored(rows, queries, w_uv, dc, dr, g, w, scale):
    """Stored-representative decode at cache length L = len(rows): walking
    L' = 1 .. L, a group that first appears at length L' is condensed then,
    with the mean of the queries at positions L'-g .. L'-1, and kept; the
    query at L-1 attends [kept representatives || window].
    queries [L][H][D] bits.  -> dict(anchors, o_lat, out)."""
    P = Problem(rows, dc, dr, w_uv, scale)
    L = len(rows)
    kept = []
    for Lp in range(1, L + 1):
        groups, _ = walk_groups(Lp, g, w)
        while len(kept) < len(groups):
            s, e = groups[len(kept)]
            kept.append(P.condense(P.summary_query(queries[Lp - g:Lp]), s, e))
    _, win0 = walk_groups(L, g, w)
    q = queries[L - 1]
    o_lat = [P.attend(q[h], kept, range(win0, L))[0] for h in range(len(q))]
    return dict(anchors=[r["anchor"] for r in kept], o_lat=o_lat, out=P.up_project(o_lat))
