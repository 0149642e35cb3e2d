"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a value the page prints, a closed form, an invariant, or a
special case that reduces to a textbook computation done independently here
(explicitly decompressed multi-head attention in numpy).  Definitions follow
"Latent-Condensed Transformer for Efficient Long Context Modeling"
(整体框架, 关键设计 1-3, 关键发现)."""
import json
import math
import os

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def bf16_bits(x) -> np.ndarray:
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def from_bits(u) -> np.ndarray:
    u = np.asarray(u, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def rand_bits(rng, shape, s=1.0):
    return bf16_bits(rng.standard_normal(shape) * s)


# ----------------------------------------------------------------- page figure
def test_storage_ratio_matches_page(ora):
    """关键发现: ~90% KV-cache compression at 128K with g=16, w=1024."""
    fig = json.load(open(os.path.join(HERE, "golden", "page_figures.json")))
    L, g, w = fig["context_tokens"], fig["group_size"], fig["window"]
    m = ora.num_groups(L, g, w)
    kept = m + (L - m * g)                  # representatives + window rows
    assert kept == 9152
    reduction = 1.0 - kept / L
    assert reduction >= fig["kv_cache_reduction"]
    assert round(reduction, 1) == pytest.approx(fig["kv_cache_reduction"], abs=0.05)
    # at 32K the same rule keeps 3008 of 32768 rows
    m32 = ora.num_groups(32768, 16, 1024)
    assert m32 + (32768 - m32 * 16) == 3008


def test_num_groups_edge_cases(ora):
    assert ora.num_groups(100, 16, 1024) == 0      # L < w: nothing condensed
    assert ora.num_groups(1024, 16, 1024) == 0     # L == w
    assert ora.num_groups(1039, 16, 1024) == 0     # fewer than g leftover
    assert ora.num_groups(1040, 16, 1024) == 1
    assert ora.num_groups(4096, 16, 1024) == 192


# ------------------------------------------------ absorbed == decompressed MHA
def decompressed_mha(c, kr, q_nope, q_rope, w_uk, w_uv, scale):
    """Textbook multi-head attention with per-head K/V decompressed from the
    latent: K_h = [W_UK,h^T c || k^R], V_h = W_UV,h^T c."""
    H = q_nope.shape[0]
    out = []
    for h in range(H):
        K = np.concatenate([c @ w_uk[h], kr], axis=1)       # [L, dn+dr]
        V = c @ w_uv[h]                                       # [L, dv]
        qh = np.concatenate([q_nope[h], q_rope[h]])
        z = scale * (K @ qh)
        p = np.exp(z - z.max())
        p /= p.sum()
        out.append(p @ V)
    return np.stack(out)


@pytest.mark.parametrize("L", [1, 7, 37])
def test_absorbed_mla_equals_decompressed(ora, L):
    rng = np.random.default_rng(1)
    H, dc, dn, dr, dv = 4, 16, 8, 8, 6
    # integer-valued projections keep q_lat = W_UK q_nope exact in bf16
    w_uk = rng.integers(-2, 3, size=(H, dc, dn)) / 4.0
    q_nope = rng.integers(-3, 4, size=(H, dn)).astype(np.float64)
    q_lat = np.einsum("hkn,hn->hk", w_uk, q_nope)
    assert np.array_equal(from_bits(bf16_bits(q_lat)), q_lat)
    q_rope_b = rand_bits(rng, (H, dr), 0.5)
    cache = rand_bits(rng, (1, L, dc + dr))
    w_uv = rand_bits(rng, (H, dc, dv), 0.3)
    q = np.concatenate([bf16_bits(q_lat), q_rope_b], axis=1)[None]
    scale = 1.0 / math.sqrt(dn + dr)
    _, out = ora.mla_decode(cache, q, w_uv, scale, dr=dr)
    c = from_bits(cache[0, :, :dc])
    kr = from_bits(cache[0, :, dc:])
    ref = decompressed_mha(c, kr, q_nope, from_bits(q_rope_b), w_uk, from_bits(w_uv), scale)
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------ special cases
def small_case(rng, B=2, L=53, H=3, dc=8, dr=4, dv=5, g=4, peak=1.0):
    cache = rand_bits(rng, (B, L, dc + dr))
    q = rand_bits(rng, (B, H, dc + dr), peak)
    older = rand_bits(rng, (B, g - 1, H, dc + dr), peak)
    q_recent = np.concatenate([older, q[:, None]], axis=1)
    w_uv = rand_bits(rng, (H, dc, dv), 0.3)
    return cache, q, q_recent, w_uv


@pytest.mark.parametrize("L,w", [(23, 5), (40, 0), (9, 9)])
def test_g1_lca_equals_mla(ora, L, w):
    """With g = 1 every group is one token: alpha = 1, rep = the token itself,
    so LCA is exact MLA attention."""
    rng = np.random.default_rng(2)
    cache, q, _, w_uv = small_case(rng, L=L, g=1)
    q_recent = q[:, None]
    ol1, o1, anchor = ora.lca_decode(cache, q_recent, q, w_uv, 1, w, 0.3, dr=4)
    ol2, o2 = ora.mla_decode(cache, q, w_uv, 0.3, dr=4)
    np.testing.assert_allclose(ol1, ol2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    m = max(0, L - w)
    assert anchor.shape == (2, m)
    assert np.array_equal(anchor, np.broadcast_to(np.arange(m), (2, m)))


@pytest.mark.parametrize("L,w", [(30, 30), (30, 64)])
def test_window_covering_everything_is_mla(ora, L, w):
    rng = np.random.default_rng(3)
    cache, q, q_recent, w_uv = small_case(rng, L=L, g=4)
    ol1, o1, anchor = ora.lca_decode(cache, q_recent, q, w_uv, 4, w, 0.3, dr=4)
    ol2, o2 = ora.mla_decode(cache, q, w_uv, 0.3, dr=4)
    assert anchor.shape[1] == 0
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)


def test_equal_scores_give_plain_mean(ora):
    """q_recent = 0 makes every importance score 0: alpha = 1/g, the
    representative is the plain group mean and the anchor is the first token."""
    rng = np.random.default_rng(4)
    g, w, dc, dr = 4, 6, 8, 4
    cache, _, q_recent, _ = small_case(rng, L=31, g=g)
    q_recent = np.zeros_like(q_recent)
    r = ora.lca_condense(cache, q_recent, g, w, 0.3, dr=dr)
    m = (31 - w) // g
    assert r["rep_c"].shape == (2, m, dc)
    np.testing.assert_array_equal(r["alpha"], np.full((2, m, g), 1.0 / g))
    c = from_bits(cache[:, : m * g, :dc]).reshape(2, m, g, dc)
    np.testing.assert_allclose(r["rep_c"], c.mean(axis=2), rtol=0, atol=1e-15)
    assert np.array_equal(r["anchor"], np.broadcast_to(np.arange(m) * g, (2, m)))
    kfirst = from_bits(cache[:, : m * g : g, dc:])
    np.testing.assert_array_equal(r["rep_k"], kfirst)


def test_score_closed_form_one_hot_queries(ora):
    """One-hot recent queries reduce every dot product to one coordinate, so
    s_i = (1/H) sum_h scale * (1/g) sum_t v_th * row_i[k_th]; coordinates are
    chosen in both the latent and the rope part."""
    rng = np.random.default_rng(5)
    H, g, dc, dr, w = 2, 2, 8, 4, 3
    D = dc + dr
    cache = rand_bits(rng, (1, 19, D))
    coords = np.array([[1, 9], [6, 11]])          # k(t, h): t-major
    vals = np.array([[0.5, -2.0], [1.0, 4.0]])    # v(t, h)
    qr = np.zeros((1, g, H, D), np.float32)
    for t in range(g):
        for h in range(H):
            qr[0, t, h, coords[t, h]] = vals[t, h]
    scale = 0.25
    r = ora.lca_condense(cache, bf16_bits(qr), g, w, scale, dr=dr)
    rows = from_bits(cache[0])
    m = (19 - w) // g
    for j in range(m):
        for i in range(g):
            row = rows[j * g + i]
            s = sum(scale * sum(vals[t, h] * row[coords[t, h]] for t in range(g)) / g
                    for h in range(H)) / H
            assert r["score"][0, j, i] == pytest.approx(s, abs=1e-15)


def test_pooling_weights_are_group_softmax(ora):
    rng = np.random.default_rng(6)
    g, w = 16, 5
    cache, _, q_recent, _ = small_case(rng, L=200, g=g, peak=30.0)
    r = ora.lca_condense(cache, q_recent, g, w, 0.3, dr=4)
    a, s = r["alpha"], r["score"]
    np.testing.assert_allclose(a.sum(-1), 1.0, rtol=0, atol=1e-15)
    assert (a > 0).all()
    # alpha_i / alpha_k = exp(s_i - s_k)
    lr = np.log(a) - np.log(a[..., :1])
    np.testing.assert_allclose(lr, s - s[..., :1], rtol=0, atol=1e-12)
    # anchors: inside the group and at its highest score
    m = a.shape[1]
    j = np.arange(m)
    assert ((r["anchor"] >= j * g) & (r["anchor"] < (j + 1) * g)).all()
    loc = r["anchor"] - j * g
    assert np.array_equal(np.take_along_axis(s, loc[..., None], -1)[..., 0], s.max(-1))
    # the anchor's rope key is copied bit-exactly
    kr = from_bits(cache[:, :, -4:])
    np.testing.assert_array_equal(r["rep_k"], kr[np.arange(2)[:, None], r["anchor"]])


def test_anchor_takes_first_index_on_exact_tie(ora):
    rng = np.random.default_rng(7)
    g, w, D = 4, 0, 12
    cache = rand_bits(rng, (1, 8, D))
    cache[0, 1] = cache[0, 3]       # group 0: tokens 1 and 3 identical
    cache[0, 6] = cache[0, 5]       # group 1: tokens 5 and 6 identical
    q_recent = rand_bits(rng, (1, g, 2, D), 5.0)
    r = ora.lca_condense(cache, q_recent, g, w, 0.3, dr=4)
    s = r["score"][0]
    for j in range(2):
        best = np.flatnonzero(s[j] == s[j].max())
        assert r["anchor"][0, j] == j * g + best[0]


def test_representative_is_weighted_mean_minimiser(ora):
    """关键设计 1, Proposition 1: c_rep minimises sum_i alpha_i ||c_i - x||^2;
    so sum_i alpha_i (c_i - c_rep) = 0, the objective grows by exactly
    ||delta||^2 away from it, and c_rep lies in the group's coordinate hull."""
    rng = np.random.default_rng(8)
    g, w, dc = 16, 3, 8
    cache, _, q_recent, _ = small_case(rng, L=99, g=g, peak=20.0)
    r = ora.lca_condense(cache, q_recent, g, w, 0.3, dr=4)
    m = r["alpha"].shape[1]
    c = from_bits(cache[:, : m * g, :dc]).reshape(2, m, g, dc)
    a = r["alpha"][..., None]
    rep = r["rep_c"]
    np.testing.assert_allclose((a * (c - rep[:, :, None])).sum(2), 0.0, atol=1e-12)
    f = lambda x: (a * (c - x[:, :, None]) ** 2).sum((2, 3))
    for _ in range(3):
        d = rng.standard_normal(rep.shape) * 0.1
        np.testing.assert_allclose(f(rep + d) - f(rep), (d ** 2).sum(-1), rtol=1e-9, atol=1e-12)
    assert (rep >= c.min(2) - 1e-12).all() and (rep <= c.max(2) + 1e-12).all()


@pytest.mark.parametrize("L", [27, 30, 33])
def test_window_boundary_closed_form(ora, L):
    """整体框架 / 关键设计 3: with a zeroed history every representative has
    logit 0 and latent 0, so o = sum_win e^z c / (m + sum_win e^z) over the
    window rows m*g .. L-1 (leftover tokens included in the window)."""
    rng = np.random.default_rng(9)
    g, w, dc, dr = 4, 6, 8, 4
    m = (L - w) // g
    cache, q, q_recent, w_uv = small_case(rng, B=1, L=L, g=g)
    cache[0, : m * g] = 0
    scale = 0.4
    ol, _, _ = ora.lca_decode(cache, q_recent, q, w_uv, g, w, scale, dr=dr)
    win = from_bits(cache[0, m * g:])
    qq = from_bits(q[0])
    for h in range(q.shape[1]):
        e = np.exp(scale * (win @ qq[h]))
        ref = (e[:, None] * win[:, :dc]).sum(0) / (m + e.sum())
        np.testing.assert_allclose(ol[0, h], ref, rtol=0, atol=1e-13)


def test_up_projection_is_per_head(ora):
    """out_h = W_UV[h]^T o_lat,h with W_UV laid out [H][dc][dv]."""
    rng = np.random.default_rng(10)
    cache, q, _, w_uv = small_case(rng, L=12, dv=7)
    ol, out = ora.mla_decode(cache, q, w_uv, 0.3, dr=4)
    ref = np.einsum("bhk,hkv->bhv", ol, from_bits(w_uv))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


# ----------------------------------------------------------------- prefill
def prefill_case(rng, L=96, H=2, dc=8, dr=4, dv=3):
    cache = rand_bits(rng, (1, L, dc + dr))
    qpre = rand_bits(rng, (1, L, H, dc + dr), 3.0)
    w_uv = rand_bits(rng, (H, dc, dv), 0.3)
    return cache, qpre, w_uv


def test_prefill_blocks_before_window_are_causal_mla(ora):
    """A block that starts at or before w condenses nothing: each of its
    queries is causal MLA attention over rows 0..t."""
    rng = np.random.default_rng(11)
    g, w = 4, 16
    cache, qpre, w_uv = prefill_case(rng)
    ol, out, _ = ora.lca_prefill(cache, qpre, w_uv, 0, 20, g, w, 0.3, dr=4)
    for t in range(20):
        ol2, o2 = ora.mla_decode(cache[:, : t + 1], qpre[:, t], w_uv, 0.3, dr=4)
        np.testing.assert_allclose(ol[:, t], ol2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(out[:, t], o2, rtol=0, atol=1e-13)


def test_prefill_agrees_with_decode_inside_block(ora):
    """Query t of the block starting at t0 (t < t0+g-1) sees exactly what a
    decode step with L = t+1 sees when the recent queries are the block's:
    the same m = floor((t0-w)/g) groups, the same summary query and the
    window rows m*g..t.  (The block's last query is one token short of the
    next group boundary, where decode would condense one more group.)"""
    rng = np.random.default_rng(12)
    g, w = 4, 8
    cache, qpre, w_uv = prefill_case(rng)
    qs, ql = 40, 32
    ol, out, anc = ora.lca_prefill(cache, qpre, w_uv, qs, ql, g, w, 0.3, dr=4, want_anchor=True)
    for t0 in range(qs, qs + ql, g):
        qrec = qpre[:, t0 : t0 + g]
        for t in range(t0, t0 + g - 1):
            ol2, o2, a2 = ora.lca_decode(cache[:, : t + 1], qrec, qpre[:, t], w_uv, g, w, 0.3, dr=4)
            np.testing.assert_allclose(ol[:, t - qs], ol2, rtol=0, atol=1e-13)
            np.testing.assert_allclose(out[:, t - qs], o2, rtol=0, atol=1e-13)
            mb = (t0 - w) // g
            assert np.array_equal(anc[:, (t0 - qs) // g, :mb], a2)


def test_prefill_block_subset_matches_full(ora):
    rng = np.random.default_rng(13)
    g, w = 4, 8
    cache, qpre, w_uv = prefill_case(rng)
    ol, out, _ = ora.lca_prefill(cache, qpre, w_uv, 16, 64, g, w, 0.3, dr=4)
    ol2, out2, _ = ora.lca_prefill(cache, qpre, w_uv, 16, 64, g, w, 0.3, dr=4, blocks=[5, 9])
    for k in (5, 9):
        sl = slice(k * g - 16, k * g - 16 + g)
        np.testing.assert_array_equal(out2[:, sl], out[:, sl])
    assert np.isnan(out2[:, 0]).all()


def test_prefill_sparse_is_mla_over_anchor_rows(ora):
    """"纯稀疏" prefill: every representative is its anchor token's own row, so
    query t of block k is exact MLA attention over the cache rows
    [anchors of groups 0 .. m_k - 1 || m_k g .. t].  The anchors are the
    method's (the same argmax)."""
    rng = np.random.default_rng(14)
    g, w = 4, 8
    cache, qpre, w_uv = prefill_case(rng)
    qs, ql = 32, 40
    ol, out, anc = ora.lca_prefill(cache, qpre, w_uv, qs, ql, g, w, 0.3, dr=4, want_anchor=True,
                                   variant=ora.SPARSE)
    _, _, anc_lca = ora.lca_prefill(cache, qpre, w_uv, qs, ql, g, w, 0.3, dr=4, want_anchor=True)
    assert np.array_equal(anc, anc_lca)
    for t in range(qs, qs + ql):
        t0 = t - t % g
        mb = max(0, (t0 - w) // g)
        rows = np.concatenate([anc[0, (t0 - qs) // g, :mb], np.arange(mb * g, t + 1)])
        ol2, o2 = ora.mla_decode(cache[:, rows], qpre[:, t], w_uv, 0.3, dr=4)
        np.testing.assert_allclose(ol[:, t - qs], ol2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(out[:, t - qs], o2, rtol=0, atol=1e-13)


def test_prefill_pool_position_attends_pooled_keys(ora):
    """"纯池化（含位置）" prefill, on a cache built so that the pooled rows are
    known exactly.  The rows of each history group share everything but one
    RoPE coordinate. The block's queries are identical, and their two heads'
    dots cancel on that coordinate. So the group's importance scores are
    equal, alpha = 1/g, and the representative is the group's mean row.
    Attending stored bf16 representatives equal to those means must then
    give the block's outputs.  The method (anchor key = the group's first
    row, which is not the mean) gives something else."""
    rng = np.random.default_rng(15)
    g, w, dc, dr = 4, 8, 8, 4
    cache, qpre, w_uv = prefill_case(rng)
    t0 = 40
    m = (t0 - w) // g
    rows = from_bits(cache).copy()
    for j in range(m):
        rows[0, j * g:(j + 1) * g] = rows[0, j * g]
        rows[0, j * g:(j + 1) * g, dc + 2] = rng.integers(-3, 4, size=g)
    cache = bf16_bits(rows)
    q = np.zeros((2, dc + dr))
    q[0, dc + 2] = 1.0
    q[1, 0], q[1, dc + 2] = 1.0, -1.0
    qpre = qpre.copy()
    qpre[0, t0:t0 + g] = bf16_bits(q)
    pooled = from_bits(cache)[0, :m * g].reshape(m, g, dc + dr).mean(axis=1)
    rep = bf16_bits(pooled)[None]
    assert np.array_equal(from_bits(rep)[0], pooled)
    ol, out, _ = ora.lca_prefill(cache, qpre, w_uv, t0, g, g, w, 0.3, dr=dr, variant=ora.POOL_POSITION)
    ol_m, _, _ = ora.lca_prefill(cache, qpre, w_uv, t0, g, g, w, 0.3, dr=dr)
    for t in range(t0, t0 + g - 1):
        ol2, o2 = ora.lca_attend_reps(cache[:, :t + 1], rep, qpre[:, t], w_uv, g, w, 0.3, dr=dr)
        np.testing.assert_allclose(ol[:, t - t0], ol2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(out[:, t - t0], o2, rtol=0, atol=1e-13)
        assert not np.allclose(ol_m[:, t - t0], ol2, rtol=0, atol=1e-6)


# ----------------------------------------------------------------- stored representatives
def stored_case(rng, B=2, L=61, H=3, dc=8, dr=4, dv=5, peak=3.0):
    cache = rand_bits(rng, (B, L, dc + dr))
    q_all = rand_bits(rng, (B, L, H, dc + dr), peak)
    w_uv = rand_bits(rng, (H, dc, dv), 0.3)
    return cache, q_all, w_uv


def test_stored_with_identical_queries_is_recompute(ora):
    """一句话总结 / 关键发现 (kept representatives): when every position has the
    same query, every group's exit-time summary query is that query, so the
    stored reading equals recomputing all groups with it."""
    rng = np.random.default_rng(21)
    cache, q_all, w_uv = stored_case(rng)
    q_all[:] = q_all[:, :1]                      # one query everywhere
    g, w = 4, 9
    ol1, o1, a1 = ora.lca_decode_stored(cache, q_all, w_uv, g, w, 0.3, dr=4)
    L = cache.shape[1]
    q_recent = np.ascontiguousarray(q_all[:, L - g:L])
    ol2, o2, a2 = ora.lca_decode(cache, q_recent, np.ascontiguousarray(q_all[:, L - 1]), w_uv, g, w,
                                 0.3, dr=4)
    assert ora.num_groups(L, g, w) == 13
    assert np.array_equal(a1, a2)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(ol1, ol2, rtol=0, atol=1e-13)


def test_stored_window_covering_everything_is_mla(ora):
    rng = np.random.default_rng(22)
    cache, q_all, w_uv = stored_case(rng, L=30)
    ol1, o1, a1 = ora.lca_decode_stored(cache, q_all, w_uv, 4, 30, 0.3, dr=4)
    ol2, o2 = ora.mla_decode(cache, np.ascontiguousarray(q_all[:, -1]), w_uv, 0.3, dr=4)
    assert a1.shape[1] == 0
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)


def test_stored_single_group_is_the_exit_step_condensation(ora):
    """At L = w + g exactly one group has left the window, at this very step,
    so the stored reading and the recompute reading coincide."""
    rng = np.random.default_rng(23)
    g, w = 4, 10
    L = w + g
    cache, q_all, w_uv = stored_case(rng, L=L)
    ol1, o1, a1 = ora.lca_decode_stored(cache, q_all, w_uv, g, w, 0.3, dr=4)
    ol2, o2, a2 = ora.lca_decode(cache, np.ascontiguousarray(q_all[:, L - g:L]),
                                 np.ascontiguousarray(q_all[:, L - 1]), w_uv, g, w, 0.3, dr=4)
    assert a1.shape == (2, 1)
    assert np.array_equal(a1, a2)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)


def test_stored_anchors_are_frozen_exit_time_condensations(ora):
    """Group j's anchor is the argmax under the summary query of the step
    where it left the window (cache length w + g (j+1)), whatever the
    current length; different queries per position make that differ from the
    recompute reading."""
    rng = np.random.default_rng(24)
    g, w = 4, 6
    cache, q_all, w_uv = stored_case(rng, L=71, peak=20.0)
    L = cache.shape[1]
    _, _, a_now = ora.lca_decode_stored(cache, q_all, w_uv, g, w, 0.3, dr=4)
    m = ora.num_groups(L, g, w)
    assert a_now.shape == (2, m)
    for j in range(m):
        Lj = w + g * (j + 1)
        r = ora.lca_condense(np.ascontiguousarray(cache[:, :Lj]), np.ascontiguousarray(q_all[:, Lj - g:Lj]),
                             g, w, 0.3, dr=4)
        assert r["anchor"].shape[1] == j + 1
        assert np.array_equal(a_now[:, j], r["anchor"][:, j])
    # an earlier length keeps the same anchors for its groups
    Le = L - 13
    _, _, a_early = ora.lca_decode_stored(np.ascontiguousarray(cache[:, :Le]),
                                          np.ascontiguousarray(q_all[:, :Le]), w_uv, g, w, 0.3, dr=4)
    assert np.array_equal(a_early, a_now[:, :a_early.shape[1]])
    # and the recompute reading (current summary query for every group) differs somewhere
    _, _, a_re = ora.lca_decode(cache, np.ascontiguousarray(q_all[:, L - g:L]),
                                np.ascontiguousarray(q_all[:, L - 1]), w_uv, g, w, 0.3, dr=4)
    assert not np.array_equal(a_re, a_now)


# ----------------------------------------------------------------- ablations (消融实验)
def test_ablation_pool_position_pools_the_key(ora):
    """"纯池化（含位置）": the RoPE key is pooled with the same weights as the
    latent.  Latent and anchor are the method's; with equal scores the pooled
    key is the plain mean; in general it satisfies sum_i alpha_i (k_i - k_rep)
    = 0 (the stationarity of 关键设计 1, here for k^R)."""
    rng = np.random.default_rng(31)
    cache, _, q_recent, _ = small_case(rng, B=2, L=45, g=4, peak=3.0)
    g, w = 4, 5
    base = ora.lca_condense(cache, q_recent, g, w, 0.3, dr=4)
    pp = ora.lca_condense(cache, q_recent, g, w, 0.3, dr=4, variant=ora.POOL_POSITION)
    assert np.array_equal(pp["rep_c"], base["rep_c"])
    assert np.array_equal(pp["anchor"], base["anchor"])
    kr = from_bits(cache)[..., 8:]
    m = base["anchor"].shape[1]
    groups = kr[:, :m * g].reshape(2, m, g, 4)
    resid = np.einsum("bjg,bjgk->bjk", pp["alpha"], groups - pp["rep_k"][:, :, None, :])
    np.testing.assert_allclose(resid, 0.0, atol=1e-13)
    assert not np.allclose(pp["rep_k"], base["rep_k"])
    zero = np.zeros_like(q_recent)
    eq = ora.lca_condense(cache, zero, g, w, 0.3, dr=4, variant=ora.POOL_POSITION)
    np.testing.assert_allclose(eq["rep_k"], groups.mean(axis=2), rtol=0, atol=1e-15)


def test_ablation_sparse_keeps_the_anchor_row(ora):
    """"纯稀疏": the representative is the most important token's own row."""
    rng = np.random.default_rng(32)
    cache, _, q_recent, _ = small_case(rng, B=2, L=45, g=4, peak=3.0)
    g, w = 4, 5
    base = ora.lca_condense(cache, q_recent, g, w, 0.3, dr=4)
    sp = ora.lca_condense(cache, q_recent, g, w, 0.3, dr=4, variant=ora.SPARSE)
    assert np.array_equal(sp["anchor"], base["anchor"])
    rows = from_bits(cache)
    for b in range(2):
        for j, a in enumerate(sp["anchor"][b]):
            assert np.array_equal(sp["rep_c"][b, j], rows[b, a, :8])
            assert np.array_equal(sp["rep_k"][b, j], rows[b, a, 8:])
    assert np.array_equal(sp["rep_k"], base["rep_k"])


# ------------------------------------------------- decode split along the cache
def _split_cases(L, g, w):
    m = max(0, (L - w) // g)
    return [[0, L], [0, g, L], [0, m * g, L], [0, 2 * g, 3 * g, m * g - g, L], [0, g, 2 * g, m * g, L]]


@pytest.mark.parametrize("w", [6, 0])
def test_shard_merge_equals_unsplit_decode(ora, w):
    """整体框架: one softmax over [representatives || window].  Merging the
    shards' outputs by their log-sum-exp gives the unsplit decode for every
    cut, including a shard of one group and a shard of the window alone."""
    rng = np.random.default_rng(31)
    g, L = 4, 47
    cache, q, q_recent, w_uv = small_case(rng, L=L, g=g)
    ol, out, anchor = ora.lca_decode(cache, q_recent, q, w_uv, g, w, 0.3, dr=4)
    for cuts in _split_cases(L, g, w):
        parts = [ora.lca_decode_shard(cache, q_recent, q, g, w, 0.3, a, b, dr=4)
                 for a, b in zip(cuts[:-1], cuts[1:])]
        ol2, out2 = ora.combine_shards([p[0] for p in parts], [p[1] for p in parts], w_uv)
        np.testing.assert_allclose(ol2, ol, rtol=0, atol=1e-13)
        np.testing.assert_allclose(out2, out, rtol=0, atol=1e-13)
        assert np.array_equal(np.concatenate([p[2] for p in parts], axis=1), anchor)


def test_shard_of_one_window_row_closed_form(ora):
    """A shard holding a single row: softmax weight 1, so o is that row's
    latent and the log-sum-exp is its one logit z = scale (q_lat.c + q_rope.k)."""
    rng = np.random.default_rng(32)
    g, w, dc, dr, L = 4, 0, 8, 4, 4 * 5 + 1
    cache, q, q_recent, _ = small_case(rng, L=L, g=g)
    o, lse, anchor = ora.lca_decode_shard(cache, q_recent, q, g, w, 0.3, L - 1, L, dr=dr)
    assert anchor.shape == (2, 0)
    row = from_bits(cache[:, L - 1])                         # [B, dc+dr]
    qq = from_bits(q)                                        # [B, H, dc+dr]
    np.testing.assert_array_equal(o, np.broadcast_to(row[:, None, :dc], o.shape))
    z = 0.3 * np.einsum("bhk,bk->bh", qq, row)
    np.testing.assert_allclose(lse, z, rtol=0, atol=1e-14)


def test_shard_of_one_uniform_group_closed_form(ora):
    """q_recent = 0 gives a uniform pool: a shard of one group attends one
    representative, the group's mean latent with its first token's key."""
    rng = np.random.default_rng(33)
    g, w, dc, dr, L = 4, 6, 8, 4, 31
    cache, q, q_recent, _ = small_case(rng, L=L, g=g)
    q_recent = np.zeros_like(q_recent)
    j = 2
    o, lse, anchor = ora.lca_decode_shard(cache, q_recent, q, g, w, 0.3, j * g, (j + 1) * g, dr=dr)
    assert np.array_equal(anchor, np.full((2, 1), j * g))
    grp = from_bits(cache[:, j * g:(j + 1) * g])             # [B, g, dc+dr]
    rep_c, rep_k = grp[:, :, :dc].mean(axis=1), grp[:, 0, dc:]
    np.testing.assert_allclose(o, np.broadcast_to(rep_c[:, None], o.shape), rtol=0, atol=1e-15)
    qq = from_bits(q)
    z = 0.3 * (np.einsum("bhk,bk->bh", qq[..., :dc], rep_c) + np.einsum("bhk,bk->bh", qq[..., dc:], rep_k))
    np.testing.assert_allclose(lse, z, rtol=0, atol=1e-14)


def test_combine_of_two_shards_closed_form(ora):
    """Two partial outputs with log-sum-exps a and b merge with weights
    e^a / (e^a + e^b) and e^b / (e^a + e^b); W_UV is the identity on the
    first dv coordinates here."""
    B, H, dc, dv = 1, 2, 4, 4
    o1 = np.arange(B * H * dc, dtype=np.float64).reshape(B, H, dc)
    o2 = -np.ones((B, H, dc))
    a, b = np.array([[0.0, 2.0]]), np.array([[math.log(3.0), 2.0]])
    eye = np.zeros((H, dc, dv))
    eye[:, np.arange(dv), np.arange(dv)] = 1.0
    ol, out = ora.combine_shards([o1, o2], [a, b], bf16_bits(eye))
    np.testing.assert_allclose(ol[0, 0], 0.25 * o1[0, 0] + 0.75 * o2[0, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(ol[0, 1], 0.5 * o1[0, 1] + 0.5 * o2[0, 1], rtol=0, atol=1e-15)
    np.testing.assert_allclose(out, ol, rtol=0, atol=1e-15)
