"""The C oracle against an independent brute-force restatement (tests/brute_force.py)
on tiny inputs in general position: group boundaries, window, anchors (exact
rational argmax), softmax weights, pooled representatives, attention output
and W_UV up-projection must agree.  Covers decode (the method, both
ablations, forced anchors), MLA, stored-representative decode and blockwise
prefill for L <= 64, g in {1, 2, 4, 16}, w in {0, 4, 8} and H in {1, 2, 16},
with the model widths scaled down (dc = 8, dr = 4, dv = 4)."""
import math
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import brute_force as bf

DC, DR, DV = 8, 4, 4
D = DC + DR
SCALE = 1.0 / math.sqrt(12.0)
TOL = 1e-11          # both sides are fp64; the brute force sums with math.fsum


def bits(shape, gen, std=1.0):
    t = (torch.randn(*shape, generator=gen, dtype=torch.float64) * std).to(torch.bfloat16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def close(a, b, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.abs(a - b).max() if a.size else 0.0
    assert err <= TOL * max(1.0, np.abs(b).max() if b.size else 1.0), f"{what}: max diff {err:.3e}"


def general_position(exact_groups, rel=1e-9):
    """True unless two different scores of a group lie within rel * max|s|
    of each other (fp64 could then order them differently from the exact
    rationals)."""
    for s in exact_groups:
        top = max(abs(x) for x in s) or Fraction(1)
        srt = sorted(s)
        for a, b in zip(srt, srt[1:]):
            if a != b and (b - a) < Fraction(rel) * top:
                return False
    return True


def decode_cases(n):
    rnd = random.Random(1234)
    out = []
    while len(out) < n:
        g = rnd.choice([1, 2, 4, 16])
        w = rnd.choice([0, 4, 8])
        H = rnd.choice([1, 2, 16])
        L = rnd.randint(1, 64)
        out.append((L, g, w, H, rnd.randrange(1 << 30)))
    return out


@pytest.fixture(scope="module")
def ora_mod(ora):
    return ora


@pytest.mark.parametrize("L,g,w,H,seed", decode_cases(24))
def test_decode_matches_brute_force(ora_mod, L, g, w, H, seed):
    gen = torch.Generator().manual_seed(seed)
    cache = bits((1, L, D), gen)
    q_recent = bits((1, g, H, D), gen, std=3.0)
    q = bits((1, H, D), gen)
    w_uv = bits((H, DC, DV), gen, std=0.3)
    ref = bf.decode(cache[0].tolist(), q_recent[0].tolist(), q[0].tolist(), w_uv.tolist(), DC, DR, g, w, SCALE)
    if not general_position(ref["exact_scores"]):
        pytest.skip("not in general position")
    m = ora_mod.num_groups(L, g, w)
    assert m == len(ref["groups"])
    assert ref["window_start"] == m * g
    assert all(e - s == g for s, e in ref["groups"])
    r = ora_mod.lca_condense(cache, q_recent, g, w, SCALE, dr=DR)
    assert r["anchor"][0].tolist() == ref["anchors"]
    close(r["alpha"][0], ref["alpha"] if m else np.zeros((0, g)), "alpha")
    close(r["rep_c"][0], ref["rep_c"] if m else np.zeros((0, DC)), "rep_c")
    close(r["rep_k"][0], ref["rep_k"] if m else np.zeros((0, DR)), "rep_k")
    o_lat, out, anchor = ora_mod.lca_decode(cache, q_recent, q, w_uv, g, w, SCALE, dr=DR)
    assert anchor[0].tolist() == ref["anchors"]
    close(o_lat[0], ref["o_lat"], "o_lat")
    close(out[0], ref["out"], "out")


@pytest.mark.parametrize("variant", [bf.POOL_POSITION, bf.SPARSE])
@pytest.mark.parametrize("seed", [5, 6, 7])
def test_ablations_match_brute_force(ora_mod, variant, seed):
    L, g, w, H = 60, 4, 8, 2
    gen = torch.Generator().manual_seed(seed)
    cache = bits((1, L, D), gen)
    q_recent = bits((1, g, H, D), gen, std=3.0)
    ref = bf.decode(cache[0].tolist(), q_recent[0].tolist(), bits((H, D), gen).tolist(),
                    bits((H, DC, DV), gen).tolist(), DC, DR, g, w, SCALE, variant=variant)
    assert general_position(ref["exact_scores"])
    r = ora_mod.lca_condense(cache, q_recent, g, w, SCALE, dr=DR, variant=variant)
    assert r["anchor"][0].tolist() == ref["anchors"]
    close(r["rep_c"][0], ref["rep_c"], "rep_c")
    close(r["rep_k"][0], ref["rep_k"], "rep_k")


def test_forced_anchors_match_brute_force(ora_mod):
    """Forcing anchors other than the argmax changes exactly the
    representative keys, the same way on both sides."""
    L, g, w, H = 64, 4, 4, 2
    gen = torch.Generator().manual_seed(9)
    cache = bits((1, L, D), gen)
    q_recent = bits((1, g, H, D), gen, std=3.0)
    q = bits((1, H, D), gen)
    w_uv = bits((H, DC, DV), gen, std=0.3)
    m = ora_mod.num_groups(L, g, w)
    forced = [j * g + (j * 7 + 1) % g for j in range(m)]
    ref = bf.decode(cache[0].tolist(), q_recent[0].tolist(), q[0].tolist(), w_uv.tolist(), DC, DR, g, w, SCALE,
                    forced=forced)
    o_lat, out, anchor = ora_mod.lca_decode(cache, q_recent, q, w_uv, g, w, SCALE, dr=DR,
                                            anchor_in=np.array([forced], np.int32))
    assert anchor[0].tolist() == forced == ref["anchors"]
    close(o_lat[0], ref["o_lat"], "o_lat")
    close(out[0], ref["out"], "out")
    free = ora_mod.lca_decode(cache, q_recent, q, w_uv, g, w, SCALE, dr=DR)
    assert np.abs(free[1] - out).max() > 1e-6      # forcing really changed the keys


def test_equal_scores_give_mean_and_first_index(ora_mod):
    """Zero recent queries make every importance score exactly 0: uniform
    weights, the plain mean, and the first index of every group."""
    L, g, w, H = 50, 16, 2, 16
    gen = torch.Generator().manual_seed(10)
    cache = bits((1, L, D), gen)
    q_recent = np.zeros((1, g, H, D), np.uint16)
    ref = bf.decode(cache[0].tolist(), q_recent[0].tolist(), bits((H, D), gen).tolist(),
                    bits((H, DC, DV), gen).tolist(), DC, DR, g, w, SCALE)
    assert ref["anchors"] == [j * g for j in range(len(ref["groups"]))]
    r = ora_mod.lca_condense(cache, q_recent, g, w, SCALE, dr=DR)
    assert r["anchor"][0].tolist() == ref["anchors"]
    close(r["alpha"][0], np.full((len(ref["groups"]), g), 1.0 / g), "alpha")
    close(r["rep_c"][0], ref["rep_c"], "rep_c")


@pytest.mark.parametrize("H", [1, 16])
def test_mla_matches_brute_force(ora_mod, H):
    gen = torch.Generator().manual_seed(11 + H)
    L = 40
    cache = bits((1, L, D), gen)
    q = bits((1, H, D), gen, std=2.0)
    w_uv = bits((H, DC, DV), gen)
    ref = bf.mla_decode(cache[0].tolist(), q[0].tolist(), w_uv.tolist(), DC, DR, SCALE)
    o_lat, out = ora_mod.mla_decode(cache, q, w_uv, SCALE, dr=DR)
    close(o_lat[0], ref["o_lat"], "o_lat")
    close(out[0], ref["out"], "out")


@pytest.mark.parametrize("L,g,w,H,variant", [(64, 4, 8, 2, bf.LCA), (48, 16, 4, 1, bf.LCA), (32, 2, 0, 2, bf.LCA),
                                             (64, 4, 4, 2, bf.POOL_POSITION), (64, 4, 4, 2, bf.SPARSE)])
def test_prefill_matches_brute_force(ora_mod, L, g, w, H, variant):
    gen = torch.Generator().manual_seed(L + g + w + H + variant)
    cache = bits((1, L, D), gen)
    qpre = bits((1, L, H, D), gen, std=3.0)
    w_uv = bits((H, DC, DV), gen, std=0.3)
    ref = bf.prefill(cache[0].tolist(), qpre[0].tolist(), w_uv.tolist(), DC, DR, g, w, SCALE, variant=variant)
    o_lat, out, anchor = ora_mod.lca_prefill(cache, qpre, w_uv, 0, L, g, w, SCALE, dr=DR, want_anchor=True,
                                             variant=variant)
    for k, a in enumerate(ref["anchors"]):
        assert anchor[0, k, :len(a)].tolist() == a, f"block {k}"
    close(o_lat[0].reshape(L, H, DC), ref["o_lat"], "o_lat")
    close(out[0].reshape(L, H, DV), ref["out"], "out")


def test_stored_decode_matches_brute_force(ora_mod):
    L, g, w, H = 64, 4, 8, 2
    gen = torch.Generator().manual_seed(21)
    cache = bits((1, L, D), gen)
    q_all = bits((1, L, H, D), gen, std=3.0)
    w_uv = bits((H, DC, DV), gen, std=0.3)
    ref = bf.decode_stored(cache[0].tolist(), q_all[0].tolist(), w_uv.tolist(), DC, DR, g, w, SCALE)
    o_lat, out, anchor = ora_mod.lca_decode_stored(cache, q_all, w_uv, g, w, SCALE, dr=DR)
    assert anchor[0].tolist() == ref["anchors"]
    close(o_lat[0], ref["o_lat"], "o_lat")
    close(out[0], ref["out"], "out")


def test_walk_agrees_with_floor_formula():
    """The positional enumeration reproduces m = floor((L - w) / g) (0 when
    L < w) on every small case."""
    for L in range(0, 80):
        for g in (1, 2, 4, 16):
            for w in (0, 4, 8, 17):
                groups, win0 = bf.walk_groups(L, g, w)
                m = max(0, (L - w) // g) if L >= w else 0
                assert len(groups) == m and win0 == m * g, (L, g, w)


def test_bf16_decoding():
    """Hand decoding of bf16 bits equals torch's widening."""
    vals = torch.tensor([0.0, -0.0, 1.0, -2.5, 3.140625, 1e-30, -7.5e-39, 65280.0, 2.0 ** -133],
                        dtype=torch.float32).to(torch.bfloat16)
    for b, v in zip(vals.view(torch.int16).numpy().view(np.uint16).tolist(), vals.float().tolist()):
        assert float(bf.bf16_fraction(b)) == v
