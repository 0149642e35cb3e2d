"""The planted near-tie inputs (tests/near_ties.py) do what the GPU tests
that use them rely on, checked on the oracle alone: the planted pair is a
near-tie under the stated rule, the oracle takes the second row, and the
other valid choice (the first row) moves the outputs far beyond the output
tolerance, so a parity check against the wrong one of the two references
would fail."""
import numpy as np

import oracle
from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs, make_prefill_inputs
from near_ties import G, plant_decode, plant_prefill
from parity import NEAR_TIE, REL_L2, rel_l2


def test_planted_decode_ties_are_valid_and_matter(ora):
    inp = make_decode_inputs(2, 1024 + 16 * 300 + 5, seed=71)
    cache, q_recent, q, planted = plant_decode(inp, 150, seed=72)
    c, qr, qb, wb = bf16_bits(cache), bf16_bits(q_recent), bf16_bits(q), bf16_bits(inp.w_uv)
    r = ora.lca_condense(c, qr, G, 1024, inp.scale)
    ol, out, a = ora.lca_decode(c, qr, qb, wb, G, 1024, inp.scale)
    forced = a.copy()
    for b, j in planted:
        s = r["score"][b, j]
        i1 = int(a[b, j]) - j * G
        assert i1 >= 1
        # the planted pair (i1 - 1, i1) is the group's top two, a near-tie
        assert 0 < s[i1] - s[i1 - 1] <= NEAR_TIE * np.abs(s).max()
        assert np.sort(s)[-2] == s[i1 - 1]
        forced[b, j] -= 1
    ol_f, out_f, _ = ora.lca_decode(c, qr, qb, wb, G, 1024, inp.scale, anchor_in=forced)
    assert rel_l2(out_f, out) > 5 * REL_L2
    assert rel_l2(ol_f, ol) > 5 * REL_L2


def test_planted_prefill_ties_are_valid(ora):
    B, L, w = 1, 16 * 200, 256
    inp = make_prefill_inputs(B, L, w=w, seed=73)
    cache, q, groups = plant_prefill(inp, 60, seed=74)
    c, qp = bf16_bits(cache), bf16_bits(q)
    ties = 0
    for k in (50, 120, 199):
        r = ora.lca_condense(np.ascontiguousarray(c[:, :G * k]), np.ascontiguousarray(qp[:, G * k:G * k + G]),
                             G, w, inp.scale)
        m = r["anchor"].shape[1]
        for j in groups:
            if j >= m:
                continue
            s = r["score"][0, j]
            top2 = np.argsort(s)[-2:]
            if abs(int(top2[0]) - int(top2[1])) == 1 and s[top2[1]] - s[top2[0]] <= NEAR_TIE * np.abs(s).max():
                ties += 1
    assert ties >= 20
