"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on
the same seeded inputs, at the bar stated in tests/parity.py (anchors
bit-exact except near-ties, which are re-checked against the oracle run with
the GPU's anchors; outputs within max-abs 2e-2, mean-abs 2e-3 and relative
L2 1e-2).  Output buffers carry guard regions that must stay untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs
from parity import (MAX_ABS, MEAN_ABS, NEAR_TIE, REL_L2, Canaries, check_anchors, compare,  # noqa: F401
                    lca_decode_reference)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


def dev(inp):
    return (inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda())


def bits(inp):
    return bf16_bits(inp.cache), bf16_bits(inp.q_recent), bf16_bits(inp.q), bf16_bits(inp.w_uv)


# ---------------------------------------------------------------- MLA decode
@pytest.mark.parametrize("B,L", [(1, 1), (2, 63), (3, 64), (2, 65), (3, 1000), (2, 4096), (200, 300)])
def test_mla_decode_parity(B, L):
    inp = make_decode_inputs(B, L, seed=100 + L)
    cache, _, q, w_uv = dev(inp)
    cn = Canaries()
    o_lat = cn.empty((B, 16, 512), torch.float32)
    out = cn.empty((B, 16, 128), torch.float32)
    api.mla_decode_attn(cache, q, w_uv, inp.scale, out=out, o_lat=o_lat)
    torch.cuda.synchronize()
    cn.check("mla_decode_attn")
    c, _, qb, wb = bits(inp)
    ol_ref, out_ref = oracle.mla_decode(c, qb, wb, inp.scale)
    compare(o_lat.cpu().numpy(), ol_ref, "o_lat")
    compare(out.cpu().numpy(), out_ref, "out")


@pytest.mark.parametrize("peak", [1.0, 30.0])
def test_mla_decode_peaked(peak):
    inp = make_decode_inputs(2, 3000, seed=7, peak=peak)
    cache, _, q, w_uv = dev(inp)
    out = api.mla_decode_attn(cache, q, w_uv, inp.scale)
    torch.cuda.synchronize()
    c, _, qb, wb = bits(inp)
    _, out_ref = oracle.mla_decode(c, qb, wb, inp.scale)
    compare(out.cpu().numpy(), out_ref, "out")


# ---------------------------------------------------------------- condense
@pytest.mark.parametrize("B,L,peak", [(2, 4096, 1.0), (3, 1024 + 16 * 37 + 5, 1.0),
                                      (2, 1040, 1.0), (2, 1000, 1.0), (2, 4096, 30.0)])
def test_condense_parity(B, L, peak):
    inp = make_decode_inputs(B, L, seed=200 + L, peak=peak)
    cache, q_recent, _, _ = dev(inp)
    m = api.num_groups(L)
    cn = Canaries()
    anchor = cn.empty((B, m), torch.int32)
    alpha = cn.empty((B, m, 16), torch.float32)
    rep = cn.empty((B, m, 576), torch.bfloat16)
    api.lca_condense(cache, q_recent, scale=inp.scale, rep=rep, anchor=anchor, alpha=alpha)
    torch.cuda.synchronize()
    cn.check("lca_condense")
    c, qr, _, _ = bits(inp)
    r = oracle.lca_condense(c, qr, 16, 1024, inp.scale)
    if m == 0:
        return
    ga = anchor.cpu().numpy()
    check_anchors(ga, r["anchor"], r["score"])
    same = ga == r["anchor"]
    rep_f = rep.float().cpu().numpy()
    compare(rep_f[:, :, :512], r["rep_c"], "rep_c")
    compare(alpha.cpu().numpy(), r["alpha"], "alpha")
    # the anchor's RoPE key is copied bit for bit
    kr_bits = c[:, :, 512:]
    rep_bits = rep.view(torch.int16).cpu().numpy().view(np.uint16)
    exp_k = kr_bits[np.arange(B)[:, None], ga]
    assert np.array_equal(rep_bits[:, :, 512:], exp_k)
    assert same.mean() > 0.99


@pytest.mark.parametrize("variant", [1, 2])
def test_condense_ablation_variants(variant):
    """The two ablations of the page's 消融实验 table: pooling the RoPE key
    too (1) and keeping only the most important token's row (2); then the
    attention over those representatives."""
    B, L = 2, 1024 + 16 * 90 + 3
    inp = make_decode_inputs(B, L, seed=260 + variant, peak=10.0)
    cache, q_recent, q, w_uv = dev(inp)
    m = api.num_groups(L)
    anchor = torch.full((B, m), -1, dtype=torch.int32, device="cuda")
    rep = api.lca_condense(cache, q_recent, scale=inp.scale, anchor=anchor, variant=variant)
    o_lat = torch.empty(B, 16, 512, device="cuda")
    out = api.lca_decode_attn(cache, rep, q, w_uv, scale=inp.scale, o_lat=o_lat)
    torch.cuda.synchronize()
    c, qr, qb, wb = bits(inp)
    r = oracle.lca_condense(c, qr, 16, 1024, inp.scale, variant=variant)
    ga = anchor.cpu().numpy()
    check_anchors(ga, r["anchor"], r["score"])
    if not np.array_equal(ga, r["anchor"]):      # near-ties: the GPU's anchors, forced
        r = oracle.lca_condense(c, qr, 16, 1024, inp.scale, variant=variant, anchor_in=ga)
    rep_bits = rep.view(torch.int16).cpu().numpy().view(np.uint16)
    rows = c[np.arange(B)[:, None], ga]                 # the GPU's anchor rows
    if variant == 2:
        assert np.array_equal(rep_bits, rows)           # whole row, bit for bit
    else:
        rep_f = rep.float().cpu().numpy()
        compare(rep_f[:, :, :512], r["rep_c"], "rep_c (pool position)")
        compare(rep_f[:, :, 512:], r["rep_k"], "rep_k (pooled)")
    ol_ref, out_ref = oracle.lca_attend_reps(c, rep_bits, qb, wb, 16, 1024, inp.scale)
    compare(o_lat.cpu().numpy(), ol_ref, "o_lat")
    compare(out.cpu().numpy(), out_ref, "out")


# ---------------------------------------------------------------- attention over stored reps
@pytest.mark.parametrize("B,L", [(2, 4096), (3, 1024 + 16 * 70 + 9), (2, 1040), (2, 700)])
def test_decode_attn_over_stored_reps(B, L):
    inp = make_decode_inputs(B, L, seed=300 + L)
    cache, _, q, w_uv = dev(inp)
    c, qr, qb, wb = bits(inp)
    m = api.num_groups(L)
    # representatives come from the oracle's condensation, stored as bf16 rows
    r = oracle.lca_condense(c, qr, 16, 1024, inp.scale)
    rep_rows = np.concatenate([r["rep_c"], r["rep_k"]], axis=2).astype(np.float32)
    rep_t = torch.from_numpy(rep_rows).to(torch.bfloat16)
    rep_bits = bf16_bits(rep_t)
    o_lat = torch.empty(B, 16, 512, device="cuda")
    out = api.lca_decode_attn(cache, rep_t.cuda() if m > 0 else None, q, w_uv, scale=inp.scale,
                              o_lat=o_lat)
    torch.cuda.synchronize()
    ol_ref, out_ref = oracle.lca_attend_reps(c, rep_bits, qb, wb, 16, 1024, inp.scale)
    compare(o_lat.cpu().numpy(), ol_ref, "o_lat")
    compare(out.cpu().numpy(), out_ref, "out")


# ---------------------------------------------------------------- fused LCA decode
@pytest.mark.parametrize("B,L,peak", [
    (2, 4096, 1.0),
    (2, 1024 + 16 * 14 + 7, 1.0),     # partial last history tile, ragged window
    (3, 1040, 1.0),                   # one group
    (2, 1000, 1.0),                   # nothing condensed (L < w)
    (1, 5000, 30.0),
    (5, 2100, 30.0),
    (70, 1100, 1.0),                  # more rows than one combine CTA holds
    # more sequences than SMs: a CTA's split-L piece spans several sequences
    (300, 1040, 1.0),                 # one group each, 17 tiles per sequence
    (200, 700, 1.0),                  # nothing condensed, one tile per sequence
    (150, 1024 + 16 * 16, 30.0),      # exactly one full history tile
])
def test_lca_decode_fused_parity(B, L, peak):
    inp = make_decode_inputs(B, L, seed=400 + L, peak=peak)
    cache, q_recent, q, w_uv = dev(inp)
    m = api.num_groups(L)
    cn = Canaries()
    anchor = cn.empty((B, m), torch.int32)
    o_lat = cn.empty((B, 16, 512), torch.float32)
    out = cn.empty((B, 16, 128), torch.float32)
    api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, out=out, o_lat=o_lat, anchor=anchor)
    torch.cuda.synchronize()
    cn.check("lca_decode")
    c, qr, qb, wb = bits(inp)
    ol_ref, out_ref, _, _ = lca_decode_reference(c, qr, qb, wb, anchor.cpu().numpy(), inp.scale)
    compare(o_lat.cpu().numpy(), ol_ref, "o_lat")
    compare(out.cpu().numpy(), out_ref, "out")


@pytest.mark.parametrize("where", ["window", "history"])
def test_reference_max_rescale(where):
    """A row placed late in the sequence whose logit dwarfs everything before
    it forces the online softmax to move its reference maximum and rescale the
    accumulated output (both for a window row and for a condensed group)."""
    B, L = 2, 20000
    inp = make_decode_inputs(B, L, seed=21)
    for b in range(B):
        qv = inp.q[b, 0].float()
        row = (qv / qv.norm() * 300.0).to(torch.bfloat16)
        pos = L - 300 if where == "window" else 16 * 900 + 3
        if where == "history":
            inp.cache[b, 16 * 900: 16 * 901] = row
        inp.cache[b, pos] = row
    cache, q_recent, q, w_uv = dev(inp)
    o_lat = torch.empty(B, 16, 512, device="cuda")
    anchor = torch.empty(B, api.num_groups(L), dtype=torch.int32, device="cuda")
    out = api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, o_lat=o_lat, anchor=anchor)
    mla = api.mla_decode_attn(cache, q, w_uv, inp.scale)
    torch.cuda.synchronize()
    c, qr, qb, wb = bits(inp)
    ol_ref, out_ref, _, _ = lca_decode_reference(c, qr, qb, wb, anchor.cpu().numpy(), inp.scale)
    compare(o_lat.cpu().numpy(), ol_ref, "o_lat")
    compare(out.cpu().numpy(), out_ref, "out")
    _, mla_ref = oracle.mla_decode(c, qb, wb, inp.scale)
    compare(mla.cpu().numpy(), mla_ref, "mla out")


def test_reference_max_rescale_on_consecutive_tiles():
    """Twenty consecutive 64-row tiles, each holding a group whose logit tops
    everything before it by more than the rescale threshold: the reference
    maximum moves, and O is rescaled, on every one of them, back to back
    (and across the CTAs' split points of the longer sequence)."""
    B, L = 2, 30000
    inp = make_decode_inputs(B, L, seed=22)
    for b in range(B):
        # the logit grows through the RoPE key alone (the latents stay O(1)):
        # q_rope . k = |q_rope| a, a step of ~11 in log2 units per tile
        qr0 = inp.q[b, 0, 512:].float()
        for k in range(20):
            key = (qr0 / qr0.norm() * (760.0 + 330.0 * k)).to(torch.bfloat16)
            j = 4 * (300 + k)                  # one group in each of tiles 300..319
            inp.cache[b, 16 * j: 16 * (j + 1), 512:] = key
    cache, q_recent, q, w_uv = dev(inp)
    o_lat = torch.empty(B, 16, 512, device="cuda")
    anchor = torch.empty(B, api.num_groups(L), dtype=torch.int32, device="cuda")
    out = api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, o_lat=o_lat, anchor=anchor)
    mla = api.mla_decode_attn(cache, q, w_uv, inp.scale)
    torch.cuda.synchronize()
    c, qr, qb, wb = bits(inp)
    ol_ref, out_ref, _, _ = lca_decode_reference(c, qr, qb, wb, anchor.cpu().numpy(), inp.scale)
    compare(o_lat.cpu().numpy(), ol_ref, "o_lat")
    compare(out.cpu().numpy(), out_ref, "out")
    _, mla_ref = oracle.mla_decode(c, qb, wb, inp.scale)
    compare(mla.cpu().numpy(), mla_ref, "mla out")


def test_q_recent_slot_order_is_irrelevant():
    """The summary query is the mean of the g recent queries, so a ring
    buffer (any rotation or order of the slots) gives the same decode up to
    the fp32 summation order."""
    inp = make_decode_inputs(3, 7000, seed=23, peak=10.0)
    cache, q_recent, q, w_uv = dev(inp)
    ring = torch.roll(q_recent, shifts=5, dims=1).contiguous()
    perm = q_recent[:, torch.randperm(16, generator=torch.Generator().manual_seed(3))].contiguous()
    outs = [api.lca_decode(cache, qr, q, w_uv, scale=inp.scale) for qr in (q_recent, ring, perm)]
    torch.cuda.synchronize()
    c, qr, qb, wb = bits(inp)
    _, out_ref, _ = oracle.lca_decode(c, qr, qb, wb, 16, 1024, inp.scale)
    for o in outs:
        compare(o.cpu().numpy(), out_ref, "out")
        a, b = o.double().cpu().numpy(), outs[0].double().cpu().numpy()
        assert np.linalg.norm(a - b) / np.linalg.norm(b) <= 1e-3


def test_fused_equals_condense_then_attend():
    """The fused pass and condense -> attend over stored reps agree up to the
    bf16 rounding of stored representatives."""
    inp = make_decode_inputs(2, 6000, seed=11, peak=5.0)
    cache, q_recent, q, w_uv = dev(inp)
    a = api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale)
    rep = api.lca_condense(cache, q_recent, scale=inp.scale)
    b = api.lca_decode_attn(cache, rep, q, w_uv, scale=inp.scale)
    torch.cuda.synchronize()
    compare(a.cpu().numpy(), b.cpu().numpy(), "fused vs two-pass")


def test_g1_is_mla():
    inp = make_decode_inputs(2, 2000, seed=12)
    cache, q_recent, q, w_uv = dev(inp)
    a = api.lca_decode(cache, q_recent[:, :1].contiguous(), q, w_uv, g=1, scale=inp.scale)
    b = api.mla_decode_attn(cache, q, w_uv, inp.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_batch_split_invariance():
    """A sequence's result does not depend on how the split-L work is spread
    over CTAs (B=1 versus inside a batch of 5).  Different split points give
    different reference maxima, so the bf16-rounded attention weights differ
    at the 2^-9 level; o_lat must agree to that level, out (after the bf16
    rounding of o_lat) to the suite's relative bound."""
    inp = make_decode_inputs(5, 9000, seed=13)
    cache, q_recent, q, w_uv = dev(inp)
    ol_full = torch.empty(5, 16, 512, device="cuda")
    ol_one = torch.empty(1, 16, 512, device="cuda")
    full = api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, o_lat=ol_full)
    one = api.lca_decode(cache[3:4].contiguous(), q_recent[3:4].contiguous(), q[3:4].contiguous(),
                         w_uv, scale=inp.scale, o_lat=ol_one)
    torch.cuda.synchronize()
    a, b = ol_full[3].double().cpu().numpy(), ol_one[0].double().cpu().numpy()
    assert np.linalg.norm(a - b) / np.linalg.norm(b) <= 2e-3
    compare(full[3].cpu().numpy(), one[0].cpu().numpy(), "out split invariance")


# ---------------------------------------------------------------- full-size workloads, sampled
def full_size_check(B, L, sample, with_mla=False):
    inp = make_decode_inputs(B, L, seed=0)
    cache, q_recent, q, w_uv = dev(inp)
    m = api.num_groups(L)
    cn = Canaries()
    anchor = cn.empty((B, m), torch.int32)
    out = cn.empty((B, 16, 128), torch.float32)
    api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, out=out, anchor=anchor)
    mla = api.mla_decode_attn(cache, q, w_uv, inp.scale) if with_mla else None
    torch.cuda.synchronize()
    cn.check("lca_decode")
    sl = list(sample)
    c = bf16_bits(inp.cache[sl])
    qr = bf16_bits(inp.q_recent[sl])
    qb = bf16_bits(inp.q[sl])
    wb = bf16_bits(inp.w_uv)
    _, out_ref, _, nt = lca_decode_reference(c, qr, qb, wb, anchor.cpu().numpy()[sl], inp.scale)
    compare(out.cpu().numpy()[sl], out_ref, "out")
    assert nt <= max(3, len(sl) * m // 1000)
    if with_mla:
        _, mla_ref = oracle.mla_decode(c, qb, wb, inp.scale)
        compare(mla.cpu().numpy()[sl], mla_ref, "mla out")


def test_full_decode_b32_l32k_sampled():
    full_size_check(32, 32768, [0, 17, 31])


def test_full_decode_b8_l128k_with_mla_sampled():
    full_size_check(8, 131072, [0, 7], with_mla=True)


def test_full_decode_b1_l1m():
    full_size_check(1, 1 << 20, [0])


def test_full_decode_b1_l4k():
    full_size_check(1, 4096, [0], with_mla=True)
