"""Planted argmax near-ties on the GPU (inputs from tests/near_ties.py).

In every planted group the fp64 oracle picks the second row of a pair whose
scores differ by ~1e-13, while an fp32 score computation sees a tie and may
pick the first; both are valid anchors.  The two choices carry very
different RoPE keys (a CPU test shows the outputs then move by far more than
the tolerance), so these tests pass only if the GPU's outputs match the
oracle re-run with the GPU's own anchors: the forced-anchor path of the
parity checks is exercised on purpose, for the fused decode, the
condense-then-attend route, the split-L shards, the blockwise prefill and the
full-size 8 x 128K decode."""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs, make_prefill_inputs
from mla_latent_space_lca_b200.split_l import shard_bounds
from near_ties import G, plant_decode, plant_prefill
from parity import FORCED_RERUNS, Canaries, check_anchors, compare, lca_decode_reference
from test_gpu_prefill import check_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


def _planted(B, L, n, seed):
    inp = make_decode_inputs(B, L, seed=seed)
    cache, q_recent, q, planted = plant_decode(inp, n, seed=seed + 1)
    return inp, cache, q_recent, q, planted


def _decode(cache, q_recent, q, w_uv, scale):
    B, L, _ = cache.shape
    m = api.num_groups(L)
    cn = Canaries()
    anchor = cn.empty((B, m), torch.int32)
    o_lat = cn.empty((B, 16, 512), torch.float32)
    out = cn.empty((B, 16, 128), torch.float32)
    api.lca_decode(cache, q_recent, q, w_uv, scale=scale, out=out, o_lat=o_lat, anchor=anchor)
    torch.cuda.synchronize()
    cn.check("lca_decode")
    return out, o_lat, anchor


def test_fused_decode_with_planted_ties():
    inp, cache, q_recent, q, planted = _planted(2, 1024 + 16 * 300 + 5, 150, seed=81)
    out, o_lat, anchor = _decode(cache.cuda(), q_recent.cuda(), q.cuda(), inp.w_uv.cuda(), inp.scale)
    c, qr, qb, wb = bf16_bits(cache), bf16_bits(q_recent), bf16_bits(q), bf16_bits(inp.w_uv)
    ol_ref, out_ref, _, flips = lca_decode_reference(c, qr, qb, wb, anchor.cpu().numpy(), inp.scale)
    print(f"fused decode: {flips} near-tie flips of {len(planted)} planted groups")
    assert flips >= 1
    compare(o_lat.cpu().numpy(), ol_ref, "o_lat (GPU anchors)")
    compare(out.cpu().numpy(), out_ref, "out (GPU anchors)")


def test_condense_then_attend_with_planted_ties():
    inp, cache, q_recent, q, planted = _planted(2, 1024 + 16 * 200 + 9, 100, seed=83)
    cd, qrd = cache.cuda(), q_recent.cuda()
    m = api.num_groups(inp.L)
    anchor = torch.empty(2, m, dtype=torch.int32, device="cuda")
    rep = api.lca_condense(cd, qrd, scale=inp.scale, anchor=anchor)
    out = api.lca_decode_attn(cd, rep, q.cuda(), inp.w_uv.cuda(), scale=inp.scale)
    torch.cuda.synchronize()
    c, qr, qb, wb = bf16_bits(cache), bf16_bits(q_recent), bf16_bits(q), bf16_bits(inp.w_uv)
    r = oracle.lca_condense(c, qr, G, 1024, inp.scale)
    ga = anchor.cpu().numpy()
    flips, _ = check_anchors(ga, r["anchor"], r["score"])
    print(f"condense: {flips} near-tie flips of {len(planted)} planted groups")
    assert flips >= 1
    rf = oracle.lca_condense(c, qr, G, 1024, inp.scale, anchor_in=ga)
    rep_bits = rep.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(rep_bits[:, :, 512:], c[np.arange(2)[:, None], ga][:, :, 512:])
    compare(rep.float().cpu().numpy()[:, :, :512], rf["rep_c"], "rep_c")
    # the whole step against the oracle with the GPU's anchors (bf16 reps)
    _, out_ref, _, _ = lca_decode_reference(c, qr, qb, wb, ga, inp.scale)
    compare(out.cpu().numpy(), out_ref, "out (GPU anchors)")


def test_split_l_shards_with_planted_ties():
    inp, cache, q_recent, q, planted = _planted(2, 1024 + 16 * 300 + 5, 150, seed=85)
    B, L = inp.B, inp.L
    cd, qrd, qd, wd = cache.cuda(), q_recent.cuda(), q.cuda(), inp.w_uv.cuda()
    cuts = [0] + [b for _, b in shard_bounds(L, 3)]
    recs = torch.empty(len(cuts) - 1, api.shard_record_floats(B), device="cuda")
    anchors = []
    for s, (r0, r1) in enumerate(zip(cuts[:-1], cuts[1:])):
        m_s = max(0, (min(r1, api.num_groups(L) * 16) - r0) // 16)
        anc = torch.empty(B, max(m_s, 1), dtype=torch.int32, device="cuda")
        api.lca_decode_shard(cd[:, r0:r1].contiguous(), qrd, qd, L, r0, part=recs[s], anchor=anc)
        anchors.append((anc[:, :m_s], r0))
    out = api.lca_combine_shards(recs, wd, B)
    torch.cuda.synchronize()
    ga = np.concatenate([a.cpu().numpy() + r0 for a, r0 in anchors], axis=1)
    c, qr, qb, wb = bf16_bits(cache), bf16_bits(q_recent), bf16_bits(q), bf16_bits(inp.w_uv)
    _, out_ref, _, flips = lca_decode_reference(c, qr, qb, wb, ga, inp.scale)
    print(f"split-L: {flips} near-tie flips of {len(planted)} planted groups")
    assert flips >= 1
    compare(out.cpu().numpy(), out_ref, "merged out (GPU anchors)")


def test_prefill_with_planted_ties():
    B, L, w = 1, 16 * 200, 256
    inp = make_prefill_inputs(B, L, w=w, seed=87)
    inp.cache, inp.q, _ = plant_prefill(inp, 60, seed=88)
    before = FORCED_RERUNS["flips"]
    flips = check_prefill(inp, 0, L, w, blocks=[17, 50, 120, 170, 199], max_flip_frac=None)
    print(f"prefill: {flips} near-tie flips")
    assert flips >= 1 and FORCED_RERUNS["flips"] > before


def test_full_size_decode_b8_l128k_with_planted_ties():
    """The benchmark's 8 x 128K workload with 200 planted ties per sequence;
    two sequences checked against the oracle with the GPU's anchors."""
    inp, cache, q_recent, q, planted = _planted(8, 131072, 200, seed=0)
    out, o_lat, anchor = _decode(cache.cuda(), q_recent.cuda(), q.cuda(), inp.w_uv.cuda(), inp.scale)
    sl = [0, 7]
    c = bf16_bits(cache[sl])
    qr, qb, wb = bf16_bits(q_recent[sl]), bf16_bits(q[sl]), bf16_bits(inp.w_uv)
    ol_ref, out_ref, _, flips = lca_decode_reference(c, qr, qb, wb, anchor.cpu().numpy()[sl], inp.scale)
    print(f"8 x 128K: {flips} near-tie flips in sequences {sl}")
    assert flips >= 1
    compare(out.cpu().numpy()[sl], out_ref, "out (GPU anchors)")
    compare(o_lat.cpu().numpy()[sl], ol_ref, "o_lat (GPU anchors)")
